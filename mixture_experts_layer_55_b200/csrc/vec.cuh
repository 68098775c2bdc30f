// vec.cuh -- 16-byte vectors of the layer's element types, added into fp32
// accumulators (8 per vector: 8 bf16 or 4 fp32 elements) and packed back with
// one rounding.  Shared by the kernels that sum expert output rows.
#pragma once
#include "common.cuh"

namespace moe {

template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    MOE_DEVICE static void add(float (&a)[8], const uint4& v)
    {
        a[0] += __uint_as_float(v.x);
        a[1] += __uint_as_float(v.y);
        a[2] += __uint_as_float(v.z);
        a[3] += __uint_as_float(v.w);
    }
    MOE_DEVICE static void add_scaled(float (&a)[8], const uint4& v, float w)
    {
        a[0] = fmaf(w, __uint_as_float(v.x), a[0]);
        a[1] = fmaf(w, __uint_as_float(v.y), a[1]);
        a[2] = fmaf(w, __uint_as_float(v.z), a[2]);
        a[3] = fmaf(w, __uint_as_float(v.w), a[3]);
    }
    MOE_DEVICE static uint4 pack(const float (&a)[8])
    {
        return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                          __float_as_uint(a[3]));
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    MOE_DEVICE static void add(float (&a)[8], const uint4& v)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[2 * i] += __uint_as_float(w[i] << 16);
            a[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    MOE_DEVICE static void add_scaled(float (&a)[8], const uint4& v, float w)
    {
        const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[2 * i] = fmaf(w, __uint_as_float(x[i] << 16), a[2 * i]);
            a[2 * i + 1] = fmaf(w, __uint_as_float(x[i] & 0xffff0000u), a[2 * i + 1]);
        }
    }
    MOE_DEVICE static uint4 pack(const float (&a)[8])
    {
        return make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                          pack_bf16x2(a[6], a[7]));
    }
};

}  // namespace moe
