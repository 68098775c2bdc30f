// combine.cu -- weighted combine back to token order.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation": every
// (token, slot) adds its weighted expert output to the token's row
// (index_add_); section "Add a capacity limit": a dropped assignment adds
// nothing, so an all-dropped token gets zero.
//
// The routing weight is already applied by the down GEMM's epilogue, so the
// combine is a plain gather-sum: one warp per token, 16-byte vector loads of
// the token's K rows of y_perm, summed in slot order in fp32 and rounded once.
// No atomics: the result is deterministic.
#include "common.cuh"
#include "internal.h"

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
    MOE_DEVICE static uint4 pack(const float (&a)[8])
    {
        return make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                          pack_bf16x2(a[6], a[7]));
    }
};

constexpr int kCombineUnroll = 2;

template <typename ET>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ row_of,
                                                      uint4* __restrict__ y, int64_t T, int K,
                                                      int64_t vec_per_row, int64_t max_rows)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
         t += warps) {
        int32_t myrow = -1;
        if (lane < K) {
            myrow = row_of[t * K + lane];
            if (myrow >= max_rows) myrow = -1;  // never read outside y_perm
        }
        int32_t rows[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) rows[k] = __shfl_sync(0xffffffffu, myrow, k);
        for (int64_t v0 = lane; v0 < vec_per_row; v0 += 32 * kCombineUnroll) {
            float acc[kCombineUnroll][8];
#pragma unroll
            for (int u = 0; u < kCombineUnroll; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (k >= K || rows[k] < 0) continue;
                const uint4* src = y_perm + (int64_t)rows[k] * vec_per_row;
                uint4 v[kCombineUnroll];
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) {
                    const int64_t vi = v0 + 32 * u;
                    v[u] = vi < vec_per_row ? __ldg(src + vi) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) Vec<ET>::add(acc[u], v[u]);
            }
#pragma unroll
            for (int u = 0; u < kCombineUnroll; ++u) {
                const int64_t vi = v0 + 32 * u;
                if (vi < vec_per_row) y[t * vec_per_row + vi] = Vec<ET>::pack(acc[u]);
            }
        }
    }
}

cudaError_t launch_combine(const moe_config& c, const void* y_perm, const int32_t* row_of,
                           void* y, int64_t max_rows, cudaStream_t s)
{
    const int64_t row_bytes = (int64_t)c.D * (c.dtype == MOE_BF16 ? 2 : 4);
    const int64_t vpr = row_bytes / 16;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (c.T + 7) / 8;
    const int64_t cap = (int64_t)sms * 8;
    if (blocks > cap) blocks = cap;
    if (c.dtype == MOE_BF16)
        combine_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            static_cast<const uint4*>(y_perm), row_of, static_cast<uint4*>(y), c.T, c.K, vpr,
            max_rows);
    else
        combine_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(y_perm),
                                                               row_of, static_cast<uint4*>(y), c.T,
                                                               c.K, vpr, max_rows);
    return cudaGetLastError();
}

}  // namespace moe
