// combine.cu -- weighted combine back to token order.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation": every
// (token, slot) adds its weighted expert output to the token's row
// (index_add_); section "Add a capacity limit": a dropped assignment adds
// nothing, so an all-dropped token gets zero; section "Add a shared expert":
// a shared expert's output is added to the routed output.
//
// The routing weight is normally applied by the down GEMM's epilogue, so the
// combine is a plain gather-sum: 16-byte vector loads of the token's K rows of
// y_perm (a warp per token), summed in slot order in fp32 and rounded once.  The training forward
// keeps the expert outputs unweighted (the backward needs them), and then the
// combine multiplies each row by its slot's weight as it adds it.
// No atomics: the result is deterministic.
#include "common.cuh"
#include "internal.h"
#include "vec.cuh"

namespace moe {

// One warp per (token, part of the row) (grid-stride): lanes k < K read slot
// k's row (and weight), the warp broadcasts them, and each lane sums
// kCombineUnroll 16-byte vectors of its part of the token's output at a time
// (K x kCombineUnroll loads in flight), in slot order, in fp32, rounded once.
// A row is split into `parts` pieces only when the tokens alone are too few
// to occupy the GPU (decode); every element is summed the same way either
// way.  An out-of-range row is never read (the slot counts as dropped).
constexpr int kCombineUnroll = 4;
constexpr int kCombineWarps = 8;

template <typename ET, int KS, bool SPLIT>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const uint4* __restrict__ y_perm,
                                                                     const int32_t* __restrict__ row_of,
                                                                     const float* __restrict__ slot_w,
                                                                     const uint4* __restrict__ y_add,
                                                                     uint4* __restrict__ y, int64_t T, int K,
                                                                     int64_t vpr, int64_t max_rows, int parts,
                                                                     int64_t vpp)
{
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kCombineWarps;
    const int64_t items = SPLIT ? T * parts : T;
    for (int64_t item = (int64_t)blockIdx.x * kCombineWarps + (threadIdx.x >> 5); item < items;
         item += nw) {
        const int64_t t = SPLIT ? item / parts : item;
        const int64_t vbeg = SPLIT ? (item % parts) * vpp : 0;
        const int64_t vend = SPLIT ? (vbeg + vpp < vpr ? vbeg + vpp : vpr) : vpr;
        int32_t r = -1;
        float wk = 1.f;
        if (lane < K) {
            r = __ldg(row_of + t * K + lane);
            if (r >= max_rows) r = -1;  // never read outside y_perm
            if (slot_w && r >= 0) wk = __ldg(slot_w + t * K + lane);
        }
        int32_t rows[KS];
        float ws[KS];
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            rows[k] = __shfl_sync(0xffffffffu, r, k);
            ws[k] = __shfl_sync(0xffffffffu, wk, k);
        }
        for (int64_t v0 = vbeg + lane; v0 < vend; v0 += 32 * kCombineUnroll) {
            float acc[kCombineUnroll][8];
#pragma unroll
            for (int u = 0; u < kCombineUnroll; ++u) {
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
                const int64_t v = v0 + 32 * u;
                if (y_add && v < vend) Vec<ET>::add(acc[u], __ldg(y_add + t * vpr + v));  // shared expert first
            }
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                if (rows[k] < 0) continue;  // slot order; dropped or absent slots add nothing
                const uint4* src = y_perm + (int64_t)rows[k] * vpr;
                uint4 val[kCombineUnroll];
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) {
                    const int64_t v = v0 + 32 * u;
                    val[u] = v < vend ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kCombineUnroll; ++u) {
                    if (slot_w) Vec<ET>::add_scaled(acc[u], val[u], ws[k]);
                    else Vec<ET>::add(acc[u], val[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kCombineUnroll; ++u) {
                const int64_t v = v0 + 32 * u;
                if (v < vend) y[t * vpr + v] = Vec<ET>::pack(acc[u]);
            }
        }
    }
}

template <typename ET>
static void launch_combine_t(const moe_config& c, int64_t blocks, const void* y_perm,
                             const int32_t* row_of, const float* slot_w, const void* y_add, void* y,
                             int64_t vpr, int64_t max_rows, int parts, int64_t vpp, cudaStream_t s)
{
    const uint4* src = static_cast<const uint4*>(y_perm);
    const uint4* add = static_cast<const uint4*>(y_add);
    uint4* dst = static_cast<uint4*>(y);
    const unsigned g = (unsigned)blocks, nt = kCombineWarps * 32;
    if (parts > 1) {
        if (c.K <= 2)
            combine_kernel<ET, 2, true><<<g, nt, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr, max_rows, parts, vpp);
        else if (c.K <= 4)
            combine_kernel<ET, 4, true><<<g, nt, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr, max_rows, parts, vpp);
        else
            combine_kernel<ET, 8, true><<<g, nt, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr, max_rows, parts, vpp);
        return;
    }
    if (c.K <= 1)
        combine_kernel<ET, 1, false><<<g, nt, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr, max_rows, parts, vpp);
    else if (c.K == 2)
        combine_kernel<ET, 2, false><<<g, nt, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr, max_rows, parts, vpp);
    else if (c.K <= 4)
        combine_kernel<ET, 4, false><<<g, nt, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr, max_rows, parts, vpp);
    else
        combine_kernel<ET, 8, false><<<g, nt, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr, max_rows, parts, vpp);
}

cudaError_t launch_combine(const moe_config& c, const void* y_perm, const int32_t* row_of,
                           const float* slot_w, const void* y_add, void* y, int64_t max_rows,
                           cudaStream_t s)
{
    const int64_t row_bytes = (int64_t)c.D * (c.dtype == MOE_BF16 ? 2 : 4);
    const int64_t vpr = row_bytes / 16;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * 16;  // blocks of 8 warps
    // parts per row: with fewer tokens than warps of a full wave (decode), enough
    // parts to fill the GPU, each at least 32 x kCombineUnroll vectors (a whole
    // pass of the warp) and a multiple of 32 vectors
    int64_t parts = 1;
    if (c.T < (int64_t)sms * kCombineWarps) {
        parts = (cap * kCombineWarps + c.T - 1) / c.T;
        const int64_t max_parts = vpr / (32 * kCombineUnroll);
        if (parts > max_parts) parts = max_parts;
        if (parts < 1) parts = 1;
    }
    const int64_t vpp = ((vpr + parts - 1) / parts + 31) / 32 * 32;
    parts = (vpr + vpp - 1) / vpp;
    int64_t blocks = (c.T * parts + kCombineWarps - 1) / kCombineWarps;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (c.dtype == MOE_BF16)
        launch_combine_t<__nv_bfloat16>(c, blocks, y_perm, row_of, slot_w, y_add, y, vpr, max_rows,
                                        (int)parts, vpp, s);
    else
        launch_combine_t<float>(c, blocks, y_perm, row_of, slot_w, y_add, y, vpr, max_rows, (int)parts,
                                vpp, s);
    return cudaGetLastError();
}

}  // namespace moe
