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
// y_perm, summed in slot order in fp32 and rounded once.  The training forward
// keeps the expert outputs unweighted (the backward needs them), and then the
// combine multiplies each row by its slot's weight as it adds it.
// No atomics: the result is deterministic.
#include "common.cuh"
#include "internal.h"
#include "vec.cuh"

namespace moe {

// Each thread produces VPT 16-byte vectors of the output, with KS >= K slots
// per token and VPT * KS = 8, so that about 8 loads are in flight per thread
// whatever K is: vectors i, i + G, ... of the flattened (T x vec_per_row)
// output, G = total threads.  row_of is shared by a row's threads through L1.
// Consecutive threads cover consecutive vectors of a row (coalesced).
template <typename ET, int KS>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ row_of,
                                                      const float* __restrict__ slot_w,
                                                      const uint4* __restrict__ y_add,
                                                      uint4* __restrict__ y, int64_t T, int K,
                                                      int64_t vec_per_row, int64_t max_rows)
{
    constexpr int VPT = 8 / KS;
    const int64_t n = T * vec_per_row;
    const int64_t G = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n; base += G * VPT) {
        uint4 vals[VPT][KS];
        int32_t rows[VPT][KS];
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
            const int64_t i = base + (int64_t)u * G;
            const int64_t t = i < n ? i / vec_per_row : 0, v = i - t * vec_per_row;
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                int32_t r = (i < n && k < K) ? __ldg(row_of + t * K + k) : -1;
                rows[u][k] = (r >= 0 && r < max_rows) ? r : -1;  // never read outside y_perm
            }
#pragma unroll
            for (int k = 0; k < KS; ++k)
                vals[u][k] = rows[u][k] >= 0 ? __ldg(y_perm + (int64_t)rows[u][k] * vec_per_row + v)
                                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
            const int64_t i = base + (int64_t)u * G;
            if (i >= n) break;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (y_add) Vec<ET>::add(acc, __ldg(y_add + i));  // shared expert output first
            const int64_t t = i / vec_per_row;
#pragma unroll
            for (int k = 0; k < KS; ++k)
                if (rows[u][k] >= 0) {  // slot order
                    if (slot_w) Vec<ET>::add_scaled(acc, vals[u][k], __ldg(slot_w + t * K + k));
                    else Vec<ET>::add(acc, vals[u][k]);
                }
            y[i] = Vec<ET>::pack(acc);
        }
    }
}

template <typename ET>
static void launch_combine_t(const moe_config& c, int64_t blocks, const void* y_perm,
                             const int32_t* row_of, const float* slot_w, const void* y_add, void* y,
                             int64_t vpr, int64_t max_rows, cudaStream_t s)
{
    const uint4* src = static_cast<const uint4*>(y_perm);
    const uint4* add = static_cast<const uint4*>(y_add);
    uint4* dst = static_cast<uint4*>(y);
    if (c.K <= 1)
        combine_kernel<ET, 1><<<(unsigned)blocks, 256, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr,
                                                                max_rows);
    else if (c.K == 2)
        combine_kernel<ET, 2><<<(unsigned)blocks, 256, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr,
                                                                max_rows);
    else if (c.K <= 4)
        combine_kernel<ET, 4><<<(unsigned)blocks, 256, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr,
                                                                max_rows);
    else
        combine_kernel<ET, 8><<<(unsigned)blocks, 256, 0, s>>>(src, row_of, slot_w, add, dst, c.T, c.K, vpr,
                                                                max_rows);
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
    const int vpt = c.K <= 1 ? 8 : c.K == 2 ? 4 : c.K <= 4 ? 2 : 1;
    int64_t blocks = (c.T * vpr + 256LL * vpt - 1) / (256LL * vpt);
    const int64_t cap = (int64_t)sms * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (c.dtype == MOE_BF16)
        launch_combine_t<__nv_bfloat16>(c, blocks, y_perm, row_of, slot_w, y_add, y, vpr, max_rows, s);
    else
        launch_combine_t<float>(c, blocks, y_perm, row_of, slot_w, y_add, y, vpr, max_rows, s);
    return cudaGetLastError();
}

}  // namespace moe
