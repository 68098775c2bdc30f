// ep.cu -- the data-movement steps of expert parallelism.
//
// "Lab: build a tiny MoE in PyTorch", "From local loop to expert
// parallelism": the distributed layer sorts the routed rows by the rank that
// owns their expert, exchanges the counts, moves the rows there (all-to-all),
// runs the owner's experts as one grouped problem, sends the results back
// (reverse all-to-all) and scatter-adds them at home -- the same mathematical
// output with different data movement.  "2.9 Mixture-of-Experts (MoE)
// Architectures", "Expert Parallelism: A Systems Preview": experts are
// sharded across devices (rank r holds a contiguous block of them).
//
// The local dispatch already orders rows expert-major, so the rows bound for
// one owner are contiguous and are sent as they are.  What arrives is ordered
// source-major ([from rank 0: its rows for my expert 0, 1, ...][from rank 1:
// ...]); the grouped GEMM wants expert-major.  These kernels compute that
// layout from the exchanged counts and move rows between the two orders.
#include "common.cuh"
#include "internal.h"

namespace moe {

// recv (W x EL) int32: rows arriving from source s for local expert e.
// Writes offsets (EL + 1, expert-major row offsets of the local experts),
// seg_src (W*EL + 1: first source-major position of segment (s, e), segments
// in source-major order) and seg_dst (W*EL: first expert-major row of that
// segment).  One block; W * EL <= 256.
__global__ void ep_layout_kernel(const int32_t* __restrict__ recv, int W, int EL, int64_t max_rows,
                                 int32_t* __restrict__ offsets, int32_t* __restrict__ seg_src,
                                 int32_t* __restrict__ seg_dst, int* status)
{
    __shared__ int32_t cnt[256];
    const int n = W * EL;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        int32_t c = recv[i];
        if (c < 0) {
            raise_flag(status, kFlagBounds, 700);
            c = 0;
        }
        cnt[i] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // expert-major: expert e's rows are its segments from sources 0..W-1 in order
        int64_t run = 0;
        for (int e = 0; e < EL; ++e) {
            offsets[e] = (int32_t)run;
            for (int s = 0; s < W; ++s) {
                seg_dst[s * EL + e] = (int32_t)run;
                run += cnt[s * EL + e];
            }
        }
        if (run > max_rows) {
            raise_flag(status, kFlagBounds, 701);
            run = max_rows;
        }
        offsets[EL] = (int32_t)run;
        // source-major: segment (s, e) follows all of source s-1's and s's experts < e
        int64_t pos = 0;
        for (int i = 0; i < n; ++i) {
            seg_src[i] = (int32_t)pos;
            pos += cnt[i];
        }
        seg_src[n] = (int32_t)(pos < max_rows ? pos : max_rows);
    }
}

// For every source-major position p < seg_src[n]: its segment by binary
// search, dst_of[p] = seg_dst[seg] + (p - seg_src[seg]) and src_of[dst] = p.
__global__ void ep_maps_kernel(const int32_t* __restrict__ seg_src, const int32_t* __restrict__ seg_dst,
                               int n, int64_t max_rows, int32_t* __restrict__ dst_of,
                               int32_t* __restrict__ src_of, int* status)
{
    __shared__ int32_t ss[257], sd[256];
    for (int i = threadIdx.x; i <= n; i += blockDim.x) ss[i] = seg_src[i];
    for (int i = threadIdx.x; i < n; i += blockDim.x) sd[i] = seg_dst[i];
    __syncthreads();
    const int64_t total = ss[n];
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < total;
         p += (int64_t)gridDim.x * blockDim.x) {
        int lo = 0, hi = n - 1;
        while (lo < hi) {  // last segment whose start is <= p (empty segments share starts)
            const int mid = (lo + hi + 1) >> 1;
            if (ss[mid] <= p) lo = mid;
            else hi = mid - 1;
        }
        while (lo + 1 < n && ss[lo + 1] <= p) ++lo;
        const int64_t d = (int64_t)sd[lo] + (p - ss[lo]);
        if (d < 0 || d >= max_rows) {
            raise_flag(status, kFlagBounds, 702);
            continue;
        }
        dst_of[p] = (int32_t)d;
        src_of[d] = (int32_t)p;
    }
}

// out[i] = in[idx[i]] for i < n, rows of vpr 16-byte vectors.  Consecutive
// threads move consecutive vectors of a row.
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ in,
                                                           const int32_t* __restrict__ idx,
                                                           uint4* __restrict__ out, int64_t n,
                                                           int64_t vpr, int64_t in_rows, int* status)
{
    const int64_t total = n * vpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / vpr, v = i - r * vpr;
        const int32_t s = __ldg(idx + r);
        if (s < 0 || s >= in_rows) {
            if (v == 0) raise_flag(status, kFlagBounds, 710);
            continue;
        }
        out[i] = __ldg(in + (int64_t)s * vpr + v);
    }
}

static int sm_count_ep()
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

cudaError_t launch_ep_layout(const int32_t* recv, int W, int EL, int64_t max_rows, int32_t* offsets,
                             int32_t* seg_src, int32_t* seg_dst, int32_t* dst_of, int32_t* src_of,
                             int* status, cudaStream_t s)
{
    ep_layout_kernel<<<1, 256, 0, s>>>(recv, W, EL, max_rows, offsets, seg_src, seg_dst, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int64_t blocks = (max_rows + 255) / 256;
    const int64_t cap = (int64_t)sm_count_ep() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    ep_maps_kernel<<<(unsigned)blocks, 256, 0, s>>>(seg_src, seg_dst, W * EL, max_rows, dst_of, src_of,
                                                    status);
    return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void* in, const int32_t* idx, void* out, int64_t n, int64_t row_bytes,
                                int64_t in_rows, int* status, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    const int64_t vpr = row_bytes / 16;
    int64_t blocks = (n * vpr + 255) / 256;
    const int64_t cap = (int64_t)sm_count_ep() * 16;
    if (blocks > cap) blocks = cap;
    permute_rows_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(in), idx,
                                                         static_cast<uint4*>(out), n, vpr, in_rows, status);
    return cudaGetLastError();
}

}  // namespace moe
