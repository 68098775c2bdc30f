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
#include "vec.cuh"

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

// ------------------------------------------------ exchange over peer memory --
//
// The same exchange done by the layer's own kernels, with every rank's
// receive buffers mapped into every other rank's address space (CUDA IPC over
// NVLink).  The dispatch kernel reads each token row once and stores it
// straight into the owner's receive buffer at its expert-major row; the owner
// runs its grouped experts there; the combine kernel loads each kept slot's
// result from the owner's output buffer and adds it, weighted, at home.  That
// replaces the host read of the sizes, both all-to-alls and both
// permutations.  The only collectives left are an all-gather of the kept
// counts (world x E int32) before the dispatch and two stream-ordered
// barriers of the caller's communication library: after the dispatch (every
// row has arrived) and after the experts (every result is ready).
//
// Row of slot (t, k) in its owner's receive buffer.  Expert e (owner
// o = e / EL, local index e - o*EL) holds, in order, the rows of sources
// 0 .. world-1; source `rank`'s rows of e follow the other sources' before it:
//   seg_base[e] = sum_{o*EL <= e' < e} sum_s kept_all[s][e']
//               + sum_{s < rank} kept_all[s][e]
//   remote_row(t, k) = seg_base[e] + (row_of[t, k] - offsets[e])
// where row_of[t, k] - offsets[e] is the slot's rank among this source's kept
// rows of e (the local expert-major dispatch).
constexpr int kPeerMaxWorld = 64;
constexpr int kPeerMaxE = 256;

// seg_base (and own_base: the first part alone) of every expert, computed by
// the whole block from the gathered counts; negative counts raise the bounds
// flag and count as 0.
MOE_DEVICE void peer_segment_bases(const int32_t* __restrict__ kept_all, int W, int E, int EL, int rank,
                                   int32_t* tot, int32_t* own_base, int32_t* seg_base, int* status)
{
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t sum = 0, before = 0;
        for (int s = 0; s < W; ++s) {
            int32_t c = kept_all[(int64_t)s * E + e];
            if (c < 0) {
                raise_flag(status, kFlagBounds, 720);
                c = 0;
            }
            sum += c;
            if (s < rank) before += c;
        }
        tot[e] = sum;
        seg_base[e] = before;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int first = (e / EL) * EL;
        int32_t acc = 0;
        for (int j = first; j < e; ++j) acc += tot[j];
        own_base[e] = acc;
        seg_base[e] += acc;
    }
    __syncthreads();
}

// Slot (t, k) -> (owner, remote row), or owner -1 for a dropped slot; an
// out-of-range id, row or remote row raises the bounds flag and drops it.
MOE_DEVICE int peer_slot(const int32_t* __restrict__ ids, const int32_t* __restrict__ row_of,
                         const int32_t* offs, const int32_t* seg_base, int64_t slot, int E, int EL,
                         int64_t recv_rows, int64_t max_rows, int32_t* remote, int* status, int where)
{
    const int32_t r = row_of[slot];
    if (r < 0) return -1;
    const int32_t e = ids[slot];
    if (e < 0 || e >= E || r >= max_rows || r < offs[e] || r >= offs[e + 1]) {
        raise_flag(status, kFlagBounds, where);
        return -1;
    }
    const int64_t d = (int64_t)seg_base[e] + (r - offs[e]);
    if (d < 0 || d >= recv_rows) {
        raise_flag(status, kFlagBounds, where + 1);
        return -1;
    }
    *remote = (int32_t)d;
    return e / EL;
}

// One warp per token (grid-stride over tokens).  Lanes k < K place slot k
// (its owner and row in the owner's buffer; remote_row, the combine's map
// back) and the warp broadcasts them; then the lanes move the token row's
// 16-byte vectors, kUnroll loads in flight per lane, each stored to every
// kept slot's destination.  Block 0 also writes this rank's local offsets.
// Every thread ends with a system-scope fence, so its peer stores are
// visible before the barrier that follows the kernel.
constexpr int kPeerUnroll = 4;
constexpr int kPeerWarps = 8;

template <int KS>
__global__ void __launch_bounds__(kPeerWarps * 32) peer_dispatch_kernel(
    const uint4* __restrict__ x, const int32_t* __restrict__ ids, const int32_t* __restrict__ row_of,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ kept_all,
    uint4* const* __restrict__ recv_bufs, int64_t T, int K, int E, int EL, int W, int rank, int64_t vpr,
    int64_t recv_rows, int64_t max_rows, int32_t* __restrict__ local_offsets,
    int32_t* __restrict__ remote_row, int* status)
{
    __shared__ int32_t tot[kPeerMaxE], own[kPeerMaxE], seg[kPeerMaxE], offs[kPeerMaxE + 1];
    __shared__ uint4* bufs[kPeerMaxWorld];
    for (int i = threadIdx.x; i <= E; i += blockDim.x) offs[i] = offsets[i];
    for (int i = threadIdx.x; i < W; i += blockDim.x) bufs[i] = recv_bufs[i];
    peer_segment_bases(kept_all, W, E, EL, rank, tot, own, seg, status);
    if (blockIdx.x == 0)
        for (int j = threadIdx.x; j <= EL; j += blockDim.x) {
            const int e = rank * EL + (j < EL ? j : EL - 1);
            local_offsets[j] = j < EL ? own[e] : own[e] + tot[e];
        }
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kPeerWarps;
    for (int64_t t = (int64_t)blockIdx.x * kPeerWarps + (threadIdx.x >> 5); t < T; t += nw) {
        int o = -1;
        int32_t d = 0;
        if (lane < K) {
            o = peer_slot(ids, row_of, offs, seg, t * K + lane, E, EL, recv_rows, max_rows, &d, status, 730);
            remote_row[t * K + lane] = o >= 0 ? d : -1;
        }
        uint4* dst[KS];
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int ok = __shfl_sync(0xffffffffu, o, k);
            const int32_t dk = __shfl_sync(0xffffffffu, d, k);
            dst[k] = ok >= 0 ? bufs[ok] + (int64_t)dk * vpr : nullptr;
        }
        const uint4* xr = x + t * vpr;
        for (int64_t v0 = lane; v0 < vpr; v0 += 32 * kPeerUnroll) {
            uint4 val[kPeerUnroll];
#pragma unroll
            for (int u = 0; u < kPeerUnroll; ++u) {
                const int64_t v = v0 + 32 * u;
                val[u] = v < vpr ? __ldg(xr + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                if (dst[k] == nullptr) continue;
#pragma unroll
                for (int u = 0; u < kPeerUnroll; ++u) {
                    const int64_t v = v0 + 32 * u;
                    if (v < vpr) dst[k][v] = val[u];
                }
            }
        }
    }
    __threadfence_system();
}

// y[t] = y_add[t] + sum over kept slots, in slot order, of topk_w[t, k] *
// (owner's y_loc)[remote_row[t, k]]: fp32 sums, rounded once.  One warp per
// token: lanes k < K read slot k's owner, row and weight, the warp broadcasts
// them, and each lane sums kPeerUnroll vectors of the row at a time (K x
// kPeerUnroll loads in flight).  The owners' rows are read with plain
// (coherent) loads: another GPU's kernel wrote them before the barrier that
// precedes this one.
template <typename ET, int KS>
__global__ void __launch_bounds__(kPeerWarps * 32) peer_combine_kernel(
    const uint4* const* __restrict__ y_bufs, const int32_t* __restrict__ ids,
    const int32_t* __restrict__ remote_row, const float* __restrict__ topk_w,
    const uint4* __restrict__ y_add, uint4* __restrict__ y, int64_t T, int K, int E, int EL, int W,
    int64_t vpr, int64_t recv_rows, int* status)
{
    __shared__ const uint4* bufs[kPeerMaxWorld];
    for (int i = threadIdx.x; i < W; i += blockDim.x) bufs[i] = y_bufs[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kPeerWarps;
    for (int64_t t = (int64_t)blockIdx.x * kPeerWarps + (threadIdx.x >> 5); t < T; t += nw) {
        const uint4* src = nullptr;
        float wk = 0.f;
        if (lane < K) {
            const int32_t d = __ldg(remote_row + t * K + lane);
            const int32_t e = __ldg(ids + t * K + lane);
            if (d >= 0) {
                if (e < 0 || e >= E || d >= recv_rows) {
                    raise_flag(status, kFlagBounds, 740);
                } else {
                    src = bufs[e / EL] + (int64_t)d * vpr;
                    wk = __ldg(topk_w + t * K + lane);
                }
            }
        }
        const uint4* srck[KS];
        float wks[KS];
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            srck[k] = reinterpret_cast<const uint4*>(
                __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), k));
            wks[k] = __shfl_sync(0xffffffffu, wk, k);
        }
        for (int64_t v0 = lane; v0 < vpr; v0 += 32 * kPeerUnroll) {
            float acc[kPeerUnroll][8];
#pragma unroll
            for (int u = 0; u < kPeerUnroll; ++u) {
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
                const int64_t v = v0 + 32 * u;
                if (y_add && v < vpr) Vec<ET>::add(acc[u], __ldg(y_add + t * vpr + v));
            }
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                if (srck[k] == nullptr) continue;
                uint4 val[kPeerUnroll];
#pragma unroll
                for (int u = 0; u < kPeerUnroll; ++u) {
                    const int64_t v = v0 + 32 * u;
                    val[u] = v < vpr ? srck[k][v] : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kPeerUnroll; ++u) Vec<ET>::add_scaled(acc[u], val[u], wks[k]);
            }
#pragma unroll
            for (int u = 0; u < kPeerUnroll; ++u) {
                const int64_t v = v0 + 32 * u;
                if (v < vpr) y[t * vpr + v] = Vec<ET>::pack(acc[u]);
            }
        }
    }
}

static unsigned peer_blocks(int64_t T)
{
    int64_t blocks = (T + kPeerWarps - 1) / kPeerWarps;
    const int64_t cap = (int64_t)sm_count_ep() * 16;
    if (blocks > cap) blocks = cap;
    return (unsigned)(blocks < 1 ? 1 : blocks);
}

cudaError_t launch_peer_dispatch(const moe_config& c, int rank, int W, const int32_t* kept_all, const void* x,
                                 const int32_t* ids, const int32_t* row_of, const int32_t* offsets,
                                 void* const* recv_bufs, int64_t recv_rows, int64_t max_rows,
                                 int32_t* local_offsets, int32_t* remote_row, int* status, cudaStream_t s)
{
    const int64_t vpr = (int64_t)c.D * (c.dtype == MOE_BF16 ? 2 : 4) / 16;
    const int EL = c.E / W;
    const unsigned blocks = peer_blocks(c.T);
    const uint4* xv = static_cast<const uint4*>(x);
    uint4* const* rb = reinterpret_cast<uint4* const*>(recv_bufs);
#define MOE_PEER_DISPATCH(KS)                                                                          \
    peer_dispatch_kernel<KS><<<blocks, kPeerWarps * 32, 0, s>>>(xv, ids, row_of, offsets, kept_all, rb, \
                                                                c.T, c.K, c.E, EL, W, rank, vpr,       \
                                                                recv_rows, max_rows, local_offsets,    \
                                                                remote_row, status)
    if (c.K <= 1) MOE_PEER_DISPATCH(1);
    else if (c.K == 2) MOE_PEER_DISPATCH(2);
    else if (c.K <= 4) MOE_PEER_DISPATCH(4);
    else MOE_PEER_DISPATCH(8);
#undef MOE_PEER_DISPATCH
    return cudaGetLastError();
}

template <typename ET>
static void launch_peer_combine_t(const moe_config& c, int W, unsigned blocks, const uint4* const* yb,
                                  const int32_t* ids, const int32_t* remote_row, const float* topk_w,
                                  const uint4* add, uint4* y, int64_t vpr, int64_t recv_rows, int* status,
                                  cudaStream_t s)
{
    const int EL = c.E / W;
#define MOE_PEER_COMBINE(KS)                                                                      \
    peer_combine_kernel<ET, KS><<<blocks, kPeerWarps * 32, 0, s>>>(yb, ids, remote_row, topk_w, add, y, \
                                                                   c.T, c.K, c.E, EL, W, vpr,         \
                                                                   recv_rows, status)
    if (c.K <= 1) MOE_PEER_COMBINE(1);
    else if (c.K == 2) MOE_PEER_COMBINE(2);
    else if (c.K <= 4) MOE_PEER_COMBINE(4);
    else MOE_PEER_COMBINE(8);
#undef MOE_PEER_COMBINE
}

cudaError_t launch_peer_combine(const moe_config& c, int W, const void* const* y_bufs, const int32_t* ids,
                                const int32_t* remote_row, const float* topk_w, int64_t recv_rows,
                                const void* y_add, void* y, int* status, cudaStream_t s)
{
    const int64_t vpr = (int64_t)c.D * (c.dtype == MOE_BF16 ? 2 : 4) / 16;
    const unsigned blocks = peer_blocks(c.T);
    const uint4* const* yb = reinterpret_cast<const uint4* const*>(y_bufs);
    const uint4* add = static_cast<const uint4*>(y_add);
    uint4* out = static_cast<uint4*>(y);
    if (c.dtype == MOE_BF16)
        launch_peer_combine_t<__nv_bfloat16>(c, W, blocks, yb, ids, remote_row, topk_w, add, out, vpr,
                                             recv_rows, status, s);
    else
        launch_peer_combine_t<float>(c, W, blocks, yb, ids, remote_row, topk_w, add, out, vpr, recv_rows,
                                     status, s);
    return cudaGetLastError();
}

}  // namespace moe
