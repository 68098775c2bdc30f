// dispatch.cu -- per-expert histogram, capacity, exclusive-scan offsets, a
// stable expert-major permutation, and the gather of token rows.
//
// "Lab: build a tiny MoE in PyTorch", sections "Full implementation" (bincount
// of the ids; gather of each expert's token rows) and "Add a capacity limit"
// (walk tokens, then slots, in order; keep an assignment while its expert has
// used fewer than C places).  Keeping the first C assignments of each expert
// in token order is exactly that rule, so the layout is computed in parallel:
//
//   1. dispatch_count_kernel  per chunk of 2048 assignments, per-expert counts
//                             (shared-memory atomics only).
//   2. dispatch_scan_kernel   one block: for each expert the running count over
//                             chunks (its rank base in every chunk), counts,
//                             kept = min(counts, C), offsets = exclusive scan.
//   3. dispatch_rank_kernel   per chunk: the rank of each assignment among the
//                             same expert's assignments, in order, from
//                             __match_any_sync within 32-wide segments plus
//                             per-segment prefix counts; keep iff rank < C;
//                             row = offsets[e] + rank.
//   4. gather_kernel          TMA bulk copies: each token row is loaded once
//                             into shared memory and stored to each of its
//                             kept rows of x_perm.
// Every result is fully determined by the ids (no atomics decide an order).
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kChunk = kDispatchChunk;  // 2048 = 256 threads x 8
constexpr int kPerThread = kChunk / 256;

__global__ void __launch_bounds__(256) dispatch_count_kernel(const int32_t* __restrict__ ids,
                                                             int64_t n, int E,
                                                             int32_t* __restrict__ blk_cnt,
                                                             int* status)
{
    __shared__ int hist[256];
    for (int e = threadIdx.x; e < 256; e += 256) hist[e] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kChunk;
    for (int i = threadIdx.x; i < kChunk; i += 256) {
        int64_t a = base + i;
        if (a >= n) break;
        int e = ids[a];
        if (e < 0 || e >= E) {
            raise_flag(status, kFlagBounds, 100);
            continue;
        }
        atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += 256) blk_cnt[(size_t)blockIdx.x * E + e] = hist[e];
}

// One block of 256 threads.  Thread e walks the chunks of expert e.
__global__ void __launch_bounds__(256) dispatch_scan_kernel(const int32_t* __restrict__ blk_cnt,
                                                            int32_t* __restrict__ blk_base,
                                                            int64_t nchunks, int E, int64_t C,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ kept,
                                                            int32_t* __restrict__ offsets)
{
    __shared__ int32_t s_scan[256];
    const int e = threadIdx.x;
    int32_t kp = 0;
    if (e < E) {
        int64_t run = 0;
        for (int64_t b = 0; b < nchunks; ++b) {
            int32_t v = blk_cnt[b * E + e];
            blk_base[b * E + e] = (int32_t)run;
            run += v;
        }
        counts[e] = (int32_t)run;
        kp = (int32_t)(run < C ? run : C);
        kept[e] = kp;
    }
    // inclusive Hillis-Steele scan over 256 entries, then shift to exclusive
    s_scan[e] = kp;
    __syncthreads();
    for (int o = 1; o < 256; o <<= 1) {
        int32_t v = e >= o ? s_scan[e - o] : 0;
        __syncthreads();
        s_scan[e] += v;
        __syncthreads();
    }
    if (e < E) offsets[e + 1] = s_scan[e];
    if (e == 0) offsets[0] = 0;
}

// Warp w of a block handles assignments [w*256, w*256 + 256) of the chunk as 8
// segments of 32, in order.
__global__ void __launch_bounds__(256) dispatch_rank_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int64_t C,
    const int32_t* __restrict__ blk_base, const int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ row_of, int64_t max_rows, int* status)
{
    __shared__ int32_t s_wcnt[8][256];  // per-warp running counts, then warp prefixes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < 8 * 256; i += 256) (&s_wcnt[0][0])[i] = 0;
    __syncthreads();

    const int64_t base = (int64_t)blockIdx.x * kChunk + (int64_t)warp * 256;
    const unsigned lt_mask = (1u << lane) - 1u;
    int32_t my_e[kPerThread];
    int32_t my_local[kPerThread];
#pragma unroll
    for (int sgm = 0; sgm < kPerThread; ++sgm) {
        const int64_t a = base + sgm * 32 + lane;
        int e = -1;
        if (a < n) {
            e = ids[a];
            if (e < 0 || e >= E) e = -1;  // counted as a bounds fault by the count kernel
        }
        // lanes holding the same expert (out-of-range lanes form their own group)
        unsigned same = __match_any_sync(0xffffffffu, e);
        int before = 0;
        if (e >= 0) before = s_wcnt[warp][e];
        __syncwarp();
        const int leader = __ffs(same) - 1;
        if (e >= 0 && lane == leader) s_wcnt[warp][e] = before + __popc(same);
        __syncwarp();
        my_e[sgm] = e;
        my_local[sgm] = before + __popc(same & lt_mask);
    }
    __syncthreads();
    // exclusive scan over the 8 warps, per expert
    for (int e = threadIdx.x; e < E; e += 256) {
        int32_t run = 0;
        for (int w = 0; w < 8; ++w) {
            int32_t v = s_wcnt[w][e];
            s_wcnt[w][e] = run;
            run += v;
        }
    }
    __syncthreads();
#pragma unroll
    for (int sgm = 0; sgm < kPerThread; ++sgm) {
        const int64_t a = base + sgm * 32 + lane;
        if (a >= n) continue;
        const int e = my_e[sgm];
        int32_t row = -1;
        if (e >= 0) {
            const int64_t rank =
                (int64_t)blk_base[(size_t)blockIdx.x * E + e] + s_wcnt[warp][e] + my_local[sgm];
            if (rank < C) {
                const int64_t r = (int64_t)offsets[e] + rank;
                if (r >= 0 && r < max_rows) {
                    row = (int32_t)r;
                    perm[r] = (int32_t)a;
                } else {
                    raise_flag(status, kFlagBounds, 101);
                }
            }
        }
        row_of[a] = row;
    }
}

cudaError_t launch_dispatch_index(const moe_config& c, int64_t C, const int32_t* ids,
                                  int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* perm,
                                  int32_t* row_of, char* ws, const WsLayout& L, cudaStream_t s)
{
    const int64_t n = c.T * c.K;
    const int64_t nch = dispatch_chunks(c);
    int* status = reinterpret_cast<int*>(ws + L.status);
    int32_t* blk_cnt = reinterpret_cast<int32_t*>(ws + L.d_cnt);
    int32_t* blk_base = reinterpret_cast<int32_t*>(ws + L.d_base);
    const int64_t max_rows = max_rows_of(c);
    dispatch_count_kernel<<<(unsigned)nch, 256, 0, s>>>(ids, n, c.E, blk_cnt, status);
    dispatch_scan_kernel<<<1, 256, 0, s>>>(blk_cnt, blk_base, nch, c.E, C, counts, kept, offsets);
    dispatch_rank_kernel<<<(unsigned)nch, 256, 0, s>>>(ids, n, c.E, C, blk_base, offsets, perm,
                                                       row_of, max_rows, status);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ gather --
// Each warp owns a contiguous range of (token, piece) work items; its lane 0
// drives a ring of kGatherBufs shared-memory buffers: bulk-load a piece of
// x[t] (the token row is read once), then bulk-store it to each kept row of
// x_perm.  Loads run kGatherBufs - 1 items ahead of the stores.
constexpr int kGatherWarps = 4;
constexpr int kGatherBufs = 4;
constexpr int kGatherPiece = 4096;  // bytes per buffer

__global__ void __launch_bounds__(kGatherWarps * 32) gather_kernel(
    const char* __restrict__ x, const int32_t* __restrict__ row_of, char* __restrict__ x_perm,
    int64_t T, int K, int64_t row_bytes, int64_t max_rows, int* status)
{
    extern __shared__ __align__(128) char g_smem[];
    __shared__ __align__(8) uint64_t bars[kGatherWarps][kGatherBufs];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    char* ring = g_smem + (size_t)warp * kGatherBufs * kGatherPiece;
    uint64_t* bar = bars[warp];
    if (lane == 0)
        for (int b = 0; b < kGatherBufs; ++b) mbar_init(&bar[b], 1);
    fence_mbar_init();
    __syncwarp();
    if (lane != 0) return;

    const int64_t pieces = (row_bytes + kGatherPiece - 1) / kGatherPiece;
    const int64_t items = T * pieces;  // item = t * pieces + piece
    const int64_t nw = (int64_t)gridDim.x * kGatherWarps;
    const int64_t per = (items + nw - 1) / nw;
    const int64_t gw = (int64_t)blockIdx.x * kGatherWarps + warp;
    const int64_t it_begin = gw * per;
    const int64_t it_end = min(items, it_begin + per);

    int64_t next = it_begin;   // next item to examine for loading
    int64_t nlive = 0;         // items loaded so far (items of all-dropped tokens are skipped)
    int64_t slot_item[kGatherBufs];

    // Load the next item that has at least one kept row into ring slot
    // nlive % kGatherBufs.  That slot was last read by the stores of live item
    // nlive - kGatherBufs, which are all committed groups but the newest one.
    auto load_next = [&]() -> bool {
        while (next < it_end) {
            const int64_t it = next++;
            const int64_t t = it / pieces;
            bool live = false;
            for (int k = 0; k < K; ++k) live |= row_of[t * K + k] >= 0;
            if (!live) continue;
            const int b = (int)(nlive % kGatherBufs);
            bulk_wait_read<1>();
            slot_item[b] = it;
            const int64_t off = (it % pieces) * kGatherPiece;
            const uint32_t bytes = (uint32_t)(row_bytes - off < kGatherPiece ? row_bytes - off : (int64_t)kGatherPiece);
            mbar_arrive_expect_tx(&bar[b], bytes);
            bulk_load_g2s(ring + (size_t)b * kGatherPiece, x + t * row_bytes + off, bytes, &bar[b]);
            ++nlive;
            return true;
        }
        return false;
    };

    for (int i = 0; i < kGatherBufs - 1; ++i)
        if (!load_next()) break;
    for (int64_t done = 0; done < nlive; ++done) {
        const int b = (int)(done % kGatherBufs);
        const uint32_t parity = (uint32_t)((done / kGatherBufs) & 1);
        if (!mbar_wait(&bar[b], parity, status, 200, nullptr)) break;
        const int64_t it = slot_item[b];
        const int64_t t = it / pieces;
        const int64_t off = (it % pieces) * kGatherPiece;
        const uint32_t bytes = (uint32_t)(row_bytes - off < kGatherPiece ? row_bytes - off : (int64_t)kGatherPiece);
        for (int k = 0; k < K; ++k) {
            const int32_t r = row_of[t * K + k];
            if (r < 0) continue;
            if (r >= max_rows) {
                raise_flag(status, kFlagBounds, 201);
                continue;
            }
            bulk_store_s2g(x_perm + (int64_t)r * row_bytes + off, ring + (size_t)b * kGatherPiece,
                           bytes);
        }
        bulk_commit();
        load_next();
    }
    bulk_wait_all<0>();
}

cudaError_t launch_gather(const moe_config& c, const void* x, const int32_t* row_of, void* x_perm,
                          int64_t max_rows, int* status, cudaStream_t s)
{
    const int64_t row_bytes = (int64_t)c.D * (c.dtype == MOE_BF16 ? 2 : 4);
    const size_t smem = (size_t)kGatherWarps * kGatherBufs * kGatherPiece;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t pieces = (row_bytes + kGatherPiece - 1) / kGatherPiece;
    const int64_t items = c.T * pieces;
    int64_t blocks = (items + kGatherWarps - 1) / kGatherWarps;
    const int64_t cap = (int64_t)sms * 3;  // 3 blocks of 64 KB per SM
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    gather_kernel<<<(unsigned)blocks, kGatherWarps * 32, smem, s>>>(
        static_cast<const char*>(x), row_of, static_cast<char*>(x_perm), c.T, c.K, row_bytes,
        max_rows, status);
    return cudaGetLastError();
}

}  // namespace moe
