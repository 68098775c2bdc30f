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
// Steps 1-3 normally run as one cooperative kernel (dispatch_index_kernel).
#include <atomic>

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
        // sixteen loads in flight at a time (clamped indices), bases in chunk order
        int64_t run = 0;
        for (int64_t b0 = 0; b0 < nchunks; b0 += 16) {
            int32_t v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int64_t b = b0 + u < nchunks ? b0 + u : nchunks - 1;
                v[u] = blk_cnt[b * E + e];
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (b0 + u < nchunks) {
                    blk_base[(b0 + u) * E + e] = (int32_t)run;
                    run += v[u];
                }
            }
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

// ------------------------------------------------- one-kernel index pass --
// The three steps above in one cooperative launch (every block resident), for
// the usual sizes: block b ranks chunk b within itself (as the rank kernel
// does) and publishes the chunk's per-expert counts; after one grid barrier
// each block reads all chunks' counts (a few thousand integers from L2) and
// derives its own rank bases and the offsets, so the scan needs no block of
// its own and no second barrier.  Same arithmetic, same results.

// Words of the workspace status region used by the grid barrier: arrivals,
// and a generation that the last block to arrive advances.  Both start at
// zero with the workspace, and the count is back at zero after every barrier.
constexpr int kGridBarCount = 17;
constexpr int kGridBarGen = 18;

// Grid-wide barrier of a cooperative launch.  Bounded: after kWaitLimitNs a
// waiting block raises the timeout flag and goes on (its results are then
// flagged as invalid).
MOE_DEVICE void grid_barrier(int* status, int where)
{
    __threadfence();  // this thread's global writes before the arrival
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile int* gen = status + kGridBarGen;
        const int my_gen = *gen;
        __threadfence();
        const int nb = (int)(gridDim.x * gridDim.y * gridDim.z);
        if (atomicAdd(status + kGridBarCount, 1) == nb - 1) {
            atomicExch(status + kGridBarCount, 0);
            __threadfence();
            atomicAdd(status + kGridBarGen, 1);
        } else {
            const uint64_t t0 = globaltimer_ns();
            uint32_t spins = 0;
            while (*gen == my_gen) {
                __nanosleep(64);
                if (((++spins) & 1023u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) {
                    raise_flag(status, kFlagTimeout, where);
                    break;
                }
            }
        }
        __threadfence();
    }
    __syncthreads();
}

__global__ void __launch_bounds__(256) dispatch_index_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int64_t C, int32_t* blk_cnt,
    int32_t* __restrict__ counts, int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ row_of, int64_t max_rows, int* status)
{
    __shared__ int32_t s_wcnt[8][256];  // per-warp counts, then warp prefixes
    __shared__ int32_t s_base[256];     // this chunk's rank base per expert
    __shared__ int32_t s_scan[256];     // kept, then its inclusive scan
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nch = (int)gridDim.x;
    for (int i = threadIdx.x; i < 8 * 256; i += 256) (&s_wcnt[0][0])[i] = 0;
    __syncthreads();

    // phase 1: ranks within the chunk, and the chunk's counts
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
            if (e < 0 || e >= E) {
                raise_flag(status, kFlagBounds, 100);
                e = -1;
            }
        }
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
    for (int e = threadIdx.x; e < E; e += 256) {
        int32_t run = 0;
        for (int w = 0; w < 8; ++w) {
            const int32_t v = s_wcnt[w][e];
            s_wcnt[w][e] = run;
            run += v;
        }
        blk_cnt[(size_t)blockIdx.x * E + e] = run;
    }
    grid_barrier(status, 102);

    // phase 2: this chunk's bases, every expert's count, kept and offset
    {
        const int e = threadIdx.x;
        int32_t kp = 0;
        if (e < E) {
            // every chunk's count of expert e, sixteen loads in flight at a time
            // (issued unconditionally at clamped indices), added in chunk order
            int64_t run = 0, mine = 0;
            for (int b0 = 0; b0 < nch; b0 += 16) {
                int32_t v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int b = b0 + u < nch ? b0 + u : nch - 1;
                    v[u] = __ldcg(blk_cnt + (size_t)b * E + e);
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    if (b0 + u < nch) {
                        if (b0 + u == (int)blockIdx.x) mine = run;
                        run += v[u];
                    }
                }
            }
            s_base[e] = (int32_t)mine;
            kp = (int32_t)(run < C ? run : C);
            if (blockIdx.x == 0) {
                counts[e] = (int32_t)run;
                kept[e] = kp;
            }
        }
        s_scan[e] = kp;
        __syncthreads();
        for (int o = 1; o < 256; o <<= 1) {  // inclusive Hillis-Steele scan
            const int32_t v = e >= o ? s_scan[e - o] : 0;
            __syncthreads();
            s_scan[e] += v;
            __syncthreads();
        }
        if (blockIdx.x == 0) {
            if (e < E) offsets[e + 1] = s_scan[e];
            if (e == 0) offsets[0] = 0;
        }
    }
    __syncthreads();

    // phase 3: keep iff rank < C; row = offset + rank
#pragma unroll
    for (int sgm = 0; sgm < kPerThread; ++sgm) {
        const int64_t a = base + sgm * 32 + lane;
        if (a >= n) continue;
        const int e = my_e[sgm];
        int32_t row = -1;
        if (e >= 0) {
            const int64_t rank = (int64_t)s_base[e] + s_wcnt[warp][e] + my_local[sgm];
            if (rank < C) {
                const int64_t r = (int64_t)(e > 0 ? s_scan[e - 1] : 0) + rank;
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

// Blocks of dispatch_index_kernel that can be resident at once (per device).
static int resident_index_blocks()
{
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int v = cached[dev].load(std::memory_order_acquire);
    if (v > 0) return v;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_index_kernel, 256, 0) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    v = per_sm * sms;
    cached[dev].store(v, std::memory_order_release);
    return v;
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
    if (dispatch_index_fused(c) && nch <= resident_index_blocks()) {
        // one cooperative launch: all chunks' blocks resident at once
        int E = c.E;
        void* args[] = {(void*)&ids, (void*)&n, (void*)&E, (void*)&C, (void*)&blk_cnt,
                        (void*)&counts, (void*)&kept, (void*)&offsets, (void*)&perm,
                        (void*)&row_of, (void*)&max_rows, (void*)&status};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(dispatch_index_kernel),
                                           dim3((unsigned)nch), dim3(256), args, 0, s);
    }
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
    static PerDeviceFlag smem_set;
    cudaError_t ae = opt_in_smem(smem_set, reinterpret_cast<const void*>(gather_kernel), smem);
    if (ae != cudaSuccess) return ae;
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
