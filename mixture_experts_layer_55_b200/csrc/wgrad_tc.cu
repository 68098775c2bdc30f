// wgrad_tc.cu -- weight gradients of the grouped expert GEMMs on the
// 5th-generation tensor cores (tcgen05 MMA, fp32 accumulators in tensor
// memory, operands staged by TMA).
//
// "Lab: build a tiny MoE in PyTorch", "Smoke test and backward pass": the
// experts' weights receive gradient from the rows routed to them.  Each
// expert's rows are one contiguous block of the expert-major layout, so every
// weight gradient is one GEMM per expert contracting over that block:
//
//   dWd_e          = h[block]^T      . dYp[block]        (M = F, N = D)
//   [dWg_e | dWu_e] = x_perm[block]^T . [dg | du][block]  (M = D, N = 2F, split at F)
//
// Both operands are row blocks of row-major (rows, M) and (rows, N) matrices,
// so both are read MN-major (128-byte swizzle, 64-column boxes); K is the
// expert's row count, ragged.  Each expert reads its operands through its own
// pair of tensor maps, whose row extent ends at the expert's last row: a K
// block that runs past it arrives with those rows zero-filled by the copy
// engine, so nothing has to be fixed up in shared memory before the MMAs.  A
// small kernel writes the maps before each launch (a host-encoded template,
// its row extent replaced on the device from the row offsets, which stay on
// the device).  An expert with no rows writes zeros.  The result is stored in
// fp32 (the precision weight gradients are accumulated in).
//
// Persistent kernel, one CTA per SM, tiles M = 128 x N = 256, 4-stage ring of
// 48 KB, double-buffered 2 x 256-column accumulators.  10 warps: warp 0 TMA,
// warp 1 MMA (one thread), warps 2..9 epilogue.  The epilogue stages each
// warp's 32 x 32 fp32 pieces in shared memory (128-byte swizzle, conflict-free)
// and writes them with TMA tensor stores over an (E, M, N) map, so the stores
// are whole lines and the map clips the tile's edges per expert.  (Measured:
// six operand stages with one staging buffer per warp beat five stages with
// two; the zero-filling maps beat zeroing the tail rows in shared memory from
// a dedicated warp by 7-8 %.)  Every wait is bounded (device status flag).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace wg {

constexpr int BN = 256;                 // output columns per tile
constexpr int BK = 64;                  // K rows per stage
constexpr int UK = 16;                  // K per tcgen05.mma (bf16)
constexpr int BOX_BYTES = 64 * 64 * 2;  // one 64-column x 64-row box
constexpr int OUT_BYTES = 32 * 32 * 4;  // one staged 32 x 32 fp32 piece
constexpr int OUT_BUFS = 1;             // staged pieces per epilogue warp
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 320;  // warp 0 TMA, 1 MMA, 2..9 epilogue
constexpr int EPI_WARPS = 8;
constexpr int MAX_E = 256;

// Single CTA: M = 128 output rows, all 256 columns in this CTA (2 A + 4 B
// boxes per stage, 4 stages).  CTA pair: M = 256, each CTA its 128 rows of A
// and 128 of the columns of B (2 + 2 boxes, 6 stages); the leader issues.
template <bool PAIR> struct Geo {
    static constexpr int CTAS = PAIR ? 2 : 1;
    static constexpr int BM = 128 * CTAS;
    static constexpr int A_BOXES = 2;
    static constexpr int B_BOXES = 4 / CTAS;
    static constexpr int A_BYTES = A_BOXES * BOX_BYTES;
    static constexpr int STAGE_BYTES = (A_BOXES + B_BOXES) * BOX_BYTES;  // 48 KB single, 32 KB pair
    static constexpr int STAGES = PAIR ? 6 : 4;
    static constexpr int EPI_ARRIVALS = EPI_WARPS * CTAS;
};

struct Misc {
    uint64_t full[6];
    uint64_t empty[6];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int off[MAX_E + 1];  // validated row offsets: expert e owns rows off[e] .. off[e+1]-1
};

template <bool PAIR> constexpr size_t smem_bytes()
{
    return 1024 + (size_t)Geo<PAIR>::STAGES * Geo<PAIR>::STAGE_BYTES +
           (size_t)EPI_WARPS * OUT_BUFS * OUT_BYTES + sizeof(Misc);
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory per block");

struct Args {
    const int32_t* offsets;  // (E + 1) row offsets of the experts' blocks
    const CUtensorMap* maps; // 2 per expert (A, B): the operands' maps, rows ending at the expert's end
    int E;
    int M;                   // output rows (A's columns)
    int Nh;                  // output columns per half
    int halves;              // 1, or 2 when B holds two Nh-column halves
    int mt;                  // ceil(M / BM)
    int nth;                 // ceil(Nh / BN)
    int n_fast;              // tile order within an expert: n tiles fastest (else m)
    int64_t max_rows;
    int* status;
};

// Tiles of one expert are consecutive; within the expert the fast index is
// the one whose operand block is the smaller, so that the concurrently running
// tiles keep that whole block in L2 and read the other block's slabs once.
MOE_DEVICE void decode(const Args& a, int bm, int t, int& e, int& m0, int& hf, int& n0)
{
    const int nn = a.nth * a.halves;  // n tiles over both halves
    const int per_e = a.mt * nn;
    e = t / per_e;
    const int r = t - e * per_e;
    int i, j;
    if (a.n_fast) {
        i = r / nn;
        j = r - i * nn;
    } else {
        j = r / a.mt;
        i = r - j * a.mt;
    }
    m0 = i * bm;
    hf = j / a.nth;
    n0 = (j - hf * a.nth) * BN;
}

// A tensor map in global memory, rewritten by the generic proxy: its row
// extent (dimension 1; dimension 0 is the contiguous one) is replaced in place;
// the writer releases the maps to the copy engine's view, each reader acquires
// the one it is about to use (which also drops a stale cached copy of it).
MOE_DEVICE void tmap_set_rows(CUtensorMap* gmap, uint32_t rows)
{
    asm volatile("tensormap.replace.tile.global_dim.global.b1024.b32 [%0], 1, %1;" ::"l"(gmap), "r"(rows)
                 : "memory");
}

MOE_DEVICE void tmap_release() { asm volatile("fence.proxy.tensormap::generic.release.gpu;" ::: "memory"); }

MOE_DEVICE void tmap_acquire(const CUtensorMap* gmap)
{
    asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(gmap) : "memory");
}

// maps[2e], maps[2e+1] = the A and B templates with the row extent cut to
// expert e's end (offsets[e+1], clamped to 1 .. max_rows: a malformed offset
// can only shorten the rows a map reaches, never extend them past the
// matrices).  One thread per expert.
__global__ void wgrad_maps_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                  const int32_t* offsets, int E, int64_t max_rows, CUtensorMap* maps)
{
    const int e = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    if (e >= E) return;
    int64_t r1 = offsets[e + 1];
    r1 = r1 < 1 ? 1 : (r1 > max_rows ? max_rows : r1);
    const uint4* srcA = reinterpret_cast<const uint4*>(&tmA);
    const uint4* srcB = reinterpret_cast<const uint4*>(&tmB);
    uint4* dA = reinterpret_cast<uint4*>(&maps[2 * e]);
    uint4* dB = reinterpret_cast<uint4*>(&maps[2 * e + 1]);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(CUtensorMap) / sizeof(uint4)); ++i) {
        dA[i] = srcA[i];
        dB[i] = srcB[i];
    }
    tmap_set_rows(&maps[2 * e], (uint32_t)r1);
    tmap_set_rows(&maps[2 * e + 1], (uint32_t)r1);
    tmap_release();
}

template <bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    wgrad_tc_kernel(const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                    const Args a)
{
    using G = Geo<PAIR>;
    constexpr int BM = G::BM, STAGES = G::STAGES, STAGE_BYTES = G::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* stages = smem;
    uint8_t* outbuf = smem + (size_t)STAGES * STAGE_BYTES;  // EPI_WARPS x OUT_BUFS pieces, 1 KB aligned
    Misc* m = reinterpret_cast<Misc*>(outbuf + (size_t)EPI_WARPS * OUT_BUFS * OUT_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = the pair's leader (issues the MMAs)
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&m->full[s], 1);
            mbar_init(&m->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&m->tfull[b], 1);
            mbar_init(&m->tempty[b], G::EPI_ARRIVALS);
        }
        mbar_init(&m->drain, 1);
        m->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmO0);
        if (a.halves == 2) prefetch_tmap(&tmO1);
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(&m->tmem_base, TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&m->tmem_base, TMEM_COLS);
            tmem_relinquish();
        }
    }
    for (int e = threadIdx.x; e <= E; e += NUM_THREADS) m->off[e] = a.offsets[e];
    __syncthreads();
    if (threadIdx.x == 0) {  // validate: offsets non-decreasing from 0, within max_rows
        int prev = 0;
        bool bad = false;
        for (int e = 0; e <= E; ++e) {
            int r = m->off[e];
            if (r < prev || (int64_t)r > a.max_rows || (e == 0 && r != 0)) {
                bad = true;
                r = prev;  // a malformed block becomes empty
            }
            m->off[e] = r;
            prev = r;
        }
        if (bad) raise_flag(a.status, kFlagBounds, 500);
    }
    tc_fence_before();
    if (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote signal
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    const int total = E * a.mt * a.nth * a.halves;
    volatile int* abort_flag = &m->abort_flag;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer (each CTA)
        int stage = 0;
        uint32_t phase = 0;       // of the ring: a stage's n-th use is its full[] phase n
        int last_par[STAGES];     // per stage: the parity of its last issued phase, -1 unused
        for (int s = 0; s < STAGES; ++s) last_par[s] = -1;
        bool ok = true;
        int last_e = -1;
        for (int t = unit; t < total && ok; t += units) {
            int e, m0, hf, n0;
            decode(a, BM, t, e, m0, hf, n0);
            const int r0 = m->off[e], r1 = m->off[e + 1];
            const CUtensorMap* mA = a.maps + 2 * e;
            const CUtensorMap* mB = mA + 1;
            if (e != last_e && r1 > r0) {  // the expert's maps, as the maps kernel wrote them
                tmap_acquire(mA);
                tmap_acquire(mB);
                last_e = e;
            }
            const int acol = m0 + 128 * (int)rank;                           // this CTA's A columns
            const int bcol = hf * a.Nh + n0 + (PAIR ? 128 * (int)rank : 0);  // and B columns
            for (int k = r0; k < r1; k += BK) {
                if (!mbar_wait(&m->empty[stage], phase ^ 1u, a.status, 510, abort_flag)) {
                    ok = false;
                    break;
                }
                uint64_t* bar = &m->full[stage];
                last_par[stage] = (int)phase;
                uint8_t* sA = stages + (size_t)stage * STAGE_BYTES;
                uint8_t* sB = sA + G::A_BYTES;
                // rows past the expert's end (and past the matrices) arrive as
                // zeros; the box's full size is counted either way
                if (PAIR) {
                    // both CTAs' bytes are counted on the leader's barrier
                    if (rank == 0) mbar_arrive_expect_tx(bar, 2 * STAGE_BYTES);
                    const uint32_t fb = mapa_shared(smem_u32(bar), 0);
#pragma unroll
                    for (int j = 0; j < G::A_BOXES; ++j)
                        tma_load_2d_pair(sA + j * BOX_BYTES, mA, acol + 64 * j, k, fb);
#pragma unroll
                    for (int j = 0; j < G::B_BOXES; ++j)
                        tma_load_2d_pair(sB + j * BOX_BYTES, mB, bcol + 64 * j, k, fb);
                } else {
                    mbar_arrive_expect_tx(bar, STAGE_BYTES);
#pragma unroll
                    for (int j = 0; j < G::A_BOXES; ++j) tma_load_2d(sA + j * BOX_BYTES, mA, acol + 64 * j, k, bar);
#pragma unroll
                    for (int j = 0; j < G::B_BOXES; ++j) tma_load_2d(sB + j * BOX_BYTES, mB, bcol + 64 * j, k, bar);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // never leave the CTA with a copy in flight (the leader sees every completion)
        if (!PAIR || rank == 0)
            for (int s = 0; s < STAGES; ++s)
                if (last_par[s] >= 0) mbar_wait(&m->full[s], (uint32_t)last_par[s], a.status, 511, nullptr);
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ---------------------------------------- MMA issuer (leader; one thread)
        // A and B MN-major: 64-column boxes 8 KB apart (LBO), 8-row K groups
        // 1024 B apart (SBO), +2048 B per 16-row K step
        constexpr uint32_t idesc = umma_idesc_bf16(BM, BN, 1, 1);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = unit; t < total && ok; t += units) {
            int e, m0, hf, n0;
            decode(a, BM, t, e, m0, hf, n0);
            const int r0 = m->off[e], r1 = m->off[e + 1];
            if (!mbar_wait(&m->tempty[acc], acc_phase ^ 1u, a.status, 520, abort_flag)) break;
            tc_fence_after();
            const uint32_t d0 = tmem_base + (uint32_t)(acc * ACC_COLS);
            for (int k = r0; k < r1; k += BK) {
                // rows of this block that belong to the expert; steps wholly past
                // the expert's last row are not issued (a partial step's tail rows
                // arrived as zeros)
                const int valid = r1 - k < BK ? r1 - k : BK;
                const int nsteps = (valid + UK - 1) / UK;
                if (!mbar_wait(&m->full[stage], phase, a.status, 521, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a32 = smem_u32(stages + (size_t)stage * STAGE_BYTES);
                const uint32_t b32 = a32 + G::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / UK; ++kk) {
                    if (kk >= nsteps) break;
                    const uint32_t accum = (k != r0 || kk != 0) ? 1u : 0u;
                    const uint64_t adesc = umma_desc_sw128(a32 + kk * 2048, BOX_BYTES, 1024);
                    const uint64_t bdesc = umma_desc_sw128(b32 + kk * 2048, BOX_BYTES, 1024);
                    if (PAIR) umma_f16_ss_pair(d0, adesc, bdesc, idesc, accum);
                    else umma_f16_ss(d0, adesc, bdesc, idesc, accum);
                }
                // frees the stage (in both CTAs) once these MMAs complete
                if (PAIR) umma_commit_pair_mc(&m->empty[stage], 0x3);
                else umma_commit(&m->empty[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            // accumulator ready for the epilogue (of both CTAs); with no rows: at once
            if (PAIR) umma_commit_pair_mc(&m->tfull[acc], 0x3);
            else umma_commit(&m->tfull[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        // wait for every MMA issued here before the allocation is released
        if (PAIR) umma_commit_pair_mc(&m->drain, 0x1);
        else umma_commit(&m->drain);
        mbar_wait(&m->drain, 0, a.status, 522, nullptr);
    } else if (warp >= 2 && warp < 2 + EPI_WARPS) {
        // -------------------------------------------------------- epilogue
        // warp w: tensor-memory lanes 32*(w%4) .. +31 (this CTA's output rows),
        // half of the 256 columns (warps 2..5 the first, 6..9 the second)
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        uint8_t* bufs = outbuf + (size_t)(warp - 2) * OUT_BUFS * OUT_BYTES;
        int nb = 0;  // the staging buffer to fill next
        const int swz = lane & 7;  // the 128-byte swizzle of this lane's staged row
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&m->tempty[0]), 0);
        const uint32_t tempty_leader1 = mapa_shared(smem_u32(&m->tempty[1]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = unit; t < total; t += units) {
            int e, m0, hf, n0;
            decode(a, BM, t, e, m0, hf, n0);
            const bool empty_block = m->off[e + 1] == m->off[e];
            // tcgen05.ld is warp-collective: the vote keeps the warp converged
            if (!__all_sync(0xffffffffu, mbar_wait(&m->tfull[acc], acc_phase, a.status, 530, abort_flag)))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * ACC_COLS);
            const CUtensorMap* tmo = hf ? &tmO1 : &tmO0;
            const int orow = m0 + 128 * (int)rank + quad * 32;
#pragma unroll 1
            for (int c = 4 * half; c < 4 * half + 4; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + c * 32, v);
                tmem_ld_wait();
                uint8_t* buf = bufs + nb * OUT_BYTES;
                nb = (nb + 1) % OUT_BUFS;
                if (lane == 0) bulk_wait_read<OUT_BUFS - 1>();  // this buffer's last store has read it
                __syncwarp();
                uint4* row = reinterpret_cast<uint4*>(buf + lane * 128);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    row[q ^ swz] = empty_block ? make_uint4(0, 0, 0, 0)
                                               : make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {  // rows >= M and columns >= Nh fall outside the map: not written
                    tma_store_3d(tmo, buf, n0 + c * 32, orow, e);
                    bulk_commit();
                }
            }
            // this warp is done reading the accumulator: one arrival, on the leader
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
                else mbar_arrive(&m->tempty[acc]);
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) bulk_wait_all<0>();  // every store of this warp has completed
        __syncwarp();
    }
    tc_fence_before();
    if (PAIR) cluster_sync();  // no CTA leaves while its peer may still signal it
    else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------- host --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encoder()
{
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 map over a row-major (rows, cols) matrix; box = 64 cols x 64 rows.
static bool map_rows(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map over (E, M, Nh) row-major outputs; box = 32 cols x 32 rows x 1,
// 128-byte swizzle (the epilogue stages its pieces in that layout).
static bool map_out(CUtensorMap* m, const float* base, uint64_t Nh, uint64_t M, uint64_t E)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {Nh, M, E};
    cuuint64_t strides[2] = {Nh * 4, Nh * M * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per device and mode: dynamic shared memory opted in, and how many CTAs (or
// CTA pairs) can be resident at once, which sizes the persistent grid.
template <bool PAIR> static cudaError_t prepare(int* units_out)
{
    static std::atomic<int> cached[32];  // 0 = not yet queried on that device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 32 && cached[dev].load(std::memory_order_acquire) > 0) {
        *units_out = cached[dev].load(std::memory_order_acquire);
        return cudaSuccess;
    }
    constexpr size_t smem = smem_bytes<PAIR>();
    e = cudaFuncSetAttribute(wgrad_tc_kernel<PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int units = 0;
    if (PAIR) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&units, wgrad_tc_kernel<true>, &cfg);
        if (e != cudaSuccess) return e;
    } else {
        e = cudaDeviceGetAttribute(&units, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    if (units < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 32) cached[dev].store(units, std::memory_order_release);
    *units_out = units;
    return cudaSuccess;
}

template <bool PAIR>
static cudaError_t launch_mode(const CUtensorMap& mO0, const CUtensorMap& mO1, Args a, cudaStream_t s)
{
    int units = 0;
    cudaError_t e = prepare<PAIR>(&units);
    if (e != cudaSuccess) return e;
    a.mt = (a.M + Geo<PAIR>::BM - 1) / Geo<PAIR>::BM;
    const int64_t total = (int64_t)a.E * a.mt * a.nth * a.halves;
    const int n = (int)(total < units ? total : units);
    constexpr size_t smem = smem_bytes<PAIR>();
    if (!PAIR) {
        wgrad_tc_kernel<false><<<n, NUM_THREADS, smem, s>>>(mO0, mO1, a);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * n), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, wgrad_tc_kernel<true>, mO0, mO1, a);
}

}  // namespace wg

size_t wgrad_maps_bytes(int E) { return (size_t)2 * E * sizeof(CUtensorMap); }

// out0/out1 (E, M, Nh) fp32 = for each expert, A[block]^T . B[block] with A
// (max_rows, M) and B (max_rows, halves * Nh) bf16 row-major.  CTA pairs
// (256-row output tiles) when M >= 256, single CTAs otherwise.  `maps`: device
// scratch of wgrad_maps_bytes(E), 128-byte aligned, that the launch rewrites
// (the experts' operand maps).
cudaError_t launch_wgrad_tc_bf16(int E, int64_t max_rows, const int32_t* offsets, const void* A,
                                 int M, const void* B, int Nh, int halves, float* out0, float* out1,
                                 void* maps, int* status, cudaStream_t s)
{
    using namespace wg;
    if (E < 1 || E > MAX_E || M < 1 || Nh < 1 || (halves != 1 && halves != 2)) return cudaErrorInvalidValue;
    if (maps == nullptr || ((uintptr_t)maps & 127) != 0) return cudaErrorInvalidValue;
    CUtensorMap mA, mB, mO0, mO1;
    if (!map_rows(&mA, A, (uint64_t)M, (uint64_t)max_rows) ||
        !map_rows(&mB, B, (uint64_t)Nh * halves, (uint64_t)max_rows) ||
        !map_out(&mO0, out0, (uint64_t)Nh, (uint64_t)M, (uint64_t)E) ||
        !map_out(&mO1, halves == 2 ? out1 : out0, (uint64_t)Nh, (uint64_t)M, (uint64_t)E))
        return cudaErrorInvalidValue;
    // the A block of an expert (M columns) larger than its B block (halves * Nh):
    // walk the n tiles fastest (e.g. the down projection's gradient, M = F)
    const int n_fast = (int64_t)M > (int64_t)Nh * halves ? 1 : 0;
    CUtensorMap* gmaps = static_cast<CUtensorMap*>(maps);
    wgrad_maps_kernel<<<(E + 127) / 128, 128, 0, s>>>(mA, mB, offsets, E, max_rows, gmaps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Args a{offsets, gmaps, E, M, Nh, halves, 0, (Nh + BN - 1) / BN, n_fast, max_rows, status};
    return M >= 256 ? launch_mode<true>(mO0, mO1, a, s) : launch_mode<false>(mO0, mO1, a, s);
}

}  // namespace moe
