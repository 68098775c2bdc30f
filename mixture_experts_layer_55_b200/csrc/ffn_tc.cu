// ffn_tc.cu -- grouped SwiGLU expert FFN on the 5th-generation tensor cores
// (tcgen05 MMA, accumulators in tensor memory, operands staged by TMA).
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation":
// SwiGLUExpert computes down(silu(gate x) * up x) with no biases, and each
// expert output is scaled by its combine weight before the scatter-add.  The
// experts' rows are contiguous blocks of x_perm (expert-major), so each
// expert is one dense GEMM over its block; both contractions run here:
//
//   gate/up:  [G | U] = x_perm[block] . [Wg_e | Wu_e]   (K = D, two fp32 accumulators)
//             h = bf16(silu(G) * U)                     (epilogue)
//   down:     Y = h[block] . Wd_e                       (K = F)
//             y_perm = bf16(topk_w[perm[row]] * Y)      (epilogue)
//
// and the two data-gradient contractions of the backward ("Lab: build a tiny
// MoE in PyTorch", "Smoke test and backward pass"), on the same tiles:
//
//   dgrad-h:  dH = dYp[block] . Wd_e^T                  (K = D; Wd_e read K-major)
//             [dg | du] = bf16(dH * u * silu'(g) | dH * silu(g))
//                         (epilogue; g, u = the forward's saved pre-activations)
//   dgrad-x:  dXp = [dg | du][block] . [Wg_e | Wu_e]^T  (K = 2F; both read K-major)
//
// Persistent kernel, one CTA per SM, either alone (M = 128 rows per tile,
// cta_group::1) or as a CTA pair on two SMs (M = 256, cta_group::2: each CTA
// holds its 128 rows of A and half of B's columns, the leader issues the MMAs
// for both).  10 warps per CTA:
//   warp 0      TMA producer: A tile 128 x 64 (K-major, 128-byte swizzle) and
//               B tiles 64 x 64 (N-major, 128-byte swizzle) into a 4-stage
//               (single) or 6-stage (pair) ring
//   warp 1      MMA issuer: tcgen05.mma.kind::f16, N = 256, K = 16 per
//               instruction (gate/up: gate and up columns interleaved in
//               64-column blocks, so one MMA feeds both accumulators);
//               it also owns the 512-column tensor-memory allocation
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (lane = row; two
//               warps per lane quadrant, each half of the columns), the
//               SwiGLU or routing-weight step, bf16 stores to global memory
// Accumulators are double-buffered in tensor memory (2 x 256 columns), so the
// epilogue of one tile overlaps the MMAs of the next.  Tiles are ordered
// (expert, n-tile, m-tile) with m fastest: concurrently running CTAs share an
// expert's weight tile through L2.  The tile -> (expert, rows) map is built
// on the device from the dispatch offsets; rows past an expert's block are
// computed but never stored.  Every wait is bounded (device status flag).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace tc {

constexpr int BK = 64;                 // K per stage: one 128-byte swizzle row of bf16
constexpr int UK = 16;                 // K per tcgen05.mma (bf16)
constexpr int BOX_BYTES = 64 * 64 * 2; // one 64 x 64 B box
constexpr int A_BYTES = 128 * BK * 2;  // this CTA's 128 rows of A per stage: 16 KB
constexpr int ACC_COLS = 256;          // tensor-memory columns per accumulator buffer
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 320;      // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int EPI_WARPS = 8;          // two per tensor-memory lane quadrant
constexpr int MAX_E = 256;

// Tile geometry.  Single CTA: M = 128 rows, all N columns of the tile's B in
// this CTA (gate/up: 128 gate + 128 up; down: 256).  CTA pair: M = 256 rows,
// 128 per CTA, and each CTA holds half of every B tile's columns.
// Contraction modes (the template argument; the forward's values are 0 and 1).
enum : int { kDown = 0, kGateUp = 1, kDgradH = 2, kDgradX = 3 };

template <int MODE, bool PAIR> struct Geo {
    static constexpr bool GATEUP = MODE == kGateUp;
    static constexpr bool B_KMAJOR = MODE == kDgradH || MODE == kDgradX;  // B = a weight, transposed
    static constexpr int CTAS = PAIR ? 2 : 1;
    static constexpr int BM = 128 * CTAS;                  // rows per tile
    static constexpr int BN = GATEUP ? 128 : 256;          // output columns per tile
    static constexpr int B_BOXES = 256 / 64 / CTAS;        // 64-wide B boxes per CTA per stage
    static constexpr int B_BYTES = B_BOXES * BOX_BYTES;    // (K-major B: one box of 256/CTAS rows)
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB single, 32 KB pair
    // the epilogue stages its 32 x 32 bf16 pieces for TMA stores: 2 KB per
    // epilogue warp; dgrad-h writes two at a time (4 KB), which costs it one
    // operand stage
    static constexpr int OUT_BYTES = MODE == kDgradH ? 4096 : 2048;
    static constexpr int STAGES = MODE == kDgradH ? (PAIR ? 5 : 3) : (PAIR ? 6 : 4);
    static constexpr int EPI_ARRIVALS = EPI_WARPS * CTAS;  // one per epilogue warp
};

struct Misc {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint64_t gbar[8];     // dgrad-h: an epilogue warp's [g | u] piece has landed (one per warp)
    uint32_t tmem_base;
    int abort_flag;
    int row0[MAX_E];
    int rowend[MAX_E];
    int pref[MAX_E + 1];  // first tile index of each expert; pref[E] = total tiles
};

template <int MODE, bool PAIR>
constexpr size_t smem_bytes()
{
    return 1024 /*alignment slack*/ + (size_t)Geo<MODE, PAIR>::STAGES * Geo<MODE, PAIR>::STAGE_BYTES +
           (size_t)EPI_WARPS * Geo<MODE, PAIR>::OUT_BYTES + sizeof(Misc);
}

struct Args {
    const int32_t* offsets;
    const int32_t* perm;
    const float* topk_w;
    __nv_bfloat16* out;  // h (gate/up), y_perm (down), [dg | du] (dgrad-h), dXp (dgrad-x)
    int E;
    int Kdim;            // D for gate/up and dgrad-h, F for down and for each half of dgrad-x
    int N;               // F for gate/up and dgrad-h, D for down and dgrad-x
    int n_tiles;         // ceil(N / BN)
    int64_t ldo;         // row stride of out in elements (N; 2N for dgrad-h)
    int64_t max_rows;
    int64_t nk;          // T * K (range of perm values)
    __nv_bfloat16* gu_out;       // gate/up: keep [g | u] here, row stride 2N (null: do not)
    const __nv_bfloat16* gu_in;  // dgrad-h: the kept [g | u], row stride 2N
    int* status;
    const CUtensorMap* amaps;    // A's map per expert, rows ending at the expert's end (null: tmA)
};

// A tensor map in global memory, rewritten by the generic proxy: its row extent
// (dimension 1; dimension 0 is the contiguous one) is replaced in place; the
// writer releases the maps to the copy engine's view, each reader acquires the
// one it is about to use (which also drops a stale cached copy of it).
MOE_DEVICE void tmap_set_rows(CUtensorMap* gmap, uint32_t rows)
{
    asm volatile("tensormap.replace.tile.global_dim.global.b1024.b32 [%0], 1, %1;" ::"l"(gmap), "r"(rows)
                 : "memory");
}

// the same for a 3-D map whose rows are dimension 2 ([dg | du] viewed as (rows, 2, F))
MOE_DEVICE void tmap_set_rows_dim2(CUtensorMap* gmap, uint32_t rows)
{
    asm volatile("tensormap.replace.tile.global_dim.global.b1024.b32 [%0], 2, %1;" ::"l"(gmap), "r"(rows)
                 : "memory");
}

MOE_DEVICE void tmap_release() { asm volatile("fence.proxy.tensormap::generic.release.gpu;" ::: "memory"); }

MOE_DEVICE void tmap_acquire(const CUtensorMap* gmap)
{
    asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(gmap) : "memory");
}

// maps[e] = tmX, maps[E + e] = tmH, each with the row extent cut to expert e's
// end (offsets[e+1], clamped to 1 .. max_rows: a malformed offset can only
// shorten the rows a map reaches).  A tile's rows past its expert's end then
// arrive as zeros from the copy engine instead of being read (their results are
// never stored).  The forward's pair is (x_perm, h), both 2-D; the backward's
// (dYp, [dg | du]), the second 3-D with its rows in dimension 2 (h_rows_dim2).
// One thread per expert.
__global__ void ffn_amaps_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmH,
                                 const int32_t* offsets, int E, int64_t max_rows, int h_rows_dim2,
                                 CUtensorMap* maps)
{
    const int e = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    if (e >= E) return;
    int64_t r1 = offsets[e + 1];
    r1 = r1 < 1 ? 1 : (r1 > max_rows ? max_rows : r1);
    const uint4* sx = reinterpret_cast<const uint4*>(&tmX);
    const uint4* sh = reinterpret_cast<const uint4*>(&tmH);
    uint4* dx = reinterpret_cast<uint4*>(&maps[e]);
    uint4* dh = reinterpret_cast<uint4*>(&maps[E + e]);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(CUtensorMap) / sizeof(uint4)); ++i) {
        dx[i] = sx[i];
        dh[i] = sh[i];
    }
    tmap_set_rows(&maps[e], (uint32_t)r1);
    if (h_rows_dim2) tmap_set_rows_dim2(&maps[E + e], (uint32_t)r1);
    else tmap_set_rows(&maps[E + e], (uint32_t)r1);
    tmap_release();
}

MOE_DEVICE void decode_tile(const Misc* m, int E, int bm, int bn, int t, int& e, int& m_row0,
                            int& row_end, int& n0)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // largest e with pref[e] <= t (its block is non-empty)
        const int mid = (lo + hi + 1) >> 1;
        if (m->pref[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    e = lo;
    const int mt = (m->rowend[e] - m->row0[e] + bm - 1) / bm;
    const int local = t - m->pref[e];
    const int n = local / mt, mm = local - n * mt;
    m_row0 = m->row0[e] + mm * bm;
    row_end = m->rowend[e];
    n0 = n * bn;
}

// silu(g) and its derivative s + g s (1 - s), s = sigmoid(g), in fp32 for the
// backward's epilogue (the exponent is clamped where s underflows anyway).
MOE_DEVICE void silu_and_grad(float g, float& silu, float& dsilu)
{
    const float s = __fdividef(1.0f, 1.0f + __expf(fminf(-g, 80.0f)));
    silu = g * s;
    dsilu = fmaf(g * s, 1.0f - s, s);
}

// One 32 x 32 bf16 piece of the output, held one row per lane (16 packed
// words), written through the warp's staging buffer (64-byte swizzle: the
// 16-byte chunk q of row r at chunk q ^ ((r >> 1) & 3), conflict-free) by a
// TMA tensor store.  The map clips columns past its extent; the caller only
// takes this path when all 32 rows are the expert's.
template <int DIMS>
MOE_DEVICE void store_piece(uint8_t* buf, int lane, const uint32_t (&p)[16], const CUtensorMap* map, int c0,
                            int c1, int c2)
{
    if (lane == 0) bulk_wait_read<0>();  // the buffer's last store has read it
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(buf + lane * 64);
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q ^ sw] = make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        if (DIMS == 2) tma_store_2d(map, buf, c0, c1);
        else tma_store_3d(map, buf, c0, c1, c2);
        bulk_commit();
    }
}

template <int MODE, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                  const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmO0,
                  const __grid_constant__ CUtensorMap tmO1, const Args a)
{
    using G = Geo<MODE, PAIR>;
    constexpr bool GATEUP = G::GATEUP;
    constexpr int BM = G::BM, BN = G::BN, STAGES = G::STAGES, STAGE_BYTES = G::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* stages = smem;
    uint8_t* outbuf = smem + (size_t)STAGES * STAGE_BYTES;  // EPI_WARPS x OUT_BYTES, 1 KB aligned
    Misc* m = reinterpret_cast<Misc*>(outbuf + (size_t)EPI_WARPS * G::OUT_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = the pair's leader (issues the MMAs)
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // pair (or CTA) index
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
        for (int w = 0; w < 8; ++w) mbar_init(&m->gbar[w], 1);
        m->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB0);
        if (GATEUP || MODE == kDgradX) prefetch_tmap(&tmB1);
        prefetch_tmap(&tmO0);
        if ((GATEUP && a.gu_out != nullptr) || MODE == kDgradH) prefetch_tmap(&tmO1);
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
    // tile table from the offsets (validated: a malformed block is treated as empty)
    for (int e = threadIdx.x; e < E; e += NUM_THREADS) {
        m->row0[e] = a.offsets[e];
        m->rowend[e] = a.offsets[e + 1];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0, prev = 0;
        for (int e = 0; e < E; ++e) {
            int r0 = m->row0[e], r1 = m->rowend[e];
            if (r0 < prev || r1 < r0 || (int64_t)r1 > a.max_rows) {
                raise_flag(a.status, kFlagBounds, 400);
                r0 = r1 = prev;
            }
            m->row0[e] = r0;
            m->rowend[e] = r1;
            prev = r1;
            m->pref[e] = run;
            run += (r1 - r0 + BM - 1) / BM * a.n_tiles;
        }
        m->pref[E] = run;
    }
    tc_fence_before();
    if (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote signal
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    const int total = m->pref[E];
    const int kh = (a.Kdim + BK - 1) / BK;                  // K blocks (per half for dgrad-x)
    const int num_kb = MODE == kDgradX ? 2 * kh : kh;
    volatile int* abort_flag = &m->abort_flag;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer (each CTA)
        int stage = 0;
        uint32_t phase = 0;
        int last_phase[STAGES];
        for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
        bool ok = true;
        int last_e = -1;
        for (int t = unit; t < total && ok; t += units) {
            int e, m_row0, row_end, n0;
            decode_tile(m, E, BM, BN, t, e, m_row0, row_end, n0);
            const int a_row = m_row0 + (int)rank * 128;
            // the expert's own A map (rows past its end read as zeros)
            const CUtensorMap* mA = &tmA;
            if (a.amaps != nullptr) {
                mA = a.amaps + e;
                if (e != last_e) {
                    tmap_acquire(mA);
                    last_e = e;
                }
            }
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(&m->empty[stage], phase ^ 1u, a.status, 410, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* sA = stages + (size_t)stage * STAGE_BYTES;
                uint8_t* sB = sA + A_BYTES;
                const int k0 = kb * BK;
                if (MODE == kDgradX) {
                    // K = [dg | du]: half 0 against Wg, half 1 against Wu (each K-major)
                    const int hf = kb >= kh ? 1 : 0;
                    const int kk0 = (kb - hf * kh) * BK;
                    const CUtensorMap* mb = hf ? &tmB1 : &tmB0;
                    if (PAIR) {
                        if (rank == 0) mbar_arrive_expect_tx(&m->full[stage], 2 * STAGE_BYTES);
                        const uint32_t fb = mapa_shared(smem_u32(&m->full[stage]), 0);
                        tma_load_3d_pair(sA, mA, kk0, hf, a_row, fb);
                        tma_load_3d_pair(sB, mb, kk0, n0 + 128 * (int)rank, e, fb);
                    } else {
                        uint64_t* fb = &m->full[stage];
                        mbar_arrive_expect_tx(fb, STAGE_BYTES);
                        tma_load_3d(sA, mA, kk0, hf, a_row, fb);
                        tma_load_3d(sB, mb, kk0, n0, e, fb);
                    }
                } else if (MODE == kDgradH) {
                    // B = Wd_e read K-major: rows n (= f) of 64 K (= d) elements
                    if (PAIR) {
                        if (rank == 0) mbar_arrive_expect_tx(&m->full[stage], 2 * STAGE_BYTES);
                        const uint32_t fb = mapa_shared(smem_u32(&m->full[stage]), 0);
                        tma_load_2d_pair(sA, mA, k0, a_row, fb);
                        tma_load_3d_pair(sB, &tmB0, k0, n0 + 128 * (int)rank, e, fb);
                    } else {
                        uint64_t* fb = &m->full[stage];
                        mbar_arrive_expect_tx(fb, STAGE_BYTES);
                        tma_load_2d(sA, mA, k0, a_row, fb);
                        tma_load_3d(sB, &tmB0, k0, n0, e, fb);
                    }
                } else if (PAIR) {
                    // both CTAs' bytes are counted on the leader's full barrier
                    if (rank == 0) mbar_arrive_expect_tx(&m->full[stage], 2 * STAGE_BYTES);
                    const uint32_t fb = mapa_shared(smem_u32(&m->full[stage]), 0);
                    tma_load_2d_pair(sA, mA, k0, a_row, fb);
                    if (GATEUP) {  // this CTA's [gate 64 | up 64] columns
                        tma_load_3d_pair(sB, &tmB0, n0 + 64 * (int)rank, k0, e, fb);
                        tma_load_3d_pair(sB + BOX_BYTES, &tmB1, n0 + 64 * (int)rank, k0, e, fb);
                    } else {       // this CTA's 128 down columns
                        tma_load_3d_pair(sB, &tmB0, n0 + 128 * (int)rank, k0, e, fb);
                        tma_load_3d_pair(sB + BOX_BYTES, &tmB0, n0 + 128 * (int)rank + 64, k0, e, fb);
                    }
                } else {
                    uint64_t* fb = &m->full[stage];
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(sA, mA, k0, a_row, fb);
                    if (GATEUP) {  // [gate n0 | up n0 | gate n0+64 | up n0+64]
                        tma_load_3d(sB, &tmB0, n0, k0, e, fb);
                        tma_load_3d(sB + BOX_BYTES, &tmB1, n0, k0, e, fb);
                        tma_load_3d(sB + 2 * BOX_BYTES, &tmB0, n0 + 64, k0, e, fb);
                        tma_load_3d(sB + 3 * BOX_BYTES, &tmB1, n0 + 64, k0, e, fb);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tma_load_3d(sB + j * BOX_BYTES, &tmB0, n0 + 64 * j, k0, e, fb);
                    }
                }
                last_phase[stage] = (int)phase;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // never leave the CTA with a copy in flight (the leader sees every completion)
        if (!PAIR || rank == 0)
            for (int s = 0; s < STAGES; ++s)
                if (last_phase[s] >= 0) mbar_wait(&m->full[s], (uint32_t)last_phase[s], a.status, 411, nullptr);
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ------------------------------------------------ MMA issuer (leader only)
        constexpr uint32_t idesc = umma_idesc_bf16(BM, 256, 0, G::B_KMAJOR ? 0 : 1);
        // B: N-major; 64-column blocks 8 KB apart (LBO), 8-row K groups 1024 B apart (SBO)
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = unit; t < total && ok; t += units) {
            if (!mbar_wait(&m->tempty[acc], acc_phase ^ 1u, a.status, 420, abort_flag)) break;
            tc_fence_after();
            const uint32_t d0 = tmem_base + (uint32_t)(acc * ACC_COLS);
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(&m->full[stage], phase, a.status, 421, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sA = smem_u32(stages + (size_t)stage * STAGE_BYTES);
                const uint32_t sB = sA + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / UK; ++kk) {
                    const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
                    // A: K-major, 8-row groups 1024 B apart; +32 B per 16-element K step
                    const uint64_t adesc = umma_desc_sw128(sA + kk * 32, 16, 1024);
                    // one N = 256 MMA: the 64-column boxes of B (for gate/up,
                    // gate and up interleaved) are 8 KB apart; a K-major B (the
                    // dgrad modes) is laid out like A
                    const uint64_t bdesc = G::B_KMAJOR ? umma_desc_sw128(sB + kk * 32, 16, 1024)
                                                       : umma_desc_sw128(sB + kk * 2048, BOX_BYTES, 1024);
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
            // accumulator ready for the epilogue (of both CTAs)
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
        mbar_wait(&m->drain, 0, a.status, 422, nullptr);
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (each CTA, its 128 rows)
        // warp w reads tensor-memory lanes 32*(w%4) .. +31 (rows), and half of
        // the tile's columns: warps 2..5 the first half, warps 6..9 the second.
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r_in_tile = (int)rank * 128 + quad * 32 + lane;
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&m->tempty[0]), 0);
        const uint32_t tempty_leader1 = mapa_shared(smem_u32(&m->tempty[1]), 0);
        uint8_t* obuf = outbuf + (size_t)(warp - 2) * G::OUT_BYTES;  // staging (dgrad-h: [dg | du])
        uint64_t* gbar = &m->gbar[warp - 2];
        uint32_t gphase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = unit; t < total; t += units) {
            int e, m_row0, row_end, n0;
            decode_tile(m, E, BM, BN, t, e, m_row0, row_end, n0);
            // tcgen05.ld is warp-collective: the vote keeps the warp converged
            if (!__all_sync(0xffffffffu, mbar_wait(&m->tfull[acc], acc_phase, a.status, 430, abort_flag)))
                break;
            tc_fence_after();
            const int64_t row = (int64_t)m_row0 + r_in_tile;
            const bool valid = row < row_end;
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * ACC_COLS);
            __nv_bfloat16* orow = a.out + row * a.ldo;
            // the warp's 32 rows all belong to the expert: its pieces go through
            // shared memory and TMA stores; otherwise each lane stores its valid row
            const int64_t warp_row0 = (int64_t)m_row0 + (int)rank * 128 + quad * 32;
            const bool warp_full = warp_row0 + 32 <= row_end;
            if (GATEUP) {
#pragma unroll 1
                for (int c = 2 * half; c < 2 * half + 2; ++c) {
                    // accumulator columns: [gate 0-63 | up 0-63 | gate 64-127 | up 64-127]
                    uint32_t g[32], u[32];
                    const uint32_t gcol = (c < 2) ? (uint32_t)(c * 32) : (uint32_t)(128 + (c - 2) * 32);
                    tmem_ld_32x32b_x32(taddr + gcol, g);
                    tmem_ld_32x32b_x32(taddr + gcol + 64, u);
                    tmem_ld_wait();
                    if (valid) {
                        uint32_t p[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float h0 = silu_bf16_path(__uint_as_float(g[2 * j])) * __uint_as_float(u[2 * j]);
                            const float h1 =
                                silu_bf16_path(__uint_as_float(g[2 * j + 1])) * __uint_as_float(u[2 * j + 1]);
                            p[j] = pack_bf16x2(h0, h1);
                        }
                        const int col = n0 + c * 32;
                        if (warp_full) {
                            if (col < a.N) store_piece<2>(obuf, lane, p, &tmO0, col, (int)warp_row0, 0);
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                if (col + 8 * q < a.N)
                                    *reinterpret_cast<uint4*>(orow + col + 8 * q) =
                                        make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
                        }
                        if (a.gu_out != nullptr) {  // keep the pre-activations for the backward
                            __nv_bfloat16* grow = a.gu_out + row * 2 * (int64_t)a.N + col;
#pragma unroll 1
                            for (int which = 0; which < 2; ++which) {  // g, then u
                                const uint32_t* src = which ? u : g;
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    p[j] = pack_bf16x2(__uint_as_float(src[2 * j]), __uint_as_float(src[2 * j + 1]));
                                if (warp_full) {
                                    if (col < a.N) store_piece<3>(obuf, lane, p, &tmO1, col, which, (int)warp_row0);
                                } else {
#pragma unroll
                                    for (int q = 0; q < 4; ++q)
                                        if (col + 8 * q < a.N)
                                            *reinterpret_cast<uint4*>(grow + which * a.N + 8 * q) =
                                                make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
                                }
                            }
                        }
                    }
                }
            } else if (MODE == kDgradH) {
#pragma unroll 1
                for (int c = 4 * half; c < 4 * half + 4; ++c) {
                    const int col = n0 + c * 32;
                    // a warp whose 32 rows all belong to the expert has its [g | u]
                    // piece copied into its staging buffer by TMA (tmO1 maps the kept
                    // [g | u] like the [dg | du] stores, 64-byte swizzle), once the
                    // last stores have read the buffer; the others load by lane
                    const bool tma_in = warp_full && col < a.N;
                    if (tma_in) {
                        if (lane == 0) {
                            bulk_wait_read<0>();
                            mbar_arrive_expect_tx(gbar, 4096);
                            tma_load_3d(obuf, &tmO1, col, 0, (int)warp_row0, gbar);
                            tma_load_3d(obuf + 2048, &tmO1, col, 1, (int)warp_row0, gbar);
                        }
                        __syncwarp();
                    }
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    tmem_ld_wait();
                    if (tma_in) {
                        // an abort elsewhere ends the first wait early: the copy is still
                        // let land (bounded) before the buffer is touched or the CTA exits
                        if (!__all_sync(0xffffffffu, mbar_wait(gbar, gphase, a.status, 432, abort_flag)))
                            mbar_wait(gbar, gphase, a.status, 433, nullptr);
                        __syncwarp();
                        gphase ^= 1u;
                    }
                    if (valid && col < a.N) {
                        const __nv_bfloat16* grow = a.gu_in + row * 2 * (int64_t)a.N + col;
                        const uint4* gsrc = reinterpret_cast<const uint4*>(obuf + lane * 64);
                        const uint4* usrc = reinterpret_cast<const uint4*>(obuf + 2048 + lane * 64);
                        const int swz = (lane >> 1) & 3;
                        uint32_t dg[16], du[16];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 gq = make_uint4(0, 0, 0, 0), uq = make_uint4(0, 0, 0, 0);
                            if (tma_in) {  // columns past F arrived as zeros
                                gq = gsrc[q ^ swz];
                                uq = usrc[q ^ swz];
                            } else if (col + 8 * q < a.N) {
                                gq = *reinterpret_cast<const uint4*>(grow + 8 * q);
                                uq = *reinterpret_cast<const uint4*>(grow + a.N + 8 * q);
                            }
                            const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
                            const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                float o[2][2];
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const float gg = __uint_as_float(hh ? (gw[i] & 0xffff0000u) : (gw[i] << 16));
                                    const float uu = __uint_as_float(hh ? (uw[i] & 0xffff0000u) : (uw[i] << 16));
                                    const float dh = __uint_as_float(v[8 * q + 2 * i + hh]);
                                    float sl, dsl;
                                    silu_and_grad(gg, sl, dsl);
                                    o[0][hh] = dh * uu * dsl;  // dg
                                    o[1][hh] = dh * sl;        // du
                                }
                                dg[4 * q + i] = pack_bf16x2(o[0][0], o[0][1]);
                                du[4 * q + i] = pack_bf16x2(o[1][0], o[1][1]);
                            }
                        }
                        if (!warp_full) {  // rows past the expert's end: per-lane stores of the valid rows
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                if (col + 8 * q < a.N) {
                                    *reinterpret_cast<uint4*>(orow + col + 8 * q) =
                                        make_uint4(dg[4 * q], dg[4 * q + 1], dg[4 * q + 2], dg[4 * q + 3]);
                                    *reinterpret_cast<uint4*>(orow + a.N + col + 8 * q) =
                                        make_uint4(du[4 * q], du[4 * q + 1], du[4 * q + 2], du[4 * q + 3]);
                                }
                        } else {
                            // the piece through shared memory (64-byte swizzle: 16-byte chunk q of
                            // row r at chunk q ^ ((r >> 1) & 3)) and two TMA stores
                            uint4* gdst = reinterpret_cast<uint4*>(obuf + lane * 64);
                            uint4* udst = reinterpret_cast<uint4*>(obuf + 2048 + lane * 64);
                            const int sw = (lane >> 1) & 3;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                gdst[q ^ sw] = make_uint4(dg[4 * q], dg[4 * q + 1], dg[4 * q + 2], dg[4 * q + 3]);
                                udst[q ^ sw] = make_uint4(du[4 * q], du[4 * q + 1], du[4 * q + 2], du[4 * q + 3]);
                            }
                        }
                    }
                    if (warp_full && col < a.N) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {  // columns >= F fall outside the map: not written
                            tma_store_3d(&tmO0, obuf, col, 0, warp_row0);
                            tma_store_3d(&tmO0, obuf + 2048, col, 1, warp_row0);
                            bulk_commit();
                        }
                    }
                }
            } else {
                float w = 0.f;
                if (valid) {
                    if (a.perm == nullptr) {
                        w = 1.f;  // unit weights (a shared expert)
                    } else {
                        const int32_t pa = a.perm[row];
                        if (pa >= 0 && (int64_t)pa < a.nk) w = a.topk_w[pa];
                        else if (half == 0) raise_flag(a.status, kFlagBounds, 431);
                    }
                }
#pragma unroll 1
                for (int c = 4 * half; c < 4 * half + 4; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    tmem_ld_wait();
                    if (valid) {
                        uint32_t p[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            p[j] = pack_bf16x2(w * __uint_as_float(v[2 * j]), w * __uint_as_float(v[2 * j + 1]));
                        const int col = n0 + c * 32;
                        if (warp_full) {
                            if (col < a.N) store_piece<2>(obuf, lane, p, &tmO0, col, (int)warp_row0, 0);
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                if (col + 8 * q < a.N)
                                    *reinterpret_cast<uint4*>(orow + col + 8 * q) =
                                        make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
                        }
                    }
                }
            }
            // this warp is done reading the accumulator: one arrival per warp, on
            // the leader's barrier (the MMA issuer waits there)
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

// 2-D bf16 map over a row-major (rows, cols) matrix; box = 64 columns x box_rows rows.
static bool map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over (E, rows, cols) row-major weights; box = 64 cols x 64 rows x 1.
static bool map_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, E};
    cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over (E, rows, cols) row-major weights read K-major (the
// weight transposed): box = 64 cols (K) x box_rows rows (N) x 1.
static bool map_3d_kmajor(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E,
                          uint32_t box_rows)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, E};
    cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map viewing a (rows, 2 * half) row-major matrix as (rows, 2, half):
// box = 64 cols x 1 half x box_rows rows, so each half pads to 64 on its own.
static bool map_halves(CUtensorMap* m, const void* base, uint64_t half, uint64_t rows, uint32_t box_rows)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {half, 2, rows};
    cuuint64_t strides[2] = {half * 2, half * 4};
    cuuint32_t box[3] = {64, 1, box_rows};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 map over a row-major (rows, cols) output for 32 x 32 stores from
// shared memory laid out with the 64-byte swizzle.
static bool map_store_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over (rows, 2 * half) viewed as (rows, 2, half) for 32 x 32
// stores from shared memory laid out with the 64-byte swizzle.
static bool map_halves_store(CUtensorMap* m, const void* base, uint64_t half, uint64_t rows)
{
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {half, 2, rows};
    cuuint64_t strides[2] = {half * 2, half * 4};
    cuuint32_t box[3] = {32, 1, 32};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per device: dynamic shared memory opted in, and the number of CTAs (or CTA
// pairs) that can be resident at once, which sizes the persistent grid.
template <int MODE, bool PAIR>
static cudaError_t prepare(int* resident_units)
{
    static std::atomic<int> cached[32];  // 0 = not yet queried on that device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 32 && cached[dev].load(std::memory_order_acquire) > 0) {
        *resident_units = cached[dev].load(std::memory_order_acquire);
        return cudaSuccess;
    }
    constexpr size_t smem = smem_bytes<MODE, PAIR>();
    e = cudaFuncSetAttribute(ffn_tc_kernel<MODE, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    int units = 0;
    if (PAIR) {
        e = cudaFuncSetAttribute(ffn_tc_kernel<MODE, PAIR>, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
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
        e = cudaOccupancyMaxActiveClusters(&units, ffn_tc_kernel<MODE, PAIR>, &cfg);
        if (e != cudaSuccess) return e;
    } else {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        units = sms;  // one CTA per SM (shared memory allows no second)
    }
    if (units < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 32) cached[dev].store(units, std::memory_order_release);
    *resident_units = units;
    return cudaSuccess;
}

template <int MODE, bool PAIR>
static cudaError_t launch_one(const CUtensorMap& mA, const CUtensorMap& mB0, const CUtensorMap& mB1,
                              const CUtensorMap& mO0, const CUtensorMap& mO1,
                              const Args& a, int64_t tiles_bound, cudaStream_t s)
{
    int units = 0;
    cudaError_t e = prepare<MODE, PAIR>(&units);
    if (e != cudaSuccess) return e;
    int64_t n = tiles_bound < units ? tiles_bound : units;
    if (n < 1) n = 1;
    constexpr size_t smem = smem_bytes<MODE, PAIR>();
    if (!PAIR) {
        ffn_tc_kernel<MODE, false><<<(unsigned)n, NUM_THREADS, smem, s>>>(mA, mB0, mB1, mO0, mO1, a);
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
    return cudaLaunchKernelEx(&cfg, ffn_tc_kernel<MODE, true>, mA, mB0, mB1, mO0, mO1, a);
}

}  // namespace tc

// CTA pairs (256-row tiles) when experts hold 128 rows or more on average;
// single CTAs (128-row tiles) otherwise, which waste fewer padded rows when
// each expert has only a few tokens (decode-shaped layers).
static bool use_pairs(const moe_config& c, int64_t max_rows) { return max_rows >= 128 * (int64_t)c.E; }

cudaError_t launch_ffn_tc_bf16(const moe_config& c, int64_t max_rows, const void* x_perm,
                               const int32_t* offsets, const int32_t* perm, const float* topk_w,
                               const void* w_gate, const void* w_up, const void* w_down, void* h,
                               void* y_perm, void* gu_keep, void* amaps, int* status, cudaStream_t s,
                               StageHook mid, void* mid_ctx)
{
    using namespace tc;
    CUtensorMap mA, mG, mU, mH, mD;
    if (!map_2d(&mA, x_perm, (uint64_t)c.D, (uint64_t)max_rows, 128) ||
        !map_3d(&mG, w_gate, (uint64_t)c.F, (uint64_t)c.D, (uint64_t)c.E) ||
        !map_3d(&mU, w_up, (uint64_t)c.F, (uint64_t)c.D, (uint64_t)c.E) ||
        !map_2d(&mH, h, (uint64_t)c.F, (uint64_t)max_rows, 128) ||
        !map_3d(&mD, w_down, (uint64_t)c.D, (uint64_t)c.F, (uint64_t)c.E))
        return cudaErrorInvalidValue;
    // the epilogues' stores: h (rows, F), [g | u] (rows, 2, F), y_perm (rows, D)
    CUtensorMap mHo, mGUo, mYo;
    if (!map_store_2d(&mHo, h, (uint64_t)c.F, (uint64_t)max_rows) ||
        !map_halves_store(&mGUo, gu_keep ? gu_keep : h, (uint64_t)c.F, (uint64_t)max_rows) ||
        !map_store_2d(&mYo, y_perm, (uint64_t)c.D, (uint64_t)max_rows))
        return cudaErrorInvalidValue;
    const bool pair = use_pairs(c, max_rows);
    const int64_t bm = pair ? 256 : 128;
    const int64_t mtiles_bound = (max_rows + bm - 1) / bm + c.E;

    // each expert's A maps (x_perm for gate/up, h for down), rows ending at the expert's end
    CUtensorMap* gmaps = nullptr;
    if (amaps != nullptr && (reinterpret_cast<uintptr_t>(amaps) & 127u) == 0) {
        gmaps = static_cast<CUtensorMap*>(amaps);
        ffn_amaps_kernel<<<(c.E + 127) / 128, 128, 0, s>>>(mA, mH, offsets, c.E, max_rows, 0, gmaps);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    Args a1{offsets, perm, topk_w, static_cast<__nv_bfloat16*>(h), c.E, c.D, c.F,
            (c.F + 127) / 128, c.F, max_rows, c.T * c.K,
            static_cast<__nv_bfloat16*>(gu_keep), nullptr, status, gmaps};
    cudaError_t err = pair ? launch_one<kGateUp, true>(mA, mG, mU, mHo, mGUo, a1, mtiles_bound * a1.n_tiles, s)
                           : launch_one<kGateUp, false>(mA, mG, mU, mHo, mGUo, a1, mtiles_bound * a1.n_tiles, s);
    if (err != cudaSuccess) return err;
    if (mid) mid(mid_ctx, s);
    Args a2{offsets, perm, topk_w, static_cast<__nv_bfloat16*>(y_perm), c.E, c.F, c.D,
            (c.D + 255) / 256, c.D, max_rows, c.T * c.K, nullptr, nullptr, status,
            gmaps ? gmaps + c.E : nullptr};
    return pair ? launch_one<kDown, true>(mH, mD, mD, mYo, mYo, a2, mtiles_bound * a2.n_tiles, s)
                : launch_one<kDown, false>(mH, mD, mD, mYo, mYo, a2, mtiles_bound * a2.n_tiles, s);
}

cudaError_t launch_dgrad_tc_bf16(const moe_config& c, int64_t max_rows, const void* dyp,
                                 const int32_t* offsets, const void* gu, const void* w_gate,
                                 const void* w_up, const void* w_down, void* dgu, void* dxp,
                                 void* amaps, int* status, cudaStream_t s, StageHook mid, void* mid_ctx)
{
    using namespace tc;
    const bool pair = use_pairs(c, max_rows);
    const uint32_t brows = pair ? 128 : 256;  // K-major B rows per CTA
    CUtensorMap mA, mWd, mDGU, mG, mU;
    if (!map_2d(&mA, dyp, (uint64_t)c.D, (uint64_t)max_rows, 128) ||
        !map_3d_kmajor(&mWd, w_down, (uint64_t)c.D, (uint64_t)c.F, (uint64_t)c.E, brows) ||
        !map_halves(&mDGU, dgu, (uint64_t)c.F, (uint64_t)max_rows, 128) ||
        !map_3d_kmajor(&mG, w_gate, (uint64_t)c.F, (uint64_t)c.D, (uint64_t)c.E, brows) ||
        !map_3d_kmajor(&mU, w_up, (uint64_t)c.F, (uint64_t)c.D, (uint64_t)c.E, brows))
        return cudaErrorInvalidValue;
    // the epilogues' stores: [dg | du] viewed as (rows, 2, F), dXp (rows, D); and the dH
    // epilogue's loads of the kept [g | u] pieces, laid out like the [dg | du] stores
    CUtensorMap mOut, mXo, mGUin;
    if (!map_halves_store(&mOut, dgu, (uint64_t)c.F, (uint64_t)max_rows) ||
        !map_store_2d(&mXo, dxp, (uint64_t)c.D, (uint64_t)max_rows) ||
        !map_halves_store(&mGUin, gu, (uint64_t)c.F, (uint64_t)max_rows))
        return cudaErrorInvalidValue;
    const int64_t bm = pair ? 256 : 128;
    const int64_t mtiles_bound = (max_rows + bm - 1) / bm + c.E;
    // each expert's A maps (dYp for dH, [dg | du] for dX), rows ending at the expert's end
    CUtensorMap* gmaps = nullptr;
    if (amaps != nullptr && (reinterpret_cast<uintptr_t>(amaps) & 127u) == 0) {
        gmaps = static_cast<CUtensorMap*>(amaps);
        ffn_amaps_kernel<<<(c.E + 127) / 128, 128, 0, s>>>(mA, mDGU, offsets, c.E, max_rows, 1, gmaps);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // dH = dYp . Wd^T (K = D), epilogue through SwiGLU into [dg | du]
    Args a1{offsets, nullptr, nullptr, static_cast<__nv_bfloat16*>(dgu), c.E, c.D, c.F,
            (c.F + 255) / 256, 2 * (int64_t)c.F, max_rows, c.T * c.K, nullptr,
            static_cast<const __nv_bfloat16*>(gu), status, gmaps};
    cudaError_t err = pair ? launch_one<kDgradH, true>(mA, mWd, mWd, mOut, mGUin, a1, mtiles_bound * a1.n_tiles, s)
                           : launch_one<kDgradH, false>(mA, mWd, mWd, mOut, mGUin, a1, mtiles_bound * a1.n_tiles, s);
    if (err != cudaSuccess) return err;
    if (mid) mid(mid_ctx, s);
    // dXp = [dg | du] . [Wg | Wu]^T (K = 2F), unit weights
    Args a2{offsets, nullptr, nullptr, static_cast<__nv_bfloat16*>(dxp), c.E, c.F, c.D,
            (c.D + 255) / 256, c.D, max_rows, c.T * c.K, nullptr, nullptr, status,
            gmaps ? gmaps + c.E : nullptr};
    return pair ? launch_one<kDgradX, true>(mDGU, mG, mU, mXo, mXo, a2, mtiles_bound * a2.n_tiles, s)
                : launch_one<kDgradX, false>(mDGU, mG, mU, mXo, mXo, a2, mtiles_bound * a2.n_tiles, s);
}

}  // namespace moe
