// router_tc.cu -- router for bf16 layers on the tensor cores: the logits GEMM,
// softmax (or sigmoid scores), top-k, the routing weights and the router
// statistics, all in one kernel.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation": fp32
// router logits, softmax over the experts, top-k, weights divided by the sum
// of the selected probabilities; the statistics (mean probability, counts,
// logsumexp) feed the balance loss and the z-loss.
//
// fp32 logits on bf16 tensor cores: x is bf16 already, and each fp32 router
// weight is split exactly into three bf16 terms w = hi + mid + lo (hi =
// bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid): 3 x 8 significand
// bits cover fp32's 24).  Every product x*term is exact in fp32 and is
// accumulated in fp32 in tensor memory, so the logits carry fp32
// accumulation error only (no bf16 rounding of the weights).  The split is a
// function of the weight alone: router_prepare_kernel writes the terms once
// (terms[p][e][d], expert rows of d_model values, rows past E zero), and
// this kernel reads them by TMA like x.
//
// One CTA per 128 tokens (M = 128) and per split of d_model.  The three
// terms are stacked along N: one MMA per K step of 16 computes
// [x.hi | x.mid | x.lo] for all experts at once (N = 3 x EPN, EPN = E rounded
// up to 16, 32, 64 or 128; two MMAs when that exceeds 256), and the epilogue
// adds the three partial logits.  Warps:
//   warp 0      TMA: the x tiles (128 tokens x 64 of d_model, 128-byte
//               swizzle) into a deep ring (up to 10 stages of 16 KB)
//   warp 1      tcgen05.mma
//   warps 2..   lane 0 of warp 2: TMA of the weight terms of each K block
//               (3 x EPN rows x 64 of d_model, 128-byte swizzle) into a ring
//               of their own, so that the x ring keeps its depth.  Warps 2..5
//               read the accumulators out of tensor memory (each its lane
//               quadrant).  Then the epilogue: four warps with two CTAs per
//               SM (one token row per thread), eight with one CTA per SM (a
//               token's two threads take half of the experts each and meet
//               in shared memory): logits (+ partials of the other splits +
//               bias + noise), max and top-K by (logit + selection bias
//               desc, id asc, an unrolled insertion network), softmax sum
//               and entropy (closed form) and scores, the group limit when
//               set, weights, normalised scores, and the per-CTA statistics
//               (counts by shared-memory atomics; column sums in a fixed
//               order).
// When the token tiles alone leave most SMs idle, d_model is split over a
// cluster of CTAs along grid y: each non-leader CTA sends its partial logits
// to the leader's shared memory (distributed shared memory), and the leader
// adds them in split order and runs the epilogue.  With more token tiles
// than SMs, two CTAs share an SM (shallower rings).  The CTA whose
// statistics land last finishes them for the whole grid
// (router_stats.cuh).  Every wait is bounded.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "router_stats.cuh"

namespace moe {
namespace rtc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB x tile per stage
// Warps: 0 x TMA, 1 MMA, 2.. weight TMA (lane 0 of warp 2) and the epilogue:
// eight epilogue warps (two per tensor-memory lane quadrant, each taking half
// of the experts of its 32 tokens) with one CTA per SM, four with two CTAs.
template <int MINB> struct Threads {
    static constexpr int EPI_WARPS = MINB == 1 ? 8 : 4;
    static constexpr int HALVES = EPI_WARPS / 4;
    static constexpr int NTH = 32 * EPI_WARPS;  // epilogue threads
    static constexpr int NT = 64 + NTH;         // block size
};
constexpr int MAX_KM = 8;
constexpr int MAX_STAGES = 10;
constexpr int MAX_WSLOTS = 6;
constexpr int MAX_SPLITS = 4;

template <int EPN> struct Geo {
    static constexpr int TERM_BYTES = EPN * 128;       // one term: EPN expert rows x 64 d_model (bf16)
    static constexpr int W_BYTES = 3 * TERM_BYTES;     // the three terms of one K block
    static constexpr int NACC = 3 * EPN;               // accumulator columns [hi | mid | lo]
    static constexpr int N0 = NACC <= 256 ? NACC : 256;  // the first MMA's N
    static constexpr int N1 = NACC - N0;                 // the second's (EPN = 128: 128)
    static constexpr int TMEM_COLS = NACC <= 64 ? 64 : NACC <= 128 ? 128 : NACC <= 256 ? 256 : 512;
    static constexpr int LDS = EPN + 1;  // epilogue row stride in floats (odd: conflict-free)
};

struct Misc {
    uint64_t xfull[MAX_STAGES];   // x tile landed
    uint64_t xempty[MAX_STAGES];  // its MMAs are done
    uint64_t wfull[MAX_WSLOTS];   // weight terms landed
    uint64_t wempty[MAX_WSLOTS];  // their MMAs are done
    uint64_t tfull;
    uint32_t tmem_base;
    int abort_flag;
    int last;         // this CTA finishes the statistics of the grid
    int cnt[128];     // this CTA's expert counts
    float psum[256];  // chunk sums of the normalised scores
    float wz[4];      // per lane-quadrant sums of lse^2
    float wh[4];      // and of the entropy
    float bias_s[128];  // router bias (0 when none)
    float sel_s[128];   // selection bias (0 when none)
};

struct Args {
    RouteOpts o;
    const float* bias;        // E or null
    const float* noise;       // T x E or null
    float* logits_out;        // T x E or null
    float* probs_out;         // T x E or null
    int32_t* ids;             // T x K
    float* wout;              // T x K
    float* blk_mp;            // tiles x E
    float* blk_z;             // tiles
    float* blk_ent;           // tiles
    int32_t* blk_cnt;         // tiles x E
    float* mean_prob;         // E or null
    float* losses;            // 3 or null
    int* counter;             // finished-CTA counter (zero between launches)
    int64_t T;
    int D, E, K;
    int with_stats;
    int* status;
    int stages;               // depth of the x ring (16 KB stages)
    int wslots;               // depth of the weight-term ring
    uint32_t w_off;           // the weight-term ring (wslots x W_BYTES), right after the x ring
    int splits;               // CTAs per token tile (cluster size along y)
    int split_kb;             // K blocks per split
    uint32_t misc_off;        // byte offsets in the aligned shared memory
    uint32_t recv_off;        // (splits - 1) x BM x EPN fp32 partial logits (leader)
};

// barrier of the NTH epilogue threads
template <int NTH> MOE_DEVICE void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NTH) : "memory"); }

MOE_DEVICE void st_cluster_f32(uint32_t cluster_addr, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}

// terms[p][e][d] = the p-th bf16 term of W_r[d][e] (p = 0 hi, 1 mid, 2 lo);
// rows e >= E are zero.  Two consecutive d per thread (D is even).
__global__ void router_prepare_kernel(const float* __restrict__ w, __nv_bfloat16* __restrict__ terms,
                                      int D, int E, int EPN)
{
    const int64_t half = (int64_t)D / 2;
    const int64_t n = (int64_t)EPN * half;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(i / half);
        const int d = (int)(i % half) * 2;
        const float a = e < E ? w[(int64_t)d * E + e] : 0.f;
        const float b = e < E ? w[(int64_t)(d + 1) * E + e] : 0.f;
        const __nv_bfloat162 hi = __floats2bfloat162_rn(a, b);
        const float2 hf = __bfloat1622float2(hi);
        const float ra = a - hf.x, rb = b - hf.y;  // exact
        const __nv_bfloat162 mid = __floats2bfloat162_rn(ra, rb);
        const float2 mf = __bfloat1622float2(mid);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(ra - mf.x, rb - mf.y);
        const int64_t o = (int64_t)e * D + d;
        const int64_t plane = (int64_t)EPN * D;
        *reinterpret_cast<__nv_bfloat162*>(terms + o) = hi;
        *reinterpret_cast<__nv_bfloat162*>(terms + plane + o) = mid;
        *reinterpret_cast<__nv_bfloat162*>(terms + 2 * plane + o) = lo;
    }
}

// The three partial logits of accumulator columns e, EPN + e and 2 EPN + e,
// added (hi + mid) + lo.
template <int EPN>
MOE_DEVICE void read_logits(uint32_t taddr, bool ok, float* dst_local, uint32_t dst_remote, bool remote)
{
    auto put = [&](int e, float v) {
        if (remote) st_cluster_f32(dst_remote + e * 4, v);
        else dst_local[e] = v;
    };
    if (EPN == 16) {
        uint32_t v0[32], v1[32];
        tmem_ld_32x32b_x32(taddr, v0);       // hi 0..15, mid 0..15
        tmem_ld_32x32b_x32(taddr + 32, v1);  // lo 0..15 (columns 48..63 unused)
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float L = (__uint_as_float(v0[e]) + __uint_as_float(v0[16 + e])) + __uint_as_float(v1[e]);
            put(e, ok ? L : 0.f);
        }
    } else {
#pragma unroll 1
        for (int c = 0; c < EPN / 32; ++c) {
            uint32_t h[32], m[32], l[32];
            tmem_ld_32x32b_x32(taddr + c * 32, h);
            tmem_ld_32x32b_x32(taddr + EPN + c * 32, m);
            tmem_ld_32x32b_x32(taddr + 2 * EPN + c * 32, l);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float L = (__uint_as_float(h[j]) + __uint_as_float(m[j])) + __uint_as_float(l[j]);
                put(c * 32 + j, ok ? L : 0.f);
            }
        }
    }
}

template <int EPN, int KM, int MINB>
__global__ void __launch_bounds__(Threads<MINB>::NT, MINB)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const Args a)
{
    using G = Geo<EPN>;
    using TH = Threads<MINB>;
    constexpr int LDS = G::LDS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* xring = smem;              // S x 16 KB, then the weight ring: together the epilogue's scratch
    uint8_t* wring = smem + a.w_off;    // WS x W_BYTES
    Misc* m = reinterpret_cast<Misc*>(smem + a.misc_off);
    float* recv = reinterpret_cast<float*>(smem + a.recv_off);
    const int S = a.stages, WS = a.wslots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * BM;
    const int split = (int)blockIdx.y;  // the CTA's rank in its cluster when splits > 1
    const int num_kb = (a.D + BK - 1) / BK;
    const int kb_begin = split * a.split_kb;                // never empty (host guarantee)
    const int kb_end = min(num_kb, kb_begin + a.split_kb);
    const int nkb = kb_end - kb_begin;
    const int E = a.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&m->xfull[s], 1);
            mbar_init(&m->xempty[s], 1);
        }
        for (int j = 0; j < WS; ++j) {
            mbar_init(&m->wfull[j], 1);
            mbar_init(&m->wempty[j], 1);
        }
        mbar_init(&m->tfull, 1);
        m->abort_flag = 0;
        m->last = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
    }
    if (warp >= 2 && threadIdx.x - 64 < 128) m->cnt[threadIdx.x - 64] = 0;
    if (warp == 1) {
        tmem_alloc(&m->tmem_base, G::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    volatile int* abort_flag = &m->abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ x tiles, S stages ahead
            int stage = 0;
            uint32_t phase = 0;
            int last_phase[MAX_STAGES];
            for (int s = 0; s < MAX_STAGES; ++s) last_phase[s] = -1;
            for (int i = 0; i < nkb; ++i) {
                if (!mbar_wait(&m->xempty[stage], phase ^ 1u, a.status, 510, abort_flag)) break;
                mbar_arrive_expect_tx(&m->xfull[stage], A_BYTES);
                tma_load_2d(xring + (size_t)stage * A_BYTES, &tmX, (kb_begin + i) * BK, (int32_t)t0,
                            &m->xfull[stage]);
                last_phase[stage] = (int)phase;
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // every copy issued has landed before the ring is reused or the CTA exits
            for (int s = 0; s < S; ++s)
                if (last_phase[s] >= 0)
                    mbar_wait(&m->xfull[s], (uint32_t)last_phase[s], a.status, 511, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc0 = umma_idesc_bf16(BM, G::N0, 0, 0);
            constexpr uint32_t idesc1 = umma_idesc_bf16(BM, G::N1 > 0 ? G::N1 : 16, 0, 0);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % S, j = i % WS;
                if (!mbar_wait(&m->xfull[s], (uint32_t)((i / S) & 1), a.status, 520, abort_flag)) break;
                if (!mbar_wait(&m->wfull[j], (uint32_t)((i / WS) & 1), a.status, 521, abort_flag)) break;
                tc_fence_after();
                const uint32_t sA = smem_u32(xring + (size_t)s * A_BYTES);
                const uint32_t sB = smem_u32(wring + (size_t)j * G::W_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t acc = (i || kk) ? 1u : 0u;
                    // both operands K-major: 8-row groups 1024 B apart, +32 B per 16-element K step
                    const uint64_t adesc = umma_desc_sw128(sA + kk * 32, 16, 1024);
                    umma_f16_ss(tmem_base, adesc, umma_desc_sw128(sB + kk * 32, 16, 1024), idesc0, acc);
                    if (G::N1 > 0)  // weight rows 256 .. 3 EPN - 1 into columns 256 ..
                        umma_f16_ss(tmem_base + 256, adesc, umma_desc_sw128(sB + 256 * 128 + kk * 32, 16, 1024),
                                    idesc1, acc);
                }
                umma_commit(&m->xempty[s]);
                umma_commit(&m->wempty[j]);
            }
            umma_commit(&m->tfull);  // also the drain: every MMA done once it fires
        }
    } else {
        if (warp == 2 && lane == 0) {
            // ------------------------------------------------ weight terms, WS slots ahead
            int slot = 0;
            uint32_t phase = 0;
            int last_phase[MAX_WSLOTS];
            for (int j = 0; j < MAX_WSLOTS; ++j) last_phase[j] = -1;
            for (int i = 0; i < nkb; ++i) {
                if (!mbar_wait(&m->wempty[slot], phase ^ 1u, a.status, 540, abort_flag)) break;
                mbar_arrive_expect_tx(&m->wfull[slot], G::W_BYTES);
                tma_load_3d(wring + (size_t)slot * G::W_BYTES, &tmW, (kb_begin + i) * BK, 0, 0,
                            &m->wfull[slot]);
                last_phase[slot] = (int)phase;
                if (++slot == WS) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            for (int j = 0; j < WS; ++j)
                if (last_phase[j] >= 0)
                    mbar_wait(&m->wfull[j], (uint32_t)last_phase[j], a.status, 541, nullptr);
        }
        __syncwarp();
        if (warp < 6) {
            // -------------------------------------------- accumulators out of tensor memory
            const int quad = warp & 3;        // the lane quadrant this warp may read
            const int r = quad * 32 + lane;   // token row in the tile
            float* Ls = reinterpret_cast<float*>(xring);  // [BM][LDS]
            // tcgen05.ld is warp-collective: the vote keeps the warp converged
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&m->tfull, 0, a.status, 530, abort_flag));
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16);
            uint32_t remote = 0;
            if (split > 0)  // this row's slot in the leader's receive buffer
                remote = mapa_shared(smem_u32(recv + ((size_t)(split - 1) * BM + r) * EPN), 0);
            read_logits<EPN>(taddr, ok, Ls + r * LDS, remote, split > 0);
        } else {
            // the second epilogue warp of each quadrant: the rings are the
            // epilogue's scratch only once every MMA (and so every copy) is done
            mbar_wait(&m->tfull, 0, a.status, 531, abort_flag);
        }
    }
    __syncwarp();
    if (a.splits > 1) cluster_sync();  // the other splits' partials are in the leader's buffer

    if (warp >= 2 && split == 0) {
        // ------------------------------------------------ epilogue: one token row per thread
        // (with two warps per lane quadrant, each of the row's two threads takes
        // half of the experts and the halves meet in shared memory)
        constexpr int HALVES = TH::HALVES, NTH = TH::NTH;
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = quad * 32 + lane;
        const int tid = threadIdx.x - 64;
        const int64_t t = t0 + r;
        const bool valid = t < a.T;
        const int K = a.K;
        const RouteOpts& o = a.o;
        float* Ls = reinterpret_cast<float*>(xring);  // logits, then normalised scores
        float* Xs = Ls + BM * LDS;                     // scores: exp(L - max), or sigmoid(L)
        float* Ns = Xs + BM * LDS;                     // this tile's logit noise
        float* Xc = Ns + BM * LDS;                     // the halves' exchange (two halves only)
        float* xm = Xc;                                // [BM] row maximum
        float* xp = Xc + BM;                           // [3][BM] partial sums, then [BM] scale
        float* xv = Xc + 4 * BM;                       // [BM][KM] the second half's top-K values
        int* xi = reinterpret_cast<int*>(Xc + (4 + KM) * BM);  // and ids
        const int G = o.n_groups, gsz = E / G;
        const int rows = a.T - t0 < BM ? (int)(a.T - t0) : BM;  // tokens of this tile
        const int eh = (E + HALVES - 1) / HALVES;               // this thread's experts [e0, e1)
        const int e0 = half * eh, e1 = e0 + eh < E ? e0 + eh : E;
        // the biases, and the tile's noise rows (one contiguous block, read coalesced)
        for (int e = tid; e < E; e += NTH) {
            m->bias_s[e] = a.bias ? a.bias[e] : 0.f;
            m->sel_s[e] = o.sel_bias ? o.sel_bias[e] : 0.f;
        }
        if (a.noise) {
            // eight loads in flight per thread, then their stores
            const float* src = a.noise + t0 * E;
            const int n = rows * E;
            for (int i0 = 0; i0 < n; i0 += 8 * NTH) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + u * NTH + tid;
                    v[u] = i < n ? __ldcs(src + i) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + u * NTH + tid;
                    if (i < n) {
                        const int rr = i / E;
                        Ns[rr * LDS + (i - rr * E)] = v[u];
                    }
                }
            }
        }
        epi_sync<NTH>();
        // top-K by (u desc, id asc), u = L + selection bias: an unrolled insertion
        // network of KM >= K slots (a displaced entry carried down keeps that order)
        float tv[KM];
        int ti[KM];
#pragma unroll
        for (int k = 0; k < KM; ++k) {
            tv[k] = -INFINITY;
            ti[k] = 0x7fffffff;
        }
        auto insert = [&](float xv_, int xi_) {
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                const bool gt = xv_ > tv[k] || (xv_ == tv[k] && xi_ < ti[k]);
                const float nv = gt ? xv_ : tv[k];
                const int ni = gt ? xi_ : ti[k];
                xv_ = gt ? tv[k] : xv_;
                xi_ = gt ? ti[k] : xi_;
                tv[k] = nv;
                ti[k] = ni;
            }
        };
        // pass 1: logits (own K range + the other splits in order, + bias + noise),
        // their maximum, and (without a group limit) the top-K
        if (a.splits > 1 || a.bias || (a.noise && valid)) {
            // the complete logits first, so that the top-K loop below stays lean
            float* Lr = Ls + r * LDS;
            for (int sp = 1; sp < a.splits; ++sp) {
                const float* Pr = recv + ((size_t)(sp - 1) * BM + r) * EPN;
#pragma unroll 4
                for (int e = e0; e < e1; ++e) Lr[e] += Pr[e];
            }
            if (a.bias) {
#pragma unroll 4
                for (int e = e0; e < e1; ++e) Lr[e] += m->bias_s[e];
            }
            if (a.noise && valid) {
#pragma unroll 4
                for (int e = e0; e < e1; ++e) Lr[e] += Ns[r * LDS + e];
            }
        }
        float mx = -INFINITY;
        if (G == 1) {
#pragma unroll 8
            for (int e = e0; e < e1; ++e) {
                const float L = Ls[r * LDS + e];
                mx = fmaxf(mx, L);
                insert(L + m->sel_s[e], e);
            }
        } else {
#pragma unroll 8
            for (int e = e0; e < e1; ++e) mx = fmaxf(mx, Ls[r * LDS + e]);
        }
        if (HALVES == 2) {
            // the second half hands its maximum and its top-K to the first
            if (half == 1) {
                xm[r] = mx;
#pragma unroll
                for (int k = 0; k < KM; ++k) {
                    xv[r * KM + k] = tv[k];
                    xi[r * KM + k] = ti[k];
                }
            }
            epi_sync<NTH>();
            if (half == 0) {
                mx = fmaxf(mx, xm[r]);
                if (G == 1) {
#pragma unroll
                    for (int k = 0; k < KM; ++k) insert(xv[r * KM + k], xi[r * KM + k]);
                }
            }
            epi_sync<NTH>();
            if (half == 0) xm[r] = mx;  // the row maximum back to the second half
            epi_sync<NTH>();
            if (half == 1) mx = xm[r];
        } else if (a.logits_out) {
            epi_sync<NTH>();
        }
        if (a.logits_out) {  // the tile's logits, one contiguous block, written coalesced
            float* dst = a.logits_out + t0 * E;
            for (int i = tid; i < rows * E; i += NTH) {
                const int rr = i / E;
                dst[i] = Ls[rr * LDS + (i - rr * E)];
            }
            // every row is copied before pass 3 rewrites its logits (with two halves
            // the exchange's barriers below already order the two)
            if (HALVES == 1) epi_sync<NTH>();
        }
        // pass 2: softmax sum, sum of exp(L - max) (L - max) for the entropy, and
        // the scores (sigmoid scores and their sum with score_func sigmoid)
        float ssum = 0.f, s1 = 0.f, scsum = 0.f;
#pragma unroll 4
        for (int e = e0; e < e1; ++e) {
            const float L = Ls[r * LDS + e];
            const float x = __expf(L - mx);
            ssum += x;
            s1 = fmaf(x, L - mx, s1);
            float sc = x;
            if (o.score_func == 1) {
                sc = 1.0f / (1.0f + __expf(-L));
                scsum += sc;
            }
            Xs[r * LDS + e] = sc;
        }
        if (HALVES == 2) {
            if (half == 1) {
                xp[r] = ssum;
                xp[BM + r] = s1;
                xp[2 * BM + r] = scsum;
            }
            epi_sync<NTH>();
            if (half == 0) {  // the halves' sums, first half first
                ssum += xp[r];
                s1 += xp[BM + r];
                scsum += xp[2 * BM + r];
            }
        }
        float scinv = 0.f, lss = 0.f, ent = 0.f;
        if (half == 0) {
            const float inv = 1.0f / ssum;
            lss = logf(ssum);
            // entropy -sum q log q = log(sum) - sum q (L - max), q = exp(L - max) / sum
            ent = lss - s1 * inv;
            // softmax scores are Xs * inv, sigmoid scores Xs itself
            const float sc_mul = o.score_func == 1 ? 1.0f : inv;
            if (G > 1) {
                // group limit: a group's score is its best selection score u = L + b
                float gm[32];
#pragma unroll
                for (int g = 0; g < 32; ++g) {
                    gm[g] = -INFINITY;
                    if (g < G)
                        for (int e = g * gsz; e < (g + 1) * gsz; ++e)
                            gm[g] = fmaxf(gm[g], Ls[r * LDS + e] + m->sel_s[e]);
                }
                uint32_t keep = 0;
                for (int rr = 0; rr < o.topk_groups; ++rr) {
                    float bv = -INFINITY;
                    int bg = 0;
#pragma unroll
                    for (int g = 0; g < 32; ++g)
                        if (g < G && !((keep >> g) & 1u) && gm[g] > bv) {  // strict: lower group id on ties
                            bv = gm[g];
                            bg = g;
                        }
                    keep |= 1u << bg;
                }
                for (int e = 0; e < E; ++e)
                    if ((keep >> (e / gsz)) & 1u) insert(Ls[r * LDS + e] + m->sel_s[e], e);
            }
            // weights from the scores of the selected experts
            float sk[KM];
            float ssel = 0.f;
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                sk[k] = k < K ? Xs[r * LDS + ti[k]] * sc_mul : 0.f;
                ssel += sk[k];
            }
            if (valid) {
#pragma unroll
                for (int k = 0; k < KM; ++k)
                    if (k < K) {
                        a.ids[t * K + k] = ti[k];
                        a.wout[t * K + k] = (o.renorm ? sk[k] / ssel : sk[k]) * o.route_scale;
                        if (a.with_stats) atomicAdd(&m->cnt[ti[k]], 1);  // integer: order-free
                    }
            }
            scinv = o.score_func == 1 ? 1.0f / scsum : inv;
        }
        if (HALVES == 2) {
            epi_sync<NTH>();  // the second half has read its partial sums
            if (half == 0) xp[r] = scinv;
            epi_sync<NTH>();
            if (half == 1) scinv = xp[r];
        }
        // pass 3: normalised scores into Ls (and probs_out); rows past T give nothing
#pragma unroll 4
        for (int e = e0; e < e1; ++e) {
            const float pn = Xs[r * LDS + e] * scinv;
            Ls[r * LDS + e] = valid ? pn : 0.f;
        }
        if (a.probs_out) {  // one contiguous block, written coalesced
            epi_sync<NTH>();
            float* dst = a.probs_out + t0 * E;
            for (int i = tid; i < rows * E; i += NTH) {
                const int rr = i / E;
                dst[i] = Ls[rr * LDS + (i - rr * E)];
            }
        }
        if (a.with_stats) {
            // per-CTA statistics, each in a fixed order
            if (half == 0) {
                const float lse = mx + lss;
                float z = valid ? lse * lse : 0.f, h = valid ? ent : 0.f;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    z += __shfl_xor_sync(0xffffffffu, z, off);
                    h += __shfl_xor_sync(0xffffffffu, h, off);
                }
                if (lane == 0) {
                    m->wz[quad] = z;
                    m->wh[quad] = h;
                }
            }
            epi_sync<NTH>();
            constexpr int CH = NTH / EPN;  // row chunks per column (EPN x CH = NTH threads)
            constexpr int RC = BM / CH;
            {
                const int col = tid % EPN, ch = tid / EPN;
                float sp = 0.f;
                if (col < E)
                    for (int rr = ch * RC; rr < (ch + 1) * RC; ++rr) sp += Ls[rr * LDS + col];
                m->psum[ch * EPN + col] = sp;
            }
            epi_sync<NTH>();
            if (tid < E) {
                float sp = 0.f;
                for (int ch = 0; ch < CH; ++ch) sp += m->psum[ch * EPN + tid];
                a.blk_mp[(size_t)blockIdx.x * E + tid] = sp;
                a.blk_cnt[(size_t)blockIdx.x * E + tid] = m->cnt[tid];
            }
            if (tid == 0) {
                a.blk_z[blockIdx.x] = ((m->wz[0] + m->wz[1]) + m->wz[2]) + m->wz[3];
                a.blk_ent[blockIdx.x] = ((m->wh[0] + m->wh[1]) + m->wh[2]) + m->wh[3];
            }
            __threadfence();
            epi_sync<NTH>();
            if (tid == 0) m->last = atomicAdd(a.counter, 1) == (int)gridDim.x - 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (split == 0 && a.with_stats && m->last) {
        // the last CTA: the statistics of the whole grid (all its threads)
        __threadfence();
        double* sd = reinterpret_cast<double*>(xring);
        long long* sc = reinterpret_cast<long long*>(sd + kStatD);
        finish_router_stats(a.blk_mp, a.blk_z, a.blk_ent, a.blk_cnt, (int)gridDim.x, a.T, E, a.K,
                            a.mean_prob, a.losses, sd, sc, TH::NT, (int)threadIdx.x,
                            [] { __syncthreads(); });
        if (threadIdx.x == 0) *a.counter = 0;
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, G::TMEM_COLS);
    }
}

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

// Ring depths and shared-memory layout for `ctas_per_sm` CTAs on each SM:
// [x ring: stages x 16 KB][weight terms: wslots x 3 x EPN x 128][Misc][split
// partials]; the two rings together are the epilogue's scratch.
struct Plan {
    int epn, splits, split_kb, ctas_per_sm, stages, wslots;
    uint32_t w_off, misc_off, recv_off;
    size_t smem;  // dynamic shared memory, with 1 KB of alignment slack
};

static int epn_of(int E) { return E <= 16 ? 16 : E <= 32 ? 32 : E <= 64 ? 64 : 128; }

static Plan make_plan(const moe_config& c, bool noise)
{
    Plan p{};
    p.epn = epn_of(c.E);
    const int tiles = router_tc_blocks(c);
    const int nkb = (c.D + BK - 1) / BK;
    const size_t w_bytes = (size_t)3 * p.epn * 128;
    const size_t misc = align_up(sizeof(Misc), 1024);
    // the epilogue scratch (and the statistics' last step) live in the rings:
    // logits, scores and noise rows ([BM][EPN + 1] fp32 each), and with one CTA
    // per SM (two epilogue threads per row) the halves' exchange, (4 + 2 KM) x BM words
    const size_t epi2 = (size_t)(noise ? 3 : 2) * BM * (p.epn + 1) * sizeof(float);
    const size_t epi1 = ((size_t)3 * BM * (p.epn + 1) + (size_t)(4 + 2 * MAX_KM) * BM) * sizeof(float);
    const size_t fin = (size_t)kStatD * sizeof(double) + (size_t)kStatC * sizeof(long long);
    // the weight ring takes up to about 45 % of the budget (its tiles come from
    // L2: a few in flight cover that latency), the x ring the rest
    auto fit = [&](size_t budget, size_t fixed, size_t epi, int& st, int& ws) {
        st = ws = 0;
        if (budget <= fixed) return false;
        const size_t room = budget - fixed;
        ws = (int)(room * 45 / 100 / w_bytes);
        if (ws > MAX_WSLOTS) ws = MAX_WSLOTS;
        if (ws < 2) ws = 2;
        if ((size_t)ws * w_bytes >= room) return false;
        st = (int)((room - (size_t)ws * w_bytes) / A_BYTES);
        if (st > MAX_STAGES) st = MAX_STAGES;
        const size_t rings = (size_t)st * A_BYTES + (size_t)ws * w_bytes;
        return st >= 3 && rings >= epi && rings >= fin;
    };
    // the d_model split the token tiles ask for, fewer when its partial logits
    // (received by each tile's leader) leave the rings too little room; one
    // split always fits (E <= 128)
    size_t recv = 0;
    int st = 0, ws = 0;
    for (int want = router_tc_splits(c); want >= 1; --want) {
        const int per = (nkb + want - 1) / want;  // K blocks per split: every split non-empty
        p.splits = (nkb + per - 1) / per;
        recv = (size_t)(p.splits - 1) * BM * p.epn * sizeof(float);
        const size_t fixed = 1024 + misc + align_up(recv, 1024);
        // two CTAs per SM when the tiles outnumber the SMs and each still gets 3 x stages
        p.ctas_per_sm = 2;
        if (tiles * p.splits > 148 && p.epn <= 64 && fit(112 * 1024, fixed, epi2, st, ws)) break;
        p.ctas_per_sm = 1;
        if (fit(226 * 1024, fixed, epi1, st, ws)) break;
        st = 0;  // no fit: the launcher rejects fewer than 3 stages (unreachable for E <= 128)
    }
    p.split_kb = (nkb + p.splits - 1) / p.splits;
    p.stages = st;
    p.wslots = ws;
    p.w_off = (uint32_t)((size_t)p.stages * A_BYTES);
    p.misc_off = p.w_off + (uint32_t)((size_t)p.wslots * w_bytes);
    p.recv_off = p.misc_off + (uint32_t)misc;
    p.smem = (size_t)p.recv_off + align_up(recv, 1024) + 1024;
    return p;
}

template <int EPN, int KM, int MINB>
static cudaError_t launch_t(const moe_config& c, const CUtensorMap& mX, const CUtensorMap& mW, const Args& a,
                            const Plan& p, cudaStream_t s)
{
    auto kern = router_tc_kernel<EPN, KM, MINB>;
    static PerDeviceFlag smem_set;
    // the largest ring this instance is launched with (one attribute per device)
    cudaError_t ae = opt_in_smem(smem_set, reinterpret_cast<const void*>(kern),
                                 MINB == 2 ? 113 * 1024 : 227 * 1024);
    if (ae != cudaSuccess) return ae;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)router_tc_blocks(c), (unsigned)p.splits, 1);
    cfg.blockDim = dim3(Threads<MINB>::NT, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)p.splits;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.splits > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, mX, mW, a);
}

template <int EPN>
static cudaError_t launch_k(const moe_config& c, const CUtensorMap& mX, const CUtensorMap& mW, const Args& a,
                            const Plan& p, cudaStream_t s)
{
    const int km = c.K <= 2 ? 2 : c.K <= 4 ? 4 : c.K <= 6 ? 6 : 8;
    if (p.ctas_per_sm == 2) {
        if constexpr (EPN <= 64) {
            return km == 2 ? launch_t<EPN, 2, 2>(c, mX, mW, a, p, s)
                 : km == 4 ? launch_t<EPN, 4, 2>(c, mX, mW, a, p, s)
                 : km == 6 ? launch_t<EPN, 6, 2>(c, mX, mW, a, p, s)
                           : launch_t<EPN, 8, 2>(c, mX, mW, a, p, s);
        }
        return cudaErrorInvalidValue;
    }
    return km == 2 ? launch_t<EPN, 2, 1>(c, mX, mW, a, p, s)
         : km == 4 ? launch_t<EPN, 4, 1>(c, mX, mW, a, p, s)
         : km == 6 ? launch_t<EPN, 6, 1>(c, mX, mW, a, p, s)
                   : launch_t<EPN, 8, 1>(c, mX, mW, a, p, s);
}

}  // namespace rtc

bool router_tc_eligible(const moe_config& c)
{
    return c.dtype == MOE_BF16 && c.E <= 128 && c.T >= 2048;
}

int router_tc_blocks(const moe_config& c) { return (int)((c.T + rtc::BM - 1) / rtc::BM); }

int router_tc_splits(const moe_config& c)
{
    // Split the contraction over d_model when the token tiles alone leave most
    // SMs idle (a large d_model with few tokens): up to 4 splits of at least
    // 8 K blocks each, so that tiles x splits stays within one wave.
    const int tiles = router_tc_blocks(c);
    const int nkb = (c.D + rtc::BK - 1) / rtc::BK;
    int sp = 148 / (tiles > 0 ? tiles : 1);
    if (sp > rtc::MAX_SPLITS) sp = rtc::MAX_SPLITS;
    if (sp > nkb / 8) sp = nkb / 8;
    if (sp < 2) return 1;
    const int per = (nkb + sp - 1) / sp;  // K blocks per split; every split non-empty
    return (nkb + per - 1) / per;
}

size_t router_terms_bytes(const moe_config& c)
{
    if (c.dtype != MOE_BF16 || c.E > 128) return 0;
    return (size_t)3 * rtc::epn_of(c.E) * (size_t)c.D * 2;
}

cudaError_t launch_router_prepare(const moe_config& c, const float* w_router, void* terms, cudaStream_t s)
{
    const int epn = rtc::epn_of(c.E);
    const int64_t n = (int64_t)epn * (c.D / 2);
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    rtc::router_prepare_kernel<<<(unsigned)blocks, 256, 0, s>>>(
        w_router, static_cast<__nv_bfloat16*>(terms), c.D, c.E, epn);
    return cudaGetLastError();
}

cudaError_t launch_router_tc(const moe_config& c, const RouteOpts& o, const void* x, const void* terms,
                             const float* bias, const float* noise, float* logits_out, float* probs_out,
                             int32_t* ids, float* w, float* blk_mp, float* blk_z, float* blk_ent,
                             int32_t* blk_cnt, float* mean_prob, float* losses, int* status, cudaStream_t s)
{
    using namespace rtc;
    const Plan p = make_plan(c, noise != nullptr);
    if (p.stages < 3) return cudaErrorInvalidConfiguration;
    EncodeTiledFn enc = encoder();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap mX, mW;
    {
        cuuint64_t dims[2] = {(cuuint64_t)c.D, (cuuint64_t)c.T};
        cuuint64_t strides[1] = {(cuuint64_t)c.D * 2};
        cuuint32_t box[2] = {64, BM};
        cuuint32_t es[2] = {1, 1};
        if (enc(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        // terms[p][e][d]: box = 64 d_model x EPN experts x 3 terms, stacked in
        // shared memory as 3 x EPN K-major rows of 128 bytes
        cuuint64_t dims[3] = {(cuuint64_t)c.D, (cuuint64_t)p.epn, 3};
        cuuint64_t strides[2] = {(cuuint64_t)c.D * 2, (cuuint64_t)p.epn * c.D * 2};
        cuuint32_t box[3] = {64, (cuuint32_t)p.epn, 3};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&mW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(terms), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    Args a{};
    a.o = o;
    a.bias = bias;
    a.noise = noise;
    a.logits_out = logits_out;
    a.probs_out = probs_out;
    a.ids = ids;
    a.wout = w;
    a.blk_mp = blk_mp;
    a.blk_z = blk_z;
    a.blk_ent = blk_ent;
    a.blk_cnt = blk_cnt;
    a.mean_prob = mean_prob;
    a.losses = losses;
    a.counter = status + kRouterCounterWord;
    a.T = c.T;
    a.D = c.D;
    a.E = c.E;
    a.K = c.K;
    a.with_stats = (mean_prob != nullptr || losses != nullptr) ? 1 : 0;
    a.status = status;
    a.stages = p.stages;
    a.wslots = p.wslots;
    a.w_off = p.w_off;
    a.splits = p.splits;
    a.split_kb = p.split_kb;
    a.misc_off = p.misc_off;
    a.recv_off = p.recv_off;
    switch (p.epn) {
        case 16: return launch_k<16>(c, mX, mW, a, p, s);
        case 32: return launch_k<32>(c, mX, mW, a, p, s);
        case 64: return launch_k<64>(c, mX, mW, a, p, s);
        default: return launch_k<128>(c, mX, mW, a, p, s);
    }
}

}  // namespace moe
