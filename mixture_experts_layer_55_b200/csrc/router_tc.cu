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
// bits cover fp32's 24).  Every product x*term is exact in fp32, and the
// three MMAs of a K step accumulate in fp32 in tensor memory, so the logits
// carry fp32 accumulation error only (no bf16 rounding of the weights).
//
// One CTA per 128 tokens (M = 128) and per split of d_model; N = EPN, the
// expert count rounded up to 16, 32, 64 or 128.  Warps:
//   warp 0      TMA: the x tiles (128 tokens x 64 of d_model, 128-byte
//               swizzle) into a deep ring (up to 10 stages of 16 KB)
//   warp 1      tcgen05.mma, three per K step of 16 (one per weight term)
//   warps 2..5  first the weight split: the 64 x E fp32 slice of W_r of each
//               K block arrives by bulk copy in a shallow ring of its own,
//               is split in shared memory into its three bf16 terms and
//               written K-major (expert rows of 64 d_model values, 128-byte
//               swizzle) into a shallow ring of weight tiles, so no weight
//               kernel runs before this one, the weight tiles are E rows
//               wide, not a padded 64, and the x ring keeps its depth; then
//               the epilogue, one token row per
//               thread: logits (+ bias + noise), max and top-K by (logit +
//               selection bias desc, id asc, an unrolled insertion network)
//               in one pass over the experts, softmax sum and entropy
//               (closed form) and scores in a second, the group limit when
//               set, weights, normalised scores in a third, and the per-CTA
//               statistics (counts by shared-memory atomics; column sums
//               in a fixed order).
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
constexpr int NUM_THREADS = 192;      // warp 0 TMA, warp 1 MMA, warps 2..5 weights + epilogue
constexpr int MAX_STAGES = 10;
constexpr int MAX_SPLITS = 4;
constexpr int CONVERTER_WARPS = 4;

template <int EPN> struct Geo {
    static constexpr int TERM_BYTES = EPN * 128;  // EPN expert rows x 64 d_model (bf16)
    static constexpr int B_BYTES = 3 * TERM_BYTES;
    static constexpr int TMEM_COLS = EPN < 32 ? 32 : EPN;
    static constexpr int LDS = EPN + 1;  // epilogue row stride in floats (odd: conflict-free)
};

constexpr int WDEPTH = 2;  // slots of the weight rings (fp32 slices and their bf16 terms)

struct Misc {
    uint64_t xfull[MAX_STAGES];   // x tile landed
    uint64_t xempty[MAX_STAGES];  // its MMAs are done
    uint64_t wl[WDEPTH];          // fp32 weight slice landed
    uint64_t bfull[WDEPTH];       // its bf16 terms are written
    uint64_t bempty[WDEPTH];      // their MMAs are done
    uint64_t wfree[WDEPTH];       // every weight warp is done reading the fp32 slice
    uint64_t tfull;
    uint32_t tmem_base;
    int abort_flag;
    int last;         // this CTA finishes the statistics of the grid
    int cnt[128];     // this CTA's expert counts
    float psum[128];  // chunk sums of the normalised scores
    float wz[4];      // per lane-quadrant sums of lse^2
    float wh[4];      // and of the entropy
};

struct Args {
    RouteOpts o;
    const float* w;           // W_r (D, E) fp32
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
    uint32_t b_off;           // the bf16 weight-term ring (WDEPTH x 3 x EPN x 128 bytes)
    uint32_t w_off;           // the fp32 weight-slice ring (WDEPTH x w_slot bytes)
    uint32_t w_slot;          // bytes per fp32 slice slot (64 x E x 4, rounded up)
    int splits;               // CTAs per token tile (cluster size along y)
    int split_kb;             // K blocks per split
    uint32_t misc_off;        // byte offsets in the aligned shared memory
    uint32_t recv_off;        // (splits - 1) x BM x EPN fp32 partial logits (leader)
};

MOE_DEVICE void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

MOE_DEVICE void st_cluster_f32(uint32_t cluster_addr, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}

// The three bf16 terms of two fp32 weights, packed in pairs (a in the low
// half): hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid), each pair
// rounded by one paired conversion.
MOE_DEVICE uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }
MOE_DEVICE void split3(float a, float b, uint32_t& hi, uint32_t& mid, uint32_t& lo)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const float ra = a - hf.x, rb = b - hf.y;
    const __nv_bfloat162 m = __floats2bfloat162_rn(ra, rb);
    const float2 mf = __bfloat1622float2(m);
    const __nv_bfloat162 l = __floats2bfloat162_rn(ra - mf.x, rb - mf.y);
    hi = bf16x2_bits(h);
    mid = bf16x2_bits(m);
    lo = bf16x2_bits(l);
}

template <int EPN, int KM, int MINB>
__global__ void __launch_bounds__(NUM_THREADS, MINB)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const Args a)
{
    using G = Geo<EPN>;
    constexpr int TERM = G::TERM_BYTES, LDS = G::LDS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* xring = smem;              // S x 16 KB; the whole ring area is the epilogue's scratch
    uint8_t* bring = smem + a.b_off;    // WDEPTH x B_BYTES
    uint8_t* wring = smem + a.w_off;    // WDEPTH x w_slot
    Misc* m = reinterpret_cast<Misc*>(smem + a.misc_off);
    float* recv = reinterpret_cast<float*>(smem + a.recv_off);
    const int S = a.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * BM;
    const int split = (int)blockIdx.y;  // the CTA's rank in its cluster when splits > 1
    const int num_kb = (a.D + BK - 1) / BK;
    const int kb_begin = split * a.split_kb;                // never empty (host guarantee)
    const int kb_end = min(num_kb, kb_begin + a.split_kb);
    const int nkb = kb_end - kb_begin;
    auto kb_at = [&](int i) { return kb_begin + i; };
    const int E = a.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&m->xfull[s], 1);
            mbar_init(&m->xempty[s], 1);
        }
        for (int j = 0; j < WDEPTH; ++j) {
            mbar_init(&m->wl[j], 1);
            mbar_init(&m->bfull[j], CONVERTER_WARPS);
            mbar_init(&m->bempty[j], 1);
            mbar_init(&m->wfree[j], CONVERTER_WARPS);
        }
        mbar_init(&m->tfull, 1);
        m->abort_flag = 0;
        m->last = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
    }
    if (warp >= 2) {
        // weight terms: rows E .. EPN-1 (if any) stay zero in every slot
        const int tid = threadIdx.x - 64;
        m->cnt[tid] = 0;
        const int pad = EPN - E;
        if (pad > 0) {
            const int per_slot = 3 * pad * 8;  // 16-byte chunks
            for (int i = tid; i < WDEPTH * per_slot; i += 128) {
                const int j = i / per_slot;
                int r = i % per_slot;
                const int p = r / (pad * 8);
                r %= pad * 8;
                uint8_t* dst = bring + (size_t)j * G::B_BYTES + p * TERM + (E + r / 8) * 128 + (r % 8) * 16;
                *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(&m->tmem_base, G::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = m->tmem_base;
    volatile int* abort_flag = &m->abort_flag;
    // the fp32 weight slice of K block kb into slot j (issued by one converter thread)
    auto load_w = [&](int kb, int j) {
        const int d0 = kb * BK;
        const int rows = min(BK, a.D - d0);  // a multiple of 8 (D % 8 == 0)
        const uint32_t bytes = (uint32_t)rows * (uint32_t)E * 4u;
        mbar_arrive_expect_tx(&m->wl[j], bytes);
        bulk_load_g2s(wring + (size_t)j * a.w_slot, a.w + (size_t)d0 * E, bytes, &m->wl[j]);
    };

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
                tma_load_2d(xring + (size_t)stage * A_BYTES, &tmX, kb_at(i) * BK, (int32_t)t0,
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
            constexpr uint32_t idesc = umma_idesc_bf16(BM, EPN, 0, 0);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % S, j = i % WDEPTH;
                if (!mbar_wait(&m->xfull[s], (uint32_t)((i / S) & 1), a.status, 520, abort_flag)) break;
                if (!mbar_wait(&m->bfull[j], (uint32_t)((i / WDEPTH) & 1), a.status, 521, abort_flag)) break;
                tc_fence_after();
                const uint32_t sA = smem_u32(xring + (size_t)s * A_BYTES);
                const uint32_t sB = smem_u32(bring + (size_t)j * G::B_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint64_t adesc = umma_desc_sw128(sA + kk * 32, 16, 1024);
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        const uint64_t bdesc = umma_desc_sw128(sB + p * TERM + kk * 32, 16, 1024);
                        umma_f16_ss(tmem_base, adesc, bdesc, idesc, (i || kk || p) ? 1u : 0u);
                    }
                }
                umma_commit(&m->xempty[s]);
                umma_commit(&m->bempty[j]);
            }
            umma_commit(&m->tfull);  // also the drain: every MMA done once it fires
        }
    } else {
        // ------------------------------------------------ weight split (warps 2..5)
        const int tid = threadIdx.x - 64;
        {
            int issued = 0;  // fp32 slices issued (slot = index % WDEPTH)
            if (tid == 0)
                for (; issued < WDEPTH && issued < nkb; ++issued) load_w(kb_at(issued), issued);
            const int pairs = E * 8;  // (expert, 8-wide chunk of d_model)
            int i = 0;
            for (; i < nkb; ++i) {
                const int j = i % WDEPTH;
                const uint32_t ph = (uint32_t)((i / WDEPTH) & 1);
                if (!mbar_wait(&m->wl[j], ph, a.status, 540, abort_flag)) break;
                if (!mbar_wait(&m->bempty[j], ph ^ 1u, a.status, 541, abort_flag)) break;
                uint8_t* sB = bring + (size_t)j * G::B_BYTES;
                const float* wsm = reinterpret_cast<const float*>(wring + (size_t)j * a.w_slot);
                const int d0 = kb_at(i) * BK;
                for (int q = tid; q < pairs; q += 128) {
                    const int e = q % E, c = q / E;
                    const bool in = d0 + c * 8 < a.D;  // D % 8 == 0: a chunk is all in or all out
                    float v[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) v[jj] = in ? wsm[(c * 8 + jj) * E + e] : 0.f;
                    uint32_t h[4], md[4], l[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) split3(v[2 * jj], v[2 * jj + 1], h[jj], md[jj], l[jj]);
                    const int off = e * 128 + ((c ^ (e & 7)) << 4);
                    *reinterpret_cast<uint4*>(sB + off) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4*>(sB + TERM + off) = make_uint4(md[0], md[1], md[2], md[3]);
                    *reinterpret_cast<uint4*>(sB + 2 * TERM + off) = make_uint4(l[0], l[1], l[2], l[3]);
                }
                fence_proxy_async_smem();  // visible to the tensor cores
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&m->bfull[j]);
                    mbar_arrive(&m->wfree[j]);
                }
                // refill fp32 slot j once every weight warp is done with it
                if (tid == 0 && issued < nkb) {
                    if (!mbar_wait(&m->wfree[j], ph, a.status, 543, abort_flag)) break;
                    load_w(kb_at(issued), issued % WDEPTH);
                    ++issued;
                }
            }
            // after an early exit, the slices still in flight land before the CTA goes on
            if (tid == 0)
                for (int k = i; k < issued; ++k)
                    mbar_wait(&m->wl[k % WDEPTH], (uint32_t)((k / WDEPTH) & 1), a.status, 542, nullptr);
        }
        // ------------------------------------------------ accumulators out of tensor memory
        const int quad = warp & 3;        // the lane quadrant this warp may read
        const int r = quad * 32 + lane;   // token row in the tile
        float* Ls = reinterpret_cast<float*>(xring);  // [BM][LDS]
        const bool ok = mbar_wait(&m->tfull, 0, a.status, 530, abort_flag);
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16);
        uint32_t remote = 0;
        if (split > 0)  // this row's slot in the leader's receive buffer
            remote = mapa_shared(smem_u32(recv + ((size_t)(split - 1) * BM + r) * EPN), 0);
#pragma unroll 1
        for (int c = 0; c < (EPN + 31) / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int e = c * 32 + j;
                if (e < EPN) {
                    const float x = ok ? __uint_as_float(v[j]) : 0.f;
                    if (split > 0)
                        st_cluster_f32(remote + e * 4, x);
                    else
                        Ls[r * LDS + e] = x;
                }
            }
        }
    }
    __syncwarp();
    if (a.splits > 1) cluster_sync();  // the other splits' partials are in the leader's buffer

    if (warp >= 2 && split == 0) {
        // ------------------------------------------------ epilogue: one token row per thread
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int tid = threadIdx.x - 64;
        const int64_t t = t0 + r;
        const bool valid = t < a.T;
        const int K = a.K;
        const RouteOpts& o = a.o;
        float* Ls = reinterpret_cast<float*>(xring);  // logits, then normalised scores
        float* Xs = Ls + BM * LDS;                     // scores: exp(L - max), or sigmoid(L)
        const int G = o.n_groups, gsz = E / G;
        // top-K by (u desc, id asc), u = L + selection bias: an unrolled insertion
        // network of KM >= K slots (a displaced entry carried down keeps that order)
        float tv[KM];
        int ti[KM];
#pragma unroll
        for (int k = 0; k < KM; ++k) {
            tv[k] = -INFINITY;
            ti[k] = 0x7fffffff;
        }
        auto insert = [&](float xv, int xi) {
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                const bool gt = xv > tv[k] || (xv == tv[k] && xi < ti[k]);
                const float nv = gt ? xv : tv[k];
                const int ni = gt ? xi : ti[k];
                xv = gt ? tv[k] : xv;
                xi = gt ? ti[k] : xi;
                tv[k] = nv;
                ti[k] = ni;
            }
        };
        // pass 1: logits (own K range + the other splits in order, + bias + noise),
        // their maximum, and (without a group limit) the top-K
        float mx = -INFINITY;
#pragma unroll 4
        for (int e = 0; e < E; ++e) {
            float L = Ls[r * LDS + e];
            for (int sp = 1; sp < a.splits; ++sp) L += recv[((size_t)(sp - 1) * BM + r) * EPN + e];
            if (a.bias) L += a.bias[e];
            if (a.noise && valid) L += a.noise[t * E + e];
            if (a.logits_out && valid) a.logits_out[t * E + e] = L;
            Ls[r * LDS + e] = L;
            mx = fmaxf(mx, L);
            if (G == 1) insert(L + (o.sel_bias ? o.sel_bias[e] : 0.f), e);
        }
        // pass 2: softmax sum, sum of exp(L - max) (L - max) for the entropy, and
        // the scores (sigmoid scores and their sum with score_func sigmoid)
        float ssum = 0.f, s1 = 0.f, scsum = 0.f;
#pragma unroll 4
        for (int e = 0; e < E; ++e) {
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
        const float inv = 1.0f / ssum;
        const float lss = logf(ssum);
        // entropy -sum q log q = log(sum) - sum q (L - max), q = exp(L - max) / sum
        const float ent = lss - s1 * inv;
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
                        gm[g] = fmaxf(gm[g], Ls[r * LDS + e] + (o.sel_bias ? o.sel_bias[e] : 0.f));
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
                if ((keep >> (e / gsz)) & 1u) insert(Ls[r * LDS + e] + (o.sel_bias ? o.sel_bias[e] : 0.f), e);
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
        // pass 3: normalised scores into Ls (and probs_out); rows past T give nothing
        const float scinv = o.score_func == 1 ? 1.0f / scsum : inv;
#pragma unroll 4
        for (int e = 0; e < E; ++e) {
            const float pn = Xs[r * LDS + e] * scinv;
            Ls[r * LDS + e] = valid ? pn : 0.f;
            if (a.probs_out && valid) a.probs_out[t * E + e] = pn;
        }
        if (a.with_stats) {
            // per-CTA statistics, each in a fixed order
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
            epi_sync();
            constexpr int CH = 128 / EPN;  // row chunks per column (EPN x CH = 128 threads)
            constexpr int RC = BM / CH;
            {
                const int col = tid % EPN, ch = tid / EPN;
                float sp = 0.f;
                if (col < E)
                    for (int rr = ch * RC; rr < (ch + 1) * RC; ++rr) sp += Ls[rr * LDS + col];
                m->psum[ch * EPN + col] = sp;
            }
            epi_sync();
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
            epi_sync();
            if (tid == 0) m->last = atomicAdd(a.counter, 1) == (int)gridDim.x - 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (split == 0 && a.with_stats && m->last) {
        // the last CTA: the statistics of the whole grid (all 192 threads)
        __threadfence();
        double* sd = reinterpret_cast<double*>(xring);
        long long* sc = reinterpret_cast<long long*>(sd + kStatD);
        finish_router_stats(a.blk_mp, a.blk_z, a.blk_ent, a.blk_cnt, (int)gridDim.x, a.T, E, a.K,
                            a.mean_prob, a.losses, sd, sc, NUM_THREADS, (int)threadIdx.x,
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

// Ring depth and shared-memory layout for `ctas_per_sm` CTAs on each SM:
// [x ring: stages x 16 KB][weight terms: WDEPTH x 3 x EPN x 128][fp32 slices:
// WDEPTH x w_slot][Misc][split partials]; the rings together are the
// epilogue's scratch.
struct Plan {
    int epn, splits, split_kb, ctas_per_sm, stages;
    uint32_t b_off, w_off, w_slot, misc_off, recv_off;
    size_t smem;  // dynamic shared memory, with 1 KB of alignment slack
};

static int epn_of(int E) { return E <= 16 ? 16 : E <= 32 ? 32 : E <= 64 ? 64 : 128; }

static Plan make_plan(const moe_config& c)
{
    Plan p{};
    p.epn = epn_of(c.E);
    const int tiles = router_tc_blocks(c);
    const int nkb = (c.D + BK - 1) / BK;
    p.splits = router_tc_splits(c);
    p.split_kb = (nkb + p.splits - 1) / p.splits;
    const size_t b_bytes = (size_t)3 * p.epn * 128;
    p.w_slot = (uint32_t)align_up((size_t)64 * c.E * 4, 1024);
    const size_t recv = (size_t)(p.splits - 1) * BM * p.epn * sizeof(float);
    const size_t misc = align_up(sizeof(Misc), 1024);
    const size_t fixed = 1024 + WDEPTH * (b_bytes + p.w_slot) + misc + align_up(recv, 1024);
    // the epilogue scratch (and the statistics' last step) live in the rings
    const size_t epi = (size_t)2 * BM * (p.epn + 1) * sizeof(float);
    const size_t fin = (size_t)kStatD * sizeof(double) + (size_t)kStatC * sizeof(long long);
    auto stages_for = [&](size_t budget) {
        if (budget <= fixed) return 0;
        int st = (int)((budget - fixed) / A_BYTES);
        if (st > MAX_STAGES) st = MAX_STAGES;
        const size_t rings = (size_t)st * A_BYTES + WDEPTH * (b_bytes + p.w_slot);
        return (rings >= epi && rings >= fin) ? st : 0;
    };
    // two CTAs per SM when the tiles outnumber the SMs and each still gets 3 x stages
    p.ctas_per_sm = 1;
    if (tiles * p.splits > 148 && p.epn <= 64 && stages_for(112 * 1024) >= 3) p.ctas_per_sm = 2;
    p.stages = stages_for(p.ctas_per_sm == 2 ? 112 * 1024 : 226 * 1024);
    p.b_off = (uint32_t)((size_t)p.stages * A_BYTES);
    p.w_off = p.b_off + (uint32_t)(WDEPTH * b_bytes);
    p.misc_off = p.w_off + (uint32_t)(WDEPTH * p.w_slot);
    p.recv_off = p.misc_off + (uint32_t)misc;
    p.smem = (size_t)p.recv_off + align_up(recv, 1024) + 1024;
    return p;
}

template <int EPN, int KM, int MINB>
static cudaError_t launch_t(const moe_config& c, const CUtensorMap& mX, const Args& a, const Plan& p,
                            cudaStream_t s)
{
    auto kern = router_tc_kernel<EPN, KM, MINB>;
    static PerDeviceFlag smem_set;
    // the largest ring this instance is launched with (one attribute per device)
    cudaError_t ae = opt_in_smem(smem_set, reinterpret_cast<const void*>(kern),
                                 MINB == 2 ? 113 * 1024 : 227 * 1024);
    if (ae != cudaSuccess) return ae;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)router_tc_blocks(c), (unsigned)p.splits, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)p.splits;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.splits > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, mX, a);
}

template <int EPN>
static cudaError_t launch_k(const moe_config& c, const CUtensorMap& mX, const Args& a, const Plan& p,
                            cudaStream_t s)
{
    const int km = c.K <= 2 ? 2 : c.K <= 4 ? 4 : c.K <= 6 ? 6 : 8;
    if (p.ctas_per_sm == 2) {
        if constexpr (EPN <= 64) {
            return km == 2 ? launch_t<EPN, 2, 2>(c, mX, a, p, s)
                 : km == 4 ? launch_t<EPN, 4, 2>(c, mX, a, p, s)
                 : km == 6 ? launch_t<EPN, 6, 2>(c, mX, a, p, s)
                           : launch_t<EPN, 8, 2>(c, mX, a, p, s);
        }
        return cudaErrorInvalidValue;
    }
    return km == 2 ? launch_t<EPN, 2, 1>(c, mX, a, p, s)
         : km == 4 ? launch_t<EPN, 4, 1>(c, mX, a, p, s)
         : km == 6 ? launch_t<EPN, 6, 1>(c, mX, a, p, s)
                   : launch_t<EPN, 8, 1>(c, mX, a, p, s);
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

cudaError_t launch_router_tc(const moe_config& c, const RouteOpts& o, const void* x,
                             const float* w_router, const float* bias, const float* noise,
                             float* logits_out, float* probs_out, int32_t* ids, float* w,
                             float* blk_mp, float* blk_z, float* blk_ent, int32_t* blk_cnt,
                             float* mean_prob, float* losses, int* status, cudaStream_t s)
{
    using namespace rtc;
    const Plan p = make_plan(c);
    EncodeTiledFn enc = encoder();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap mX;
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
    Args a{};
    a.o = o;
    a.w = w_router;
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
    a.b_off = p.b_off;
    a.w_off = p.w_off;
    a.w_slot = p.w_slot;
    a.splits = p.splits;
    a.split_kb = p.split_kb;
    a.misc_off = p.misc_off;
    a.recv_off = p.recv_off;
    switch (p.epn) {
        case 16: return launch_k<16>(c, mX, a, p, s);
        case 32: return launch_k<32>(c, mX, a, p, s);
        case 64: return launch_k<64>(c, mX, a, p, s);
        default: return launch_k<128>(c, mX, a, p, s);
    }
}

}  // namespace moe
