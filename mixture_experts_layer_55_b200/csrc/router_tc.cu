// router_tc.cu -- router for bf16 layers on the tensor cores: the logits GEMM,
// softmax, top-k and renormalised weights fused in one kernel.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation": fp32
// router logits, softmax over the experts, top-k, weights divided by the sum
// of the selected probabilities; the statistics (mean probability, counts,
// logsumexp) feed the balance loss and the z-loss.
//
// fp32 logits on bf16 tensor cores: x is bf16 already, and each fp32 router
// weight is split exactly into three bf16 terms w = hi + mid + lo (hi =
// bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid): 3 x 8 significand
// bits cover fp32's 24).  Every product x*part is exact in fp32, and the
// three MMAs accumulate in fp32 in tensor memory, so the logits carry fp32
// accumulation error only (no bf16 rounding of the weights).
//
//   router_wsplit_kernel  W_r (D, E) fp32 -> (3, D, EP) bf16, EP = E rounded
//                         up to 64 (zero columns), N-major for TMA.
//   router_tc_kernel      one CTA per 128 tokens (and per split of d_model when
//                         the token tiles leave most SMs idle).  With splits,
//                         or more than 16 experts, it writes fp32 (partial)
//                         logits, which the top-k kernel of the SIMT router sums
//                         in split order and routes; otherwise the fused
//                         epilogue below routes: warp 0 TMA (x tile 128 x 64,
//                         three 64 x EP weight tiles per stage), warp 1
//                         tcgen05.mma M=128, N=EP, three per K step into one
//                         accumulator; warps 2..5 own one token row each:
//                         logits (+ bias + noise) staged in shared memory,
//                         max, softmax sum, entropy, scores (softmax or
//                         sigmoid), the group limit, top-K by (logit +
//                         selection bias desc, id asc) with an unrolled
//                         insertion network, weights, normalised scores, and
//                         fixed-order per-CTA statistics.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace rtc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int BOX_BYTES = 64 * 64 * 2;     // 8 KB
constexpr int NUM_THREADS = 192;

template <int EPB> struct Geo {            // EPB = EP / 64 (1 or 2)
    static constexpr int EP = 64 * EPB;
    static constexpr int B_BYTES = 3 * EPB * BOX_BYTES;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 40 KB or 64 KB
    static constexpr int STAGES = EPB == 1 ? 4 : 3;
    static constexpr int TMEM_COLS = EP;                   // 64 or 128 (powers of two)
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
};

struct Misc {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t tfull;
    uint32_t tmem_base;
    int abort_flag;
};

struct Args {
    RouteOpts o;
    const float* bias;        // E or null
    const float* noise;       // T x E or null
    float* logits_out;        // T x E or null
    float* probs_out;         // T x E or null
    int32_t* ids;             // T x K
    float* wout;              // T x K
    float* blk_mp;            // grid x E
    float* blk_z;             // grid
    float* blk_ent;           // grid
    int32_t* blk_cnt;         // grid x E
    int64_t T;
    int D, E, K;
    int with_stats;
    int* status;
    float* part;              // split mode: (splits, T, E) fp32 partial logits, else null
    int split_kb;             // split mode: K blocks per split (blockIdx.y = split)
};

__global__ void __launch_bounds__(256) router_wsplit_kernel(const float* __restrict__ w,
                                                            __nv_bfloat16* __restrict__ out, int D,
                                                            int E, int EP)
{
    const int64_t n = (int64_t)D * EP;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int d = (int)(i / EP), e = (int)(i % EP);
        const float v = e < E ? w[(int64_t)d * E + e] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
        out[i] = hi;
        out[n + i] = mid;
        out[2 * n + i] = lo;
    }
}

MOE_DEVICE void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int EPB>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const Args a)
{
    using G = Geo<EPB>;
    constexpr int EP = G::EP, STAGES = G::STAGES, STAGE_BYTES = G::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* stages = smem;
    Misc* m = reinterpret_cast<Misc*>(smem + (size_t)STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * BM;
    const int num_kb = (a.D + BK - 1) / BK;
    // this CTA's K blocks: all of them, or its split's share (never empty)
    const int kb_begin = a.part ? (int)blockIdx.y * a.split_kb : 0;
    const int kb_end = a.part ? min(num_kb, kb_begin + a.split_kb) : num_kb;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&m->full[s], 1);
            mbar_init(&m->empty[s], 1);
        }
        mbar_init(&m->tfull, 1);
        m->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
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

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0;
        int last_phase[STAGES];
        for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
            if (!mbar_wait(&m->empty[stage], phase ^ 1u, a.status, 510, abort_flag)) break;
            uint8_t* sA = stages + (size_t)stage * STAGE_BYTES;
            uint8_t* sB = sA + A_BYTES;
            uint64_t* fb = &m->full[stage];
            mbar_arrive_expect_tx(fb, STAGE_BYTES);
            const int k0 = kb * BK;
            tma_load_2d(sA, &tmX, k0, (int32_t)t0, fb);
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int j = 0; j < EPB; ++j)
                    tma_load_3d(sB + (p * EPB + j) * BOX_BYTES, &tmW, 64 * j, k0, p, fb);
            last_phase[stage] = (int)phase;
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        for (int s = 0; s < STAGES; ++s)
            if (last_phase[s] >= 0) mbar_wait(&m->full[s], (uint32_t)last_phase[s], a.status, 511, nullptr);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = umma_idesc_bf16(BM, EP, 0, 1);
        int stage = 0;
        uint32_t phase = 0;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
            if (!mbar_wait(&m->full[stage], phase, a.status, 520, abort_flag)) break;
            tc_fence_after();
            const uint32_t sA = smem_u32(stages + (size_t)stage * STAGE_BYTES);
            const uint32_t sB = sA + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
                const uint64_t adesc = umma_desc_sw128(sA + kk * 32, 16, 1024);
#pragma unroll
                for (int p = 0; p < 3; ++p) {
                    const uint64_t bdesc =
                        umma_desc_sw128(sB + p * EPB * BOX_BYTES + kk * 2048, BOX_BYTES, 1024);
                    umma_f16_ss(tmem_base, adesc, bdesc, idesc, (kb != kb_begin || kk || p) ? 1u : 0u);
                }
            }
            umma_commit(&m->empty[stage]);
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        umma_commit(&m->tfull);  // also the drain: every MMA done once it fires
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue: one token row per thread
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // row in tile = tensor-memory lane
        const int64_t t = t0 + r;
        const bool valid = t < a.T;
        const int E = a.E, K = a.K;
        const RouteOpts& o = a.o;
        // the pipeline buffers are free once the accumulator is complete
        float* Ls = reinterpret_cast<float*>(stages);  // [BM][EP + 1] logits, then scores
        constexpr int LDS = EP + 1;
        const bool ok = mbar_wait(&m->tfull, 0, a.status, 530, abort_flag);
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16);
        if (a.part != nullptr) {
            // split mode: this split's partial logits of the row, summed (in split
            // order) with bias and noise by the top-k kernel
            float* prow = a.part + ((size_t)blockIdx.y * a.T + t) * E;
#pragma unroll 1
            for (int c = 0; c < EP / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(taddr + c * 32, v);
                tmem_ld_wait();
                if (valid)
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c * 32 + j < E) prow[c * 32 + j] = ok ? __uint_as_float(v[j]) : 0.f;
            }
        } else {
        // pass 1: logits (+ bias + noise) to shared memory and their maximum
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < EP / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int e = c * 32 + j;
                float L = -INFINITY;
                if (e < E && ok) {
                    L = __uint_as_float(v[j]);
                    if (a.bias) L += a.bias[e];
                    if (a.noise && valid) L += a.noise[t * E + e];
                    if (a.logits_out && valid) a.logits_out[t * E + e] = L;
                }
                Ls[r * LDS + e] = L;
                mx = fmaxf(mx, L);
            }
        }
        // pass 2: softmax sum, entropy, score sum
        float ssum = 0.f;
        for (int e = 0; e < E; ++e) ssum += expf(Ls[r * LDS + e] - mx);
        const float inv = 1.0f / ssum;
        float ent = 0.f, scsum = 0.f;
        for (int e = 0; e < E; ++e) {
            const float L = Ls[r * LDS + e];
            const float q = expf(L - mx) * inv;
            ent -= q * logf(fmaxf(q, 1e-9f));
            scsum += o.score_func == 1 ? 1.0f / (1.0f + expf(-L)) : q;
        }
        // group limit: a group's score is its best selection score u = L + b
        uint32_t keep = 0xffffffffu;
        const int G = o.n_groups, gsz = E / G;
        if (G > 1) {
            float gm[32];
#pragma unroll
            for (int g = 0; g < 32; ++g) {
                gm[g] = -INFINITY;
                if (g < G)
                    for (int e = g * gsz; e < (g + 1) * gsz; ++e)
                        gm[g] = fmaxf(gm[g], Ls[r * LDS + e] + (o.sel_bias ? o.sel_bias[e] : 0.f));
            }
            keep = 0;
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
        }
        // pass 3: top-K over the eligible experts by (u desc, id asc), an unrolled
        // insertion network (a displaced entry carried down keeps that order too)
        float tv[8];
        int ti[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            tv[k] = -INFINITY;
            ti[k] = 0x7fffffff;
        }
        for (int e = 0; e < E; ++e) {
            if (G > 1 && !((keep >> (e / gsz)) & 1u)) continue;
            float x = Ls[r * LDS + e] + (o.sel_bias ? o.sel_bias[e] : 0.f);
            int xi = e;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const bool gt = x > tv[k] || (x == tv[k] && xi < ti[k]);
                const float nv = gt ? x : tv[k];
                const int ni = gt ? xi : ti[k];
                x = gt ? tv[k] : x;
                xi = gt ? ti[k] : xi;
                tv[k] = nv;
                ti[k] = ni;
            }
        }
        // weights from the scores of the selected experts
        float sk[8];
        float ssel = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            sk[k] = 0.f;
            if (k < K) {
                const float L = Ls[r * LDS + ti[k]];
                sk[k] = o.score_func == 1 ? 1.0f / (1.0f + expf(-L)) : expf(L - mx) * inv;
            }
            ssel += sk[k];
        }
        if (valid) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < K) {
                    a.ids[t * K + k] = ti[k];
                    a.wout[t * K + k] = (o.renorm ? sk[k] / ssel : sk[k]) * o.route_scale;
                }
        }
        // pass 4: normalised scores into shared memory (and probs_out)
        const float scinv = 1.0f / scsum;
        for (int e = 0; e < E; ++e) {
            const float L = Ls[r * LDS + e];
            const float pn = (o.score_func == 1 ? 1.0f / (1.0f + expf(-L)) : expf(L - mx) * inv) *
                             (o.score_func == 1 ? scinv : 1.0f);
            Ls[r * LDS + e] = valid ? pn : 0.f;  // rows past T contribute nothing
            if (a.probs_out && valid) a.probs_out[t * E + e] = pn;
        }
        if (a.with_stats) {
            // per-CTA statistics in a fixed order: column sums over the rows
            const float lse = mx + logf(ssum);
            int* sid = reinterpret_cast<int*>(Ls + BM * LDS);  // [BM][8]
            float* sz = reinterpret_cast<float*>(sid + BM * 8);
            float* sh = sz + BM;
#pragma unroll
            for (int k = 0; k < 8; ++k) sid[r * 8 + k] = (valid && k < K) ? ti[k] : -1;
            sz[r] = valid ? lse * lse : 0.f;
            sh[r] = valid ? ent : 0.f;
            epi_sync();
            const int tid = threadIdx.x - 64;
            for (int e = tid; e < E; e += 128) {
                float sp = 0.f;
                int cn = 0;
                for (int rr = 0; rr < BM; ++rr) {
                    sp += Ls[rr * LDS + e];
#pragma unroll
                    for (int k = 0; k < 8; ++k) cn += sid[rr * 8 + k] == e;
                }
                a.blk_mp[(size_t)blockIdx.x * E + e] = sp;
                a.blk_cnt[(size_t)blockIdx.x * E + e] = cn;
            }
            if (tid == 0) {
                float zs = 0.f, hs = 0.f;
                for (int rr = 0; rr < BM; ++rr) {
                    zs += sz[rr];
                    hs += sh[rr];
                }
                a.blk_z[blockIdx.x] = zs;
                a.blk_ent[blockIdx.x] = hs;
            }
        }
        }  // fused epilogue
    }
    tc_fence_before();
    __syncthreads();
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

template <int EPB>
static cudaError_t launch_t(const moe_config& c, const void* x, const __nv_bfloat16* wsplit,
                            const Args& a, cudaStream_t s)
{
    using G = Geo<EPB>;
    static int done_mask = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 31 || !((done_mask >> dev) & 1)) {
        cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<EPB>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
        if (e != cudaSuccess) return e;
        if (dev < 31) done_mask |= 1 << dev;
    }
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
        cuuint64_t dims[3] = {(cuuint64_t)G::EP, (cuuint64_t)c.D, 3};
        cuuint64_t strides[2] = {(cuuint64_t)G::EP * 2, (cuuint64_t)G::EP * c.D * 2};
        cuuint32_t box[3] = {64, 64, 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&mW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(wsplit), dims,
                strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int nkb = (c.D + BK - 1) / BK;
    const unsigned splits = a.part ? (unsigned)((nkb + a.split_kb - 1) / a.split_kb) : 1u;
    const dim3 grid((unsigned)((c.T + BM - 1) / BM), splits);
    router_tc_kernel<EPB><<<grid, NUM_THREADS, G::SMEM, s>>>(mX, mW, a);
    return cudaGetLastError();
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
    if (sp > 4) sp = 4;
    if (sp > nkb / 8) sp = nkb / 8;
    if (sp < 2) return 1;
    const int per = (nkb + sp - 1) / sp;  // K blocks per split; every split non-empty
    return (nkb + per - 1) / per;
}

bool router_tc_partial(const moe_config& c)
{
    // the fused epilogue gives each token to one thread, which walks all E
    // experts several times; above 16 experts the SIMT top-k kernel (a warp
    // per token, the experts spread over its lanes) routes faster from the
    // logits the tensor cores wrote
    return router_tc_splits(c) > 1 || c.E > 16;
}

size_t router_tc_wsplit_bytes(const moe_config& c)
{
    const int ep = (c.E + 63) / 64 * 64;
    return (size_t)3 * c.D * ep * sizeof(__nv_bfloat16);
}

cudaError_t launch_router_tc(const moe_config& c, const RouteOpts& o, const void* x,
                             const float* w_router, const float* bias, const float* noise,
                             float* logits_out, float* probs_out, int32_t* ids, float* w,
                             float* blk_mp, float* blk_z, float* blk_ent, int32_t* blk_cnt,
                             int with_stats, void* wsplit_scratch, void* part_out, int* status,
                             cudaStream_t s)
{
    using namespace rtc;
    const int ep = (c.E + 63) / 64 * 64;
    __nv_bfloat16* wsplit = static_cast<__nv_bfloat16*>(wsplit_scratch);
    const int64_t n = (int64_t)c.D * ep;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    router_wsplit_kernel<<<(unsigned)blocks, 256, 0, s>>>(w_router, wsplit, c.D, c.E, ep);
    const int splits = router_tc_splits(c);
    const int nkb = (c.D + BK - 1) / BK;
    Args a{o, bias, noise, logits_out, probs_out, ids, w, blk_mp, blk_z, blk_ent, blk_cnt,
           c.T, c.D, c.E, c.K, with_stats, status,
           router_tc_partial(c) ? static_cast<float*>(part_out) : nullptr, (nkb + splits - 1) / splits};
    return ep == 64 ? launch_t<1>(c, x, wsplit, a, s) : launch_t<2>(c, x, wsplit, a, s);
}

}  // namespace moe
