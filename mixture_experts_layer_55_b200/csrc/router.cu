// router.cu -- fp32 router: logits GEMM, softmax + top-k + renormalised
// weights, and the router statistics (mean probability, z-loss, balance loss).
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation": router
// logits in fp32, softmax over all experts, top-k, weights divided by the sum
// of the selected probabilities, bincount of the ids, balance loss
// E * sum_e f_e P_e and z-loss mean_t logsumexp_t^2.
//
// Kernels:
//   router_logits_kernel  tiled SIMT fp32 GEMM (T x D) * (D x E), optionally
//                         split over d_model; partial sums go to scratch.
//   router_splitsum_kernel sums the d-split partials in split order (more than
//                         kTopkMaxSplits splits; fewer, the top-k kernel adds them).
//   router_topk_kernel    one warp per token: adds bias and noise, softmax, top-k by
//                         (logit desc, id asc) with warp shuffles, weights,
//                         and per-block statistic partials, which the block
//                         that finishes last reduces in a fixed order into
//                         the mean probabilities, z-loss and balance loss
//                         (router_stats.cuh).
// bf16 layers with E <= 128 and T >= 2048 route on the tensor cores instead
// (router_tc.cu).
#include "common.cuh"
#include "internal.h"
#include "router_stats.cuh"

namespace moe {

constexpr int kLogitsBD = 32;  // d_model per shared-memory step
// tokens per top-k block: 8 warps x 2, or x 1 when the tokens are too few to
// give every SM several blocks of two (decode-sized batches)
inline int topk_tokens_per_block(int64_t T) { return T <= 148 * 16 * 2 ? 8 : 16; }

// Tokens per logits block for an expert tile of be columns (see the kernel's
// thread layout): 128 for be = 8, else 64.
static int logits_bt(int be) { return be == 8 ? 128 : 64; }

RouterPlan router_plan(const moe_config& c)
{
    RouterPlan p;
    p.be = c.E <= 8 ? 8 : c.E <= 16 ? 16 : c.E <= 32 ? 32 : 64;
    const int bt = logits_bt(p.be);
    p.grid_t = (int)((c.T + bt - 1) / bt);
    p.grid_e = (c.E + p.be - 1) / p.be;
    int64_t base = (int64_t)p.grid_t * p.grid_e;
    int want = (int)((6 * 148 + base - 1) / base);  // enough blocks to hide load latency
    // at least 256 of d_model per split, or down to 64 for up to 4 splits (a short
    // d_model with few tokens)
    int max_splits = c.D / 256;
    const int short_splits = c.D / 64 < 4 ? c.D / 64 : 4;
    if (max_splits < short_splits) max_splits = short_splits;
    if (max_splits < 1) max_splits = 1;
    if (want > max_splits) want = max_splits;
    if (want < 1) want = 1;
    int dps = (c.D + want - 1) / want;
    dps = (dps + kLogitsBD - 1) / kLogitsBD * kLogitsBD;
    p.d_per_split = dps;
    p.splits = (c.D + dps - 1) / dps;
    p.tpb_topk = topk_tokens_per_block(c.T);
    p.nb_topk = (int)((c.T + p.tpb_topk - 1) / p.tpb_topk);
    return p;
}

template <typename XT> struct XVec;  // 16-byte vector of x elements
template <> struct XVec<float> {
    static constexpr int N = 4;
    MOE_DEVICE static void to_f32(const uint4& v, float* o)
    {
        o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
    }
};
template <> struct XVec<__nv_bfloat16> {
    static constexpr int N = 8;
    MOE_DEVICE static void to_f32(const uint4& v, float* o)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// Logits GEMM partials: part[z][t][e] = sum over this block's d-split of
// x[t][d] * W_r[d][e].  256 threads = NTY token groups x NTX expert groups;
// thread (ty, tx) owns tokens ty*TM .. ty*TM+TM-1 (one float4 of the
// transposed x tile) and experts tx + j*NTX.  x arrives as 16-byte vectors;
// the next tile is prefetched into registers while the current one is used.
template <typename XT, int BE, int TM, int TE>
__global__ void __launch_bounds__(256) router_logits_kernel(const XT* __restrict__ x,
                                                            const float* __restrict__ w,
                                                            float* __restrict__ part, int64_t T,
                                                            int D, int E, int dps)
{
    constexpr int BD = kLogitsBD;
    constexpr int NTX = BE / TE, NTY = 256 / NTX, BT = NTY * TM;
    static_assert(TM == 4, "float4 token reads");
    constexpr int VN = XVec<XT>::N;                   // elements per 16-byte vector
    constexpr int XV = BT * BD / VN / 256;            // x vectors per thread per step
    constexpr int WV = BD * BE / 256;                 // w scalars per thread per step
    static_assert(XV >= 1 && WV >= 1, "tile sizes");
    __shared__ __align__(16) float xs[2][BD][BT + 4];
    __shared__ float wsm[2][BD][BE];

    const int tid = threadIdx.x;
    const int tx = tid % NTX, ty = tid / NTX;
    const int64_t t0 = (int64_t)blockIdx.x * BT;
    const int e0 = blockIdx.y * BE;
    const int d_begin = blockIdx.z * dps;
    const int d_end = min(D, d_begin + dps);

    uint4 xr[XV];
    float wr[WV];
    auto load = [&](int d0) {
#pragma unroll
        for (int i = 0; i < XV; ++i) {
            const int idx = tid + i * 256;
            const int tt = idx / (BD / VN), dv = idx % (BD / VN);
            const int64_t t = t0 + tt;
            const int d = d0 + dv * VN;
            xr[i] = (t < T && d < d_end) ? __ldg(reinterpret_cast<const uint4*>(x + t * D + d))
                                         : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < WV; ++i) {
            const int idx = tid + i * 256;
            const int dd = idx / BE, ee = idx % BE;
            const int d = d0 + dd, e = e0 + ee;
            wr[i] = (d < d_end && e < E) ? __ldg(w + (int64_t)d * E + e) : 0.f;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int i = 0; i < XV; ++i) {
            const int idx = tid + i * 256;
            const int tt = idx / (BD / VN), dv = idx % (BD / VN);
            float v[VN];
            XVec<XT>::to_f32(xr[i], v);
#pragma unroll
            for (int k = 0; k < VN; ++k) xs[buf][dv * VN + k][tt] = v[k];
        }
#pragma unroll
        for (int i = 0; i < WV; ++i) {
            const int idx = tid + i * 256;
            wsm[buf][idx / BE][idx % BE] = wr[i];
        }
    };

    float acc[TM][TE];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

    int buf = 0;
    load(d_begin);
    store(0);
    __syncthreads();
    for (int d0 = d_begin; d0 < d_end; d0 += BD) {
        const bool more = d0 + BD < d_end;
        if (more) load(d0 + BD);
#pragma unroll 8
        for (int dd = 0; dd < BD; ++dd) {
            const float4 xv = *reinterpret_cast<const float4*>(&xs[buf][dd][ty * TM]);
            float wv[TE];
#pragma unroll
            for (int j = 0; j < TE; ++j) wv[j] = wsm[buf][dd][tx + j * NTX];
#pragma unroll
            for (int j = 0; j < TE; ++j) {
                acc[0][j] = fmaf(xv.x, wv[j], acc[0][j]);
                acc[1][j] = fmaf(xv.y, wv[j], acc[1][j]);
                acc[2][j] = fmaf(xv.z, wv[j], acc[2][j]);
                acc[3][j] = fmaf(xv.w, wv[j], acc[3][j]);
            }
        }
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    float* out = part + (size_t)blockIdx.z * (size_t)T * E;
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int64_t t = t0 + ty * TM + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < TE; ++j) {
            const int e = e0 + tx + j * NTX;
            if (e < E) out[t * E + e] = acc[i][j];
        }
    }
}

// part[0][t][e] = sum over s of part[s][t][e] (in place, in split order), so
// that the per-token kernel reads one value per logit.  One thread per logit.
__global__ void __launch_bounds__(256) router_splitsum_kernel(float* __restrict__ part, int splits,
                                                              int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        float v = part[i];
        for (int sp = 1; sp < splits; ++sp) v += part[(size_t)sp * n + i];
        part[i] = v;
    }
}

// (value desc, id asc) ordering: does candidate (va, ia) rank before (vb, ib)?
MOE_DEVICE bool ranks_before(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// One warp per token.  Lane l holds experts l, l+32, ... (EPL of them).
// Scores (softmax or sigmoid), the selection score u = L + selection bias,
// optional group limit, top-K on (u desc, id asc), weights from the scores of
// the selected experts (renormalised or not, times route_scale), and per-block
// statistic partials (normalised scores, counts, lse^2, softmax entropy).
template <int EPL>
__global__ void __launch_bounds__(256) router_topk_kernel(
    const float* __restrict__ part, int splits, const float* __restrict__ bias,
    const float* __restrict__ noise, RouteOpts o, float* __restrict__ logits_out,
    float* __restrict__ probs_out, int32_t* __restrict__ ids, float* __restrict__ wout,
    float* __restrict__ blk_mp, float* __restrict__ blk_z, float* __restrict__ blk_ent,
    int32_t* __restrict__ blk_cnt, int64_t T, int E, int K, int with_stats,
    float* __restrict__ mean_prob, float* __restrict__ losses, int* __restrict__ counter, int tpb)
{
    __shared__ float s_mp[8][256];
    __shared__ int s_cnt[8][256];
    __shared__ float s_u[8][256];  // a warp's selection scores, for group maxima
    __shared__ float s_z[8], s_ent[8];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float mp_acc[EPL];
    int cnt_acc[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        mp_acc[j] = 0.f;
        cnt_acc[j] = 0;
    }
    float z_acc = 0.f, ent_acc = 0.f;
    const int G = o.n_groups, gsz = E / G;

    const int64_t tbase = (int64_t)blockIdx.x * tpb;
    for (int i = 0; i < tpb / 8; ++i) {  // tokens warp, warp + 8, ...
        const int64_t t = tbase + warp + 8 * i;
        if (t >= T) break;
        float L[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            int e = lane + 32 * j;
            float v = -INFINITY;
            if (e < E) {
                v = part[t * E + e];
                for (int sp = 1; sp < splits; ++sp) v += part[(size_t)sp * T * E + t * E + e];
                if (bias) v += bias[e];
                if (noise) v += noise[t * E + e];
                if (logits_out) logits_out[t * E + e] = v;
            }
            L[j] = v;
        }
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < EPL; ++j) m = fmaxf(m, L[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float ex[EPL];
        float ssum = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            ex[j] = (lane + 32 * j < E) ? expf(L[j] - m) : 0.f;
            ssum += ex[j];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
        const float inv = 1.0f / ssum;
        // softmax probabilities q, scores sc, normalised scores pn
        float q[EPL], sc[EPL];
        float hpart = 0.f, scsum = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            q[j] = ex[j] * inv;
            const bool in = lane + 32 * j < E;
            if (in) hpart -= q[j] * logf(fmaxf(q[j], 1e-9f));
            sc[j] = !in ? 0.f : (o.score_func == 1 ? 1.0f / (1.0f + expf(-L[j])) : q[j]);
            scsum += sc[j];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            hpart += __shfl_xor_sync(0xffffffffu, hpart, off);
            scsum += __shfl_xor_sync(0xffffffffu, scsum, off);
        }
        const float scinv = o.score_func == 1 ? 1.0f / scsum : 1.0f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            if (e < E) {
                const float pn = o.score_func == 1 ? sc[j] * scinv : q[j];
                if (probs_out) probs_out[t * E + e] = pn;
                mp_acc[j] += pn;
            }
        }
        if (lane == 0) {
            const float lse = m + logf(ssum);
            z_acc = fmaf(lse, lse, z_acc);
            ent_acc += hpart;
        }
        // selection scores and the group limit
        float u[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            u[j] = (e < E) ? L[j] + (o.sel_bias ? o.sel_bias[e] : 0.f) : -INFINITY;
        }
        uint32_t elig = 0xffffffffu;  // bit j: expert lane + 32j may be selected
        if (G > 1) {
#pragma unroll
            for (int j = 0; j < EPL; ++j)
                if (lane + 32 * j < E) s_u[warp][lane + 32 * j] = u[j];
            __syncwarp();
            float gm = -INFINITY;  // lane g < G: its group's best selection score
            if (lane < G)
                for (int e = lane * gsz; e < (lane + 1) * gsz; ++e) gm = fmaxf(gm, s_u[warp][e]);
            uint32_t keep = 0;
            for (int r = 0; r < o.topk_groups; ++r) {
                float bv = (lane < G && !((keep >> lane) & 1u)) ? gm : -INFINITY;
                int bi = (lane < G && !((keep >> lane) & 1u)) ? lane : 0x7fffffff;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                    if (ranks_before(ov, oi, bv, bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                keep |= 1u << bi;
            }
            elig = 0;
#pragma unroll
            for (int j = 0; j < EPL; ++j)
                if (lane + 32 * j < E && ((keep >> ((lane + 32 * j) / gsz)) & 1u)) elig |= 1u << j;
            __syncwarp();  // s_u is rewritten by the next token
        }
        // top-K: K rounds of a warp-wide arg-best over the eligible, not yet taken
        uint32_t taken = 0;  // bit j: expert lane+32j already selected
        float sel_s[8];
        int sel_id[8];
        float ssel = 0.f;
        for (int k = 0; k < K; ++k) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                int e = lane + 32 * j;
                if (e < E && ((elig >> j) & 1u) && !((taken >> j) & 1u) &&
                    ranks_before(u[j], e, bv, bi)) {
                    bv = u[j];
                    bi = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (ranks_before(ov, oi, bv, bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            // the owner lane marks it taken and broadcasts its score
            float sk = 0.f;
            if ((bi & 31) == lane) {
                int j = bi >> 5;
#pragma unroll
                for (int jj = 0; jj < EPL; ++jj)
                    if (jj == j) {
                        taken |= 1u << jj;
                        sk = sc[jj];
                        cnt_acc[jj] += 1;
                    }
            }
            sk = __shfl_sync(0xffffffffu, sk, bi & 31);
            sel_s[k] = sk;
            sel_id[k] = bi;
            ssel += sk;
        }
        if (lane < K) {
            float sk = 0.f;
            int idk = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k == lane) {
                    sk = sel_s[k];
                    idk = sel_id[k];
                }
            ids[t * K + lane] = idk;
            wout[t * K + lane] = (o.renorm ? sk / ssel : sk) * o.route_scale;
        }
    }
    if (!with_stats) return;
    // per-block partials, reduced over warps in a fixed order
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        int e = lane + 32 * j;
        if (e < 256) {
            s_mp[warp][e] = mp_acc[j];
            s_cnt[warp][e] = cnt_acc[j];
        }
    }
    if (lane == 0) {
        s_z[warp] = z_acc;
        s_ent[warp] = ent_acc;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float a = 0.f;
        int cn = 0;
        for (int wv = 0; wv < 8; ++wv) {
            a += s_mp[wv][e];
            cn += s_cnt[wv][e];
        }
        blk_mp[(size_t)blockIdx.x * E + e] = a;
        blk_cnt[(size_t)blockIdx.x * E + e] = cn;
    }
    if (threadIdx.x == 0) {
        float a = 0.f, h = 0.f;
        for (int wv = 0; wv < 8; ++wv) {
            a += s_z[wv];
            h += s_ent[wv];
        }
        blk_z[blockIdx.x] = a;
        blk_ent[blockIdx.x] = h;
    }
    // the block that finishes last reduces every block's partials
    __threadfence();
    __syncthreads();
    __shared__ int s_last;
    if (threadIdx.x == 0) s_last = atomicAdd(counter, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    __shared__ double s_d[kStatD];
    __shared__ long long s_c[kStatC];
    finish_router_stats(blk_mp, blk_z, blk_ent, blk_cnt, (int)gridDim.x, T, E, K, mean_prob, losses,
                        s_d, s_c, (int)blockDim.x, (int)threadIdx.x, [] { __syncthreads(); });
    if (threadIdx.x == 0) *counter = 0;
}

// DeepSeek-V3 selection-bias step: b[e] += gamma * sign(mean(counts) - counts[e]).
__global__ void __launch_bounds__(256) update_bias_kernel(const int32_t* __restrict__ counts, int E,
                                                          float gamma, float* __restrict__ b)
{
    __shared__ long long s_sum;
    if (threadIdx.x == 0) {
        long long sum = 0;
        for (int e = 0; e < E; ++e) sum += counts[e];
        s_sum = sum;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        // sign(sum/E - c) == sign(sum - c*E): exact in integers
        const long long d = s_sum - (long long)counts[e] * E;
        const float sg = d > 0 ? 1.0f : (d < 0 ? -1.0f : 0.0f);
        b[e] += gamma * sg;
    }
}

cudaError_t launch_update_bias(int E, const int32_t* counts, float gamma, float* bias, cudaStream_t s)
{
    update_bias_kernel<<<1, 256, 0, s>>>(counts, E, gamma, bias);
    return cudaGetLastError();
}

template <typename XT>
static void launch_logits(const moe_config& c, const RouterPlan& rp, const XT* x, const float* w,
                          float* part, cudaStream_t s)
{
    dim3 grid(rp.grid_t, rp.grid_e, rp.splits);
    switch (rp.be) {
        case 8:
            router_logits_kernel<XT, 8, 4, 1><<<grid, 256, 0, s>>>(x, w, part, c.T, c.D, c.E,
                                                                   rp.d_per_split);
            break;
        case 16:
            router_logits_kernel<XT, 16, 4, 1><<<grid, 256, 0, s>>>(x, w, part, c.T, c.D, c.E,
                                                                    rp.d_per_split);
            break;
        case 32:
            router_logits_kernel<XT, 32, 4, 2><<<grid, 256, 0, s>>>(x, w, part, c.T, c.D, c.E,
                                                                    rp.d_per_split);
            break;
        default:
            router_logits_kernel<XT, 64, 4, 4><<<grid, 256, 0, s>>>(x, w, part, c.T, c.D, c.E,
                                                                    rp.d_per_split);
            break;
    }
}

// softmax / sigmoid, top-k, weights and statistic partials from `splits`
// partial logit buffers (T x E each), summed in split order
static cudaError_t launch_topk(const moe_config& c, const RouteOpts& o, const float* part, int splits,
                               const float* bias, const float* noise, float* logits_out, float* probs_out,
                               int32_t* ids, float* w, float* blk_mp, float* blk_z, float* blk_ent,
                               int32_t* blk_cnt, int with_stats, float* mean_prob, float* losses,
                               int* counter, const RouterPlan& rp, cudaStream_t s)
{
    const int epl = (c.E + 31) / 32;
    dim3 grid(rp.nb_topk);
#define MOE_TOPK(N)                                                                                     \
    router_topk_kernel<N><<<grid, 256, 0, s>>>(part, splits, bias, noise, o, logits_out, probs_out, ids, \
                                               w, blk_mp, blk_z, blk_ent, blk_cnt, c.T, c.E, c.K,       \
                                               with_stats, mean_prob, losses, counter, rp.tpb_topk)
    switch (epl) {
        case 1: MOE_TOPK(1); break;
        case 2: MOE_TOPK(2); break;
        case 3:
        case 4: MOE_TOPK(4); break;
        default: MOE_TOPK(8); break;
    }
#undef MOE_TOPK
    return cudaGetLastError();
}

cudaError_t launch_router(const moe_config& c, const RouterPlan& rp, const void* x,
                          const float* w_router, const void* terms, const float* bias,
                          const float* sel_bias, const float* noise, const float* logits_in, float* logits_out,
                          float* probs_out, int32_t* ids, float* w, float* mean_prob,
                          float* losses, char* ws, const WsLayout& L, cudaStream_t s)
{
    const RouteOpts o = route_opts(c, sel_bias);
    const int with_stats = (mean_prob != nullptr || losses != nullptr) ? 1 : 0;
    float* blk_mp = reinterpret_cast<float*>(ws + L.r_mp);
    float* blk_z = reinterpret_cast<float*>(ws + L.r_z);
    float* blk_ent = reinterpret_cast<float*>(ws + L.r_ent);
    int32_t* blk_cnt = reinterpret_cast<int32_t*>(ws + L.r_cnt);
    int* status = reinterpret_cast<int*>(ws + L.status);
    const float* part;
    int splits = 1;
    // bf16 layers with enough tokens: the tensor-core router, on the caller's
    // prepared weight terms or on terms split here into the workspace
    if (!logits_in && router_tc_eligible(c)) {
        if (terms == nullptr) {
            void* own = ws + L.r_terms;
            const cudaError_t e = launch_router_prepare(c, w_router, own, s);
            if (e != cudaSuccess) return e;
            terms = own;
        }
        return launch_router_tc(c, o, x, terms, bias, noise, logits_out, probs_out, ids, w, blk_mp,
                                blk_z, blk_ent, blk_cnt, mean_prob, losses, status, s);
    }
    if (logits_in) {
        part = logits_in;
        bias = nullptr;
        noise = nullptr;
    } else {
        float* p = reinterpret_cast<float*>(ws + L.r_part);
        if (c.dtype == MOE_BF16)
            launch_logits(c, rp, static_cast<const __nv_bfloat16*>(x), w_router, p, s);
        else
            launch_logits(c, rp, static_cast<const float*>(x), w_router, p, s);
        if (rp.splits > kTopkMaxSplits) {
            const int64_t n = c.T * c.E;
            int64_t blocks = (n + 255) / 256;
            if (blocks > 148 * 16) blocks = 148 * 16;
            router_splitsum_kernel<<<(unsigned)blocks, 256, 0, s>>>(p, rp.splits, n);
        } else {
            splits = rp.splits;  // few splits: the top-k kernel adds them in order
        }
        part = p;
    }
    return launch_topk(c, o, part, splits, bias, noise, logits_out, probs_out, ids, w, blk_mp, blk_z,
                       blk_ent, blk_cnt, with_stats, mean_prob, losses, status + kRouterCounterWord, rp, s);
}

}  // namespace moe
