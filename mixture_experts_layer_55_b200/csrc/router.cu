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
//   router_topk_kernel    one warp per token: sums the split partials in a
//                         fixed order, adds bias and noise, softmax, top-k by
//                         (logit desc, id asc) with warp shuffles, weights,
//                         and per-block statistic partials.
//   router_finalize_kernel fixed-order reduction of the block partials.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kLogitsBT = 64;  // tokens per logits block
constexpr int kLogitsBD = 32;  // d_model per smem step
constexpr int kTopkTPB = 64;   // tokens per top-k block (8 warps x 8)

RouterPlan router_plan(const moe_config& c)
{
    RouterPlan p;
    p.be = c.E <= 8 ? 8 : c.E <= 16 ? 16 : c.E <= 32 ? 32 : 64;
    p.grid_t = (int)((c.T + kLogitsBT - 1) / kLogitsBT);
    p.grid_e = (c.E + p.be - 1) / p.be;
    int64_t base = (int64_t)p.grid_t * p.grid_e;
    int want = (int)((2 * 148 + base - 1) / base);
    int max_splits = c.D / 256 > 1 ? c.D / 256 : 1;
    if (want > max_splits) want = max_splits;
    if (want < 1) want = 1;
    int dps = (c.D + want - 1) / want;
    dps = (dps + kLogitsBD - 1) / kLogitsBD * kLogitsBD;
    p.d_per_split = dps;
    p.splits = (c.D + dps - 1) / dps;
    p.nb_topk = (int)((c.T + kTopkTPB - 1) / kTopkTPB);
    return p;
}

// Thread layout: 256 threads = (BT/TM) token groups x (BE/TE) expert groups.
// Thread (ty, tx) owns tokens ty + i*(BT/TM) and experts tx + j*(BE/TE), so
// that neighbouring threads read neighbouring shared-memory words.
template <typename XT, int BE, int TM, int TE>
__global__ void __launch_bounds__(256) router_logits_kernel(const XT* __restrict__ x,
                                                            const float* __restrict__ w,
                                                            float* __restrict__ part, int64_t T,
                                                            int D, int E, int dps)
{
    constexpr int BT = kLogitsBT, BD = kLogitsBD;
    constexpr int NTX = BE / TE, NTY = BT / TM;
    static_assert(NTX * NTY == 256, "256 threads");
    __shared__ float xs[BD][BT + 1];
    __shared__ float wsm[BD][BE];

    const int tid = threadIdx.x;
    const int tx = tid % NTX, ty = tid / NTX;
    const int64_t t0 = (int64_t)blockIdx.x * BT;
    const int e0 = blockIdx.y * BE;
    const int d_begin = blockIdx.z * dps;
    const int d_end = min(D, d_begin + dps);

    float acc[TM][TE];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

    for (int d0 = d_begin; d0 < d_end; d0 += BD) {
        // x tile: BT tokens x BD columns, stored transposed (d-major).
        for (int idx = tid; idx < BT * BD; idx += 256) {
            int tt = idx / BD, dd = idx % BD;
            int64_t t = t0 + tt;
            int d = d0 + dd;
            float v = 0.f;
            if (t < T && d < d_end) v = to_f32(x[t * D + d]);
            xs[dd][tt] = v;
        }
        for (int idx = tid; idx < BD * BE; idx += 256) {
            int dd = idx / BE, ee = idx % BE;
            int d = d0 + dd, e = e0 + ee;
            wsm[dd][ee] = (d < d_end && e < E) ? w[(int64_t)d * E + e] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int dd = 0; dd < BD; ++dd) {
            float xv[TM], wv[TE];
#pragma unroll
            for (int i = 0; i < TM; ++i) xv[i] = xs[dd][ty + i * NTY];
#pragma unroll
            for (int j = 0; j < TE; ++j) wv[j] = wsm[dd][tx + j * NTX];
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TE; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* out = part + (size_t)blockIdx.z * (size_t)T * E;
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        int64_t t = t0 + ty + i * NTY;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < TE; ++j) {
            int e = e0 + tx + j * NTX;
            if (e < E) out[t * E + e] = acc[i][j];
        }
    }
}

// (value desc, id asc) ordering: does candidate (va, ia) rank before (vb, ib)?
MOE_DEVICE bool ranks_before(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// One warp per token.  Lane l holds experts l, l+32, ... (EPL of them).
template <int EPL>
__global__ void __launch_bounds__(256) router_topk_kernel(
    const float* __restrict__ part, int splits, const float* __restrict__ bias,
    const float* __restrict__ noise, float* __restrict__ logits_out, float* __restrict__ probs_out,
    int32_t* __restrict__ ids, float* __restrict__ wout, float* __restrict__ blk_mp,
    float* __restrict__ blk_z, int32_t* __restrict__ blk_cnt, int64_t T, int E, int K,
    int with_stats)
{
    __shared__ float s_mp[8][256];
    __shared__ int s_cnt[8][256];
    __shared__ float s_z[8];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float mp_acc[EPL];
    int cnt_acc[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        mp_acc[j] = 0.f;
        cnt_acc[j] = 0;
    }
    float z_acc = 0.f;

    const int64_t tbase = (int64_t)blockIdx.x * kTopkTPB;
    for (int i = 0; i < kTopkTPB / 8; ++i) {
        const int64_t t = tbase + warp + 8 * i;
        if (t >= T) break;
        float L[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            int e = lane + 32 * j;
            float v = -INFINITY;
            if (e < E) {
                v = part[t * E + e];
                for (int s = 1; s < splits; ++s) v += part[(size_t)s * T * E + t * E + e];
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
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float ex[EPL];
        float ssum = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            ex[j] = (lane + 32 * j < E) ? expf(L[j] - m) : 0.f;
            ssum += ex[j];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
        const float inv = 1.0f / ssum;
        float p[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            p[j] = ex[j] * inv;
            int e = lane + 32 * j;
            if (e < E) {
                if (probs_out) probs_out[t * E + e] = p[j];
                mp_acc[j] += p[j];
            }
        }
        if (lane == 0) {
            float lse = m + logf(ssum);
            z_acc = fmaf(lse, lse, z_acc);
        }
        // top-K: K rounds of a warp-wide arg-best over the not-yet-taken experts.
        uint32_t taken = 0;  // bit j: expert lane+32j already selected
        float sel_p[8];
        int sel_id[8];
        float psum = 0.f;
        for (int k = 0; k < K; ++k) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                int e = lane + 32 * j;
                if (e < E && !((taken >> j) & 1u) && ranks_before(L[j], e, bv, bi)) {
                    bv = L[j];
                    bi = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ranks_before(ov, oi, bv, bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            // the owner lane marks it taken and broadcasts its probability
            float pk = 0.f;
            if ((bi & 31) == lane) {
                int j = bi >> 5;
#pragma unroll
                for (int jj = 0; jj < EPL; ++jj)
                    if (jj == j) {
                        taken |= 1u << jj;
                        pk = p[jj];
                        cnt_acc[jj] += 1;
                    }
            }
            pk = __shfl_sync(0xffffffffu, pk, bi & 31);
            sel_p[k] = pk;
            sel_id[k] = bi;
            psum += pk;
        }
        if (lane < K) {
            float pk = 0.f;
            int idk = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k == lane) {
                    pk = sel_p[k];
                    idk = sel_id[k];
                }
            ids[t * K + lane] = idk;
            wout[t * K + lane] = pk / psum;
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
    if (lane == 0) s_z[warp] = z_acc;
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
        float a = 0.f;
        for (int wv = 0; wv < 8; ++wv) a += s_z[wv];
        blk_z[blockIdx.x] = a;
    }
}

// One block: mean_prob[e] = (1/T) sum_b blk_mp[b][e]; losses = {z, balance}.
// Cross-block sums in double, in block order.
__global__ void __launch_bounds__(256) router_finalize_kernel(const float* __restrict__ blk_mp,
                                                              const float* __restrict__ blk_z,
                                                              const int32_t* __restrict__ blk_cnt,
                                                              int nb, int64_t T, int E, int K,
                                                              float* __restrict__ mean_prob,
                                                              float* __restrict__ losses)
{
    __shared__ double s_term[256];
    const int e = threadIdx.x;
    double term = 0.0;
    if (e < E) {
        double mp = 0.0;
        long long cn = 0;
        for (int b = 0; b < nb; ++b) {
            mp += (double)blk_mp[(size_t)b * E + e];
            cn += blk_cnt[(size_t)b * E + e];
        }
        mp /= (double)T;
        if (mean_prob) mean_prob[e] = (float)mp;
        term = ((double)cn / ((double)T * (double)K)) * mp;
    }
    s_term[e] = term;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (e < o) s_term[e] += s_term[e + o];
        __syncthreads();
    }
    if (e == 0 && losses) {
        double z = 0.0;
        for (int b = 0; b < nb; ++b) z += (double)blk_z[b];
        losses[0] = (float)(z / (double)T);
        losses[1] = (float)((double)E * s_term[0]);
    }
}

template <typename XT>
static void launch_logits(const moe_config& c, const RouterPlan& rp, const XT* x, const float* w,
                          float* part, cudaStream_t s)
{
    dim3 grid(rp.grid_t, rp.grid_e, rp.splits);
    switch (rp.be) {
        case 8:
            router_logits_kernel<XT, 8, 2, 1><<<grid, 256, 0, s>>>(x, w, part, c.T, c.D, c.E,
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

cudaError_t launch_router(const moe_config& c, const RouterPlan& rp, const void* x,
                          const float* w_router, const float* bias, const float* noise,
                          const float* logits_in, float* logits_out, float* probs_out,
                          int32_t* ids, float* w, float* mean_prob, float* losses, char* ws,
                          const WsLayout& L, cudaStream_t s)
{
    const float* part;
    int splits;
    if (logits_in) {
        part = logits_in;
        splits = 1;
        bias = nullptr;
        noise = nullptr;
    } else {
        float* p = reinterpret_cast<float*>(ws + L.r_part);
        if (c.dtype == MOE_BF16)
            launch_logits(c, rp, static_cast<const __nv_bfloat16*>(x), w_router, p, s);
        else
            launch_logits(c, rp, static_cast<const float*>(x), w_router, p, s);
        part = p;
        splits = rp.splits;
    }
    const int with_stats = (mean_prob != nullptr || losses != nullptr) ? 1 : 0;
    float* blk_mp = reinterpret_cast<float*>(ws + L.r_mp);
    float* blk_z = reinterpret_cast<float*>(ws + L.r_z);
    int32_t* blk_cnt = reinterpret_cast<int32_t*>(ws + L.r_cnt);
    const int epl = (c.E + 31) / 32;
    dim3 grid(rp.nb_topk);
#define MOE_TOPK(N)                                                                              \
    router_topk_kernel<N><<<grid, 256, 0, s>>>(part, splits, bias, noise, logits_out, probs_out, \
                                               ids, w, blk_mp, blk_z, blk_cnt, c.T, c.E, c.K,   \
                                               with_stats)
    switch (epl) {
        case 1: MOE_TOPK(1); break;
        case 2: MOE_TOPK(2); break;
        case 3:
        case 4: MOE_TOPK(4); break;
        default: MOE_TOPK(8); break;
    }
#undef MOE_TOPK
    if (with_stats)
        router_finalize_kernel<<<1, 256, 0, s>>>(blk_mp, blk_z, blk_cnt, rp.nb_topk, c.T, c.E, c.K,
                                                 mean_prob, losses);
    return cudaGetLastError();
}

}  // namespace moe
