// bwd.cu -- the memory-bound steps of the layer's backward.
//
// "Lab: build a tiny MoE in PyTorch", "Smoke test and backward pass": the
// training loss main + c_bal * balance + c_z * z is differentiated through
// the layer; "2.9 Mixture-of-Experts (MoE) Architectures", "The Router": the
// top-k index decision is a stop-gradient, so the router learns only through
// the kept gate weights and the auxiliary losses.  With dY the gradient of y:
//
//   rows       dYp[r] = w_r * dY[t_r] (in the layer dtype),  dw_r = <dY[t_r], o_r>
//              (o_r = the expert's unweighted output the forward kept)
//   router     dL[t] from the gate weights' dw (renormalised or not, route
//              scale), the balance loss through the normalised scores (counts
//              fixed) and the z-loss through the logsumexp
//   linear     dW_r = x^T dL (split over tokens, then a fixed-order sum of the
//              splits), db = sum_t dL[t] (a fixed-order tree): deterministic
//   dx         dx[t] = dL[t] W_r^T + sum over kept slots of dXp[row] (+ the
//              shared expert's), rounded once
// No atomics anywhere: every result is bit-reproducible.
#include "common.cuh"
#include "internal.h"

namespace moe {

// ------------------------------------------------------------------- rows --
// One warp per row of the expert-major layout; 16-byte vectors (8 bf16 or 4
// fp32 elements).
template <typename ET>
__global__ void __launch_bounds__(256) bwd_rows_kernel(const uint4* __restrict__ dy,
                                                       const uint4* __restrict__ o,
                                                       const int32_t* __restrict__ offsets,
                                                       const int32_t* __restrict__ perm,
                                                       const float* __restrict__ topk_w,
                                                       uint4* __restrict__ dyp, float* __restrict__ dw_row,
                                                       int E, int K, int64_t vpr, int64_t nk,
                                                       int64_t max_rows, int* status)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    int64_t rows = offsets[E];
    if (rows > max_rows || rows < 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_flag(status, kFlagBounds, 600);
        rows = rows < 0 ? 0 : max_rows;
    }
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int32_t pa = perm[r];
        if (pa < 0 || (int64_t)pa >= nk) {
            if (lane == 0) raise_flag(status, kFlagBounds, 601);
            continue;
        }
        const int64_t t = pa / K;
        const float w = topk_w[pa];
        const uint4* dyt = dy + t * vpr;
        const uint4* orow = o + r * vpr;
        uint4* drow = dyp + r * vpr;
        float dot = 0.f;
        for (int64_t v = lane; v < vpr; v += 32) {
            const uint4 a = __ldg(dyt + v), b = __ldg(orow + v);
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
            uint32_t pw[4];
            if constexpr (sizeof(ET) == 2) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float a0 = __uint_as_float(aw[i] << 16), a1 = __uint_as_float(aw[i] & 0xffff0000u);
                    const float b0 = __uint_as_float(bw[i] << 16), b1 = __uint_as_float(bw[i] & 0xffff0000u);
                    dot = fmaf(a0, b0, dot);
                    dot = fmaf(a1, b1, dot);
                    pw[i] = pack_bf16x2(w * a0, w * a1);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float a0 = __uint_as_float(aw[i]), b0 = __uint_as_float(bw[i]);
                    dot = fmaf(a0, b0, dot);
                    pw[i] = __float_as_uint(w * a0);
                }
            }
            drow[v] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        }
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, s);
        if (lane == 0) dw_row[r] = dot;
    }
}

// ----------------------------------------------------------------- router --
constexpr int kMaxEPerLane = 8;  // E <= 256 = 32 lanes x 8

MOE_DEVICE float warp_sum(float v)
{
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
    return v;
}

MOE_DEVICE float warp_max(float v)
{
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, s));
    return v;
}

// One warp per token; lane l holds experts l, l + 32, ...
__global__ void __launch_bounds__(256) router_bwd_kernel(const float* __restrict__ logits,
                                                         const int32_t* __restrict__ ids,
                                                         const int32_t* __restrict__ row_of,
                                                         const float* __restrict__ dw_row,
                                                         const int32_t* __restrict__ counts,
                                                         float* __restrict__ dlogits, int64_t T, int E,
                                                         int K, int score_func, int renorm,
                                                         float route_scale, float c_bal, float c_z,
                                                         int64_t max_rows, int* status)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* L = logits + t * E;
    float l[kMaxEPerLane];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxEPerLane; ++j) {
        const int e = lane + 32 * j;
        l[j] = e < E ? L[e] : -INFINITY;
        mx = fmaxf(mx, l[j]);
    }
    mx = warp_max(mx);
    float se = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxEPerLane; ++j) se += (lane + 32 * j < E) ? expf(l[j] - mx) : 0.f;
    se = warp_sum(se);
    const float lse = mx + logf(se);
    const bool sig = score_func == 1;
    // gate weights: every lane evaluates the K chosen scores itself
    float S = 0.f, sdw = 0.f;
    int idk[8];
    float dwk[8], sck[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        idk[k] = -1;
        dwk[k] = 0.f;
        sck[k] = 0.f;
        if (k < K) {
            int id = ids[t * K + k];
            if (id < 0 || id >= E) {
                if (lane == 0) raise_flag(status, kFlagBounds, 610);
                continue;
            }
            idk[k] = id;
            const float li = L[id];
            sck[k] = sig ? 1.f / (1.f + expf(-li)) : expf(li - mx) / se;
            const int32_t r = row_of[t * K + k];
            dwk[k] = (r >= 0 && r < max_rows) ? dw_row[r] : 0.f;  // a dropped slot: 0
            S += sck[k];
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) sdw += dwk[k] * sck[k] / S;
    float p[kMaxEPerLane], sc[kMaxEPerLane], ds[kMaxEPerLane];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxEPerLane; ++j) {
        const int e = lane + 32 * j;
        const bool in = e < E;
        p[j] = in ? expf(l[j] - mx) / se : 0.f;
        sc[j] = in ? (sig ? 1.f / (1.f + expf(-l[j])) : p[j]) : 0.f;
        ss += sc[j];
        float d = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (idk[k] == e) d += renorm ? route_scale / S * (dwk[k] - sdw) : route_scale * dwk[k];
        ds[j] = d;
    }
    // the balance loss: d n[e] = c_bal * E * f_e / T, f_e = counts_e / (T K)
    const float bal_scale = c_bal * (float)E / ((float)T * (float)K) / (float)T;
    if (sig) {
        ss = warp_sum(ss);
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxEPerLane; ++j) {
            const int e = lane + 32 * j;
            if (e < E) dot += bal_scale * (float)counts[e] * (sc[j] / ss);
        }
        dot = warp_sum(dot);
#pragma unroll
        for (int j = 0; j < kMaxEPerLane; ++j) {
            const int e = lane + 32 * j;
            if (e < E) ds[j] += (bal_scale * (float)counts[e] - dot) / ss;
        }
    } else {
#pragma unroll
        for (int j = 0; j < kMaxEPerLane; ++j) {
            const int e = lane + 32 * j;
            if (e < E) ds[j] += bal_scale * (float)counts[e];
        }
    }
    // the scores from the logits, then the z-loss
    float dot2 = 0.f;
    if (!sig) {
#pragma unroll
        for (int j = 0; j < kMaxEPerLane; ++j) dot2 += p[j] * ds[j];
        dot2 = warp_sum(dot2);
    }
    const float zc = c_z * 2.f * lse / (float)T;
#pragma unroll
    for (int j = 0; j < kMaxEPerLane; ++j) {
        const int e = lane + 32 * j;
        if (e >= E) continue;
        const float g = sig ? ds[j] * sc[j] * (1.f - sc[j]) : p[j] * (ds[j] - dot2);
        dlogits[t * E + e] = g + zc * p[j];
    }
}

// ---------------------------------------------------- router weight grads --
// 8 consecutive d of x as fp32 (one 16-byte load for bf16, two for fp32).
MOE_DEVICE void load8(const __nv_bfloat16* p, float (&v)[8])
{
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
MOE_DEVICE void load8(const float* p, float (&v)[8])
{
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
MOE_DEVICE void store8(__nv_bfloat16* p, const float (&v)[8])
{
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                              pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}
MOE_DEVICE void store8(float* p, const float (&v)[8])
{
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

constexpr int kRwCols = 256;  // d per block
constexpr int kRwE = 32;      // experts per block
constexpr int kRwTok = 32;    // tokens staged per step

// part[z][d][e] = sum over the tokens of split z of x[t,d] * dL[t,e].  Block:
// 256 d x 32 experts, 256 threads; thread (ty = warp, tx = lane) owns
// d = 8 tx .. 8 tx + 7 and experts 4 ty .. 4 ty + 3.  Tokens are staged 32 at
// a time (x with 16-byte loads; dL reads in the loop are warp broadcasts).
template <typename XT>
__global__ void __launch_bounds__(256) router_wgrad_partial_kernel(const XT* __restrict__ x,
                                                                   const float* __restrict__ dL,
                                                                   float* __restrict__ part, int64_t T,
                                                                   int D, int E, int64_t t_per_split)
{
    __shared__ __align__(16) XT sx[kRwTok][kRwCols];
    __shared__ float sdl[kRwTok][kRwE];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int dblk = blockIdx.x * kRwCols;
    const int e0 = blockIdx.y * kRwE;
    const int64_t t0 = (int64_t)blockIdx.z * t_per_split;
    const int64_t t1 = t0 + t_per_split < T ? t0 + t_per_split : T;
    constexpr int VEC = 16 / sizeof(XT);  // elements per 16-byte load
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int64_t tc = t0; tc < t1; tc += kRwTok) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kRwTok * kRwCols / VEC; idx += 256) {
            const int tt = idx / (kRwCols / VEC), v = idx - tt * (kRwCols / VEC);
            const int d = dblk + v * VEC;
            uint4 q = make_uint4(0, 0, 0, 0);
            if (tc + tt < t1 && d < D) q = __ldg(reinterpret_cast<const uint4*>(x + (tc + tt) * D + d));
            *reinterpret_cast<uint4*>(&sx[tt][v * VEC]) = q;
        }
        for (int idx = threadIdx.x; idx < kRwTok * kRwE; idx += 256) {
            const int tt = idx / kRwE, el = idx - tt * kRwE;
            sdl[tt][el] = (tc + tt < t1 && e0 + el < E) ? __ldg(dL + (tc + tt) * E + e0 + el) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < kRwTok; ++tt) {
            float xv[8];
            if constexpr (sizeof(XT) == 2) {
                const uint4 q = *reinterpret_cast<const uint4*>(&sx[tt][tx * 8]);
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    xv[2 * i] = __uint_as_float(w[i] << 16);
                    xv[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) xv[i] = to_f32(sx[tt][tx * 8 + i]);
            }
            float g[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) g[j] = sdl[tt][ty * 4 + j];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xv[i], g[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int d = dblk + tx * 8 + i;
        if (d >= D) break;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + ty * 4 + j;
            if (e < E) part[((int64_t)blockIdx.z * D + d) * E + e] = acc[i][j];
        }
    }
}

// dW[d][e] = sum over splits in order.
__global__ void router_wgrad_reduce_kernel(const float* __restrict__ part, int splits, int D, int E,
                                           float* __restrict__ dw)
{
    const int64_t n = (int64_t)D * E;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int k = 0; k < splits; ++k) s += part[(int64_t)k * n + i];
        dw[i] = s;
    }
}

// db[e] = sum_t dL[t,e]: one block per expert, a fixed-order tree.
__global__ void __launch_bounds__(256) router_bias_grad_kernel(const float* __restrict__ dL, int64_t T,
                                                               int E, float* __restrict__ db)
{
    __shared__ float red[256];
    const int e = blockIdx.x;
    float s = 0.f;
    for (int64_t t = threadIdx.x; t < T; t += 256) s += dL[t * E + e];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) db[e] = red[0];
}

// --------------------------------------------------------------------- dx --
// Block: 64 tokens x 256 d, 256 threads; thread (ty = warp, tx = lane) owns
// tokens 8 ty .. 8 ty + 7 and d = 8 tx .. 8 tx + 7 of the tile.  The router
// term dL W_r^T is a small product over the experts, 32 at a time: the
// chunk's W_r^T (32 x 256, fp32) and dL (64 x 32) are staged in shared memory
// (lanes walk d when writing W_r^T, so the stores are conflict-free; the
// 16-byte reads of a W_r^T row are too, and dL reads are warp broadcasts).
// Then each token's kept rows of dXp (slot order) and the shared expert's row
// are added as 16-byte vectors, and the sum is rounded once.
constexpr int kDxTok = 64;
constexpr int kDxCols = 256;
constexpr int kDxE = 32;

template <typename ET, int KS>
__global__ void __launch_bounds__(256) dx_assemble_kernel(const float* __restrict__ dL,
                                                          const float* __restrict__ w_r,
                                                          const ET* __restrict__ dxp,
                                                          const int32_t* __restrict__ row_of,
                                                          const ET* __restrict__ dx_shared,
                                                          ET* __restrict__ dx, int64_t T, int D, int E,
                                                          int K, int64_t max_rows)
{
    __shared__ __align__(16) float swt[kDxE][kDxCols];
    __shared__ float sdl[kDxTok][kDxE + 1];
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int dblk = blockIdx.x * kDxCols;
    const int64_t tb = (int64_t)blockIdx.y * kDxTok;
    const int d0 = dblk + tx * 8;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int e0 = 0; e0 < E; e0 += kDxE) {
        __syncthreads();  // the previous chunk's shared reads are done
        for (int idx = threadIdx.x; idx < kDxE * kDxCols; idx += 256) {
            const int el = idx / kDxCols, dl = idx - el * kDxCols;
            const int d = dblk + dl;
            swt[el][dl] = (d < D && e0 + el < E) ? __ldg(w_r + (int64_t)d * E + e0 + el) : 0.f;
        }
        for (int idx = threadIdx.x; idx < kDxTok * kDxE; idx += 256) {
            const int tt = idx / kDxE, el = idx - tt * kDxE;
            sdl[tt][el] = (tb + tt < T && e0 + el < E) ? __ldg(dL + (tb + tt) * E + e0 + el) : 0.f;
        }
        __syncthreads();
        const int ne = E - e0 < kDxE ? E - e0 : kDxE;
        for (int e = 0; e < ne; ++e) {
            const float4 lo = *reinterpret_cast<const float4*>(&swt[e][tx * 8]);
            const float4 hi = *reinterpret_cast<const float4*>(&swt[e][tx * 8 + 4]);
            const float w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float g = sdl[ty * 8 + i][e];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(g, w[j], acc[i][j]);
            }
        }
    }
    if (d0 >= D) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t t = tb + ty * 8 + i;
        if (t >= T) break;
        // the token's KS >= K slot rows: indices first, then all loads in flight together
        int32_t rows[KS];
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int32_t r = k < K ? __ldg(row_of + t * K + k) : -1;
            rows[k] = (r >= 0 && r < max_rows) ? r : -1;
        }
        float v[KS][8];
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            if (rows[k] >= 0) load8(dxp + (int64_t)rows[k] * D + d0, v[k]);
            else
#pragma unroll
                for (int j = 0; j < 8; ++j) v[k][j] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < KS; ++k)  // slot order
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] += v[k][j];
        if (dx_shared) {
            float v[8];
            load8(dx_shared + t * D + d0, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] += v[j];
        }
        store8(dx + t * D + d0, acc[i]);
    }
}

// ------------------------------------------------------------------ host --
static int sm_count()
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

cudaError_t launch_bwd_rows(const moe_config& c, const void* dy, const void* o, const int32_t* offsets,
                            const int32_t* perm, const float* topk_w, void* dyp, float* dw_row,
                            int64_t max_rows, int* status, cudaStream_t s)
{
    const int64_t vpr = (int64_t)c.D * (c.dtype == MOE_BF16 ? 2 : 4) / 16;
    int64_t blocks = (max_rows + 7) / 8;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const uint4* dyv = static_cast<const uint4*>(dy);
    const uint4* ov = static_cast<const uint4*>(o);
    if (c.dtype == MOE_BF16)
        bwd_rows_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            dyv, ov, offsets, perm, topk_w, static_cast<uint4*>(dyp), dw_row, c.E, c.K, vpr, c.T * c.K,
            max_rows, status);
    else
        bwd_rows_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(
            dyv, ov, offsets, perm, topk_w, static_cast<uint4*>(dyp), dw_row, c.E, c.K, vpr, c.T * c.K,
            max_rows, status);
    return cudaGetLastError();
}

cudaError_t launch_router_bwd(const moe_config& c, const float* logits, const int32_t* ids,
                              const int32_t* row_of, const float* dw_row, const int32_t* counts,
                              float c_bal, float c_z, float* dlogits, int64_t max_rows, int* status,
                              cudaStream_t s)
{
    const int64_t blocks = (c.T + 7) / 8;
    router_bwd_kernel<<<(unsigned)blocks, 256, 0, s>>>(logits, ids, row_of, dw_row, counts, dlogits,
                                                        c.T, c.E, c.K, c.score_func, c.renormalize,
                                                        c.route_scale, c_bal, c_z, max_rows, status);
    return cudaGetLastError();
}

int router_wgrad_splits(const moe_config& c)
{
    // about four waves of blocks; each split at least 64 tokens
    const int64_t dblocks = (c.D + kRwCols - 1) / kRwCols;
    const int64_t eblocks = (c.E + kRwE - 1) / kRwE;
    int64_t want = (int64_t)sm_count() * 4 / (dblocks * eblocks);
    int64_t most = (c.T + 63) / 64;
    int64_t sp = want < most ? want : most;
    if (sp < 1) sp = 1;
    if (sp > 256) sp = 256;
    return (int)sp;
}

size_t router_wgrad_part_bytes(const moe_config& c, int splits)
{
    return (size_t)splits * (size_t)c.D * c.E * sizeof(float);
}

cudaError_t launch_router_wgrad(const moe_config& c, const void* x, const float* dL, float* part,
                                int splits, float* dw, float* db, cudaStream_t s)
{
    const int64_t tps = (c.T + splits - 1) / splits;
    const dim3 grid((unsigned)((c.D + kRwCols - 1) / kRwCols), (unsigned)((c.E + kRwE - 1) / kRwE),
                    (unsigned)splits);
    if (c.dtype == MOE_BF16)
        router_wgrad_partial_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(x), dL, part, c.T, c.D, c.E, tps);
    else
        router_wgrad_partial_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(x), dL, part,
                                                                c.T, c.D, c.E, tps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)c.D * c.E;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    router_wgrad_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(part, splits, c.D, c.E, dw);
    e = cudaGetLastError();
    if (e != cudaSuccess || db == nullptr) return e;
    router_bias_grad_kernel<<<(unsigned)c.E, 256, 0, s>>>(dL, c.T, c.E, db);
    return cudaGetLastError();
}

template <typename ET, int KS>
static void dx_launch(const moe_config& c, dim3 grid, const float* dL, const float* w_r, const void* dxp,
                      const int32_t* row_of, const void* dx_shared, void* dx, int64_t max_rows,
                      cudaStream_t s)
{
    dx_assemble_kernel<ET, KS><<<grid, 256, 0, s>>>(dL, w_r, static_cast<const ET*>(dxp), row_of,
                                                    static_cast<const ET*>(dx_shared), static_cast<ET*>(dx),
                                                    c.T, c.D, c.E, c.K, max_rows);
}

template <typename ET>
static void dx_launch_k(const moe_config& c, dim3 grid, const float* dL, const float* w_r, const void* dxp,
                        const int32_t* row_of, const void* dx_shared, void* dx, int64_t max_rows,
                        cudaStream_t s)
{
    if (c.K <= 1) dx_launch<ET, 1>(c, grid, dL, w_r, dxp, row_of, dx_shared, dx, max_rows, s);
    else if (c.K == 2) dx_launch<ET, 2>(c, grid, dL, w_r, dxp, row_of, dx_shared, dx, max_rows, s);
    else if (c.K <= 4) dx_launch<ET, 4>(c, grid, dL, w_r, dxp, row_of, dx_shared, dx, max_rows, s);
    else dx_launch<ET, 8>(c, grid, dL, w_r, dxp, row_of, dx_shared, dx, max_rows, s);
}

cudaError_t launch_dx_assemble(const moe_config& c, const float* dL, const float* w_r, const void* dxp,
                               const int32_t* row_of, const void* dx_shared, void* dx,
                               int64_t max_rows, cudaStream_t s)
{
    const dim3 grid((unsigned)((c.D + kDxCols - 1) / kDxCols), (unsigned)((c.T + kDxTok - 1) / kDxTok));
    if (c.dtype == MOE_BF16)
        dx_launch_k<__nv_bfloat16>(c, grid, dL, w_r, dxp, row_of, dx_shared, dx, max_rows, s);
    else
        dx_launch_k<float>(c, grid, dL, w_r, dxp, row_of, dx_shared, dx, max_rows, s);
    return cudaGetLastError();
}

}  // namespace moe
