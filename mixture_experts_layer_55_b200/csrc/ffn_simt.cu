// ffn_simt.cu -- grouped SwiGLU expert FFN in true fp32 on the SIMT pipes
// (no TF32), for layers whose dtype is fp32.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation"
// (SwiGLUExpert: down(silu(gate x) * up x); each expert output scaled by its
// combine weight).  Two launches over each expert's contiguous row block:
//   gate/up: h = silu(x_perm Wg_e) * (x_perm Wu_e)         (rows x F)
//            (the training forward also keeps [g | u], rows x 2F)
//   down:    y_perm = topk_w[perm[row]] * (h Wd_e)         (rows x D)
// Tiles are 64 rows x 64 columns; the m-tile -> (expert, first row) map is
// derived on the device from the offsets (no host synchronisation).
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kSBM = 64, kSBN = 64, kSBK = 16;

// s_pref[e] = number of kSBM-row tiles of experts < e; s_pref[E] = total.
MOE_DEVICE void simt_tile_prefix(const int32_t* offsets, int E, int64_t max_rows, int* s_off,
                                 int* s_pref, int* status)
{
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        int prev = 0;
        for (int e = 0; e < E; ++e) {
            int a = s_off[e], b = s_off[e + 1];
            if (a < prev || b < a || b > max_rows) {  // malformed offsets: treat as empty
                raise_flag(status, kFlagBounds, 300);
                b = a = prev;
            }
            prev = b;
            s_pref[e] = run;
            run += (b - a + kSBM - 1) / kSBM;
        }
        s_pref[E] = run;
    }
    __syncthreads();
}

template <typename T, bool GATEUP>
__global__ void __launch_bounds__(256) ffn_simt_kernel(const T* __restrict__ A,
                                                       const T* __restrict__ B0,
                                                       const T* __restrict__ B1, T* __restrict__ out,
                                                       const int32_t* __restrict__ offsets,
                                                       const int32_t* __restrict__ perm,
                                                       const float* __restrict__ topk_w, int E,
                                                       int Kd, int N, int64_t max_rows, int64_t nk,
                                                       T* __restrict__ gu_keep, int* status)
{
    __shared__ int s_off[257];
    __shared__ int s_pref[257];
    __shared__ float As[kSBK][kSBM + 4];
    __shared__ float Bs0[kSBK][kSBN];
    __shared__ float Bs1[GATEUP ? kSBK : 1][kSBN];

    simt_tile_prefix(offsets, E, max_rows, s_off, s_pref, status);
    const int mt = blockIdx.y;
    if (mt >= s_pref[E]) return;
    int e = 0;
    while (e + 1 < E && s_pref[e + 1] <= mt) ++e;  // experts with no tiles are skipped
    const int64_t row0 = (int64_t)s_off[e] + (int64_t)(mt - s_pref[e]) * kSBM;
    const int64_t row_end = s_off[e + 1];
    const int n0 = blockIdx.x * kSBN;

    const T* Bg = B0 + (size_t)e * Kd * N;
    const T* Bu = GATEUP ? B1 + (size_t)e * Kd * N : nullptr;

    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;  // 4x4 outputs: rows ty+16i, cols tx+16j
    float acc0[4][4], acc1[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.f;

    for (int k0 = 0; k0 < Kd; k0 += kSBK) {
        for (int idx = tid; idx < kSBM * kSBK; idx += 256) {
            int r = idx / kSBK, kk = idx % kSBK;
            int64_t row = row0 + r;
            int k = k0 + kk;
            As[kk][r] = (row < row_end && k < Kd) ? to_f32(A[row * Kd + k]) : 0.f;
        }
        for (int idx = tid; idx < kSBK * kSBN; idx += 256) {
            int kk = idx / kSBN, cc = idx % kSBN;
            int k = k0 + kk, col = n0 + cc;
            bool ok = k < Kd && col < N;
            Bs0[kk][cc] = ok ? to_f32(Bg[(size_t)k * N + col]) : 0.f;
            if (GATEUP) Bs1[kk][cc] = ok ? to_f32(Bu[(size_t)k * N + col]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kSBK; ++kk) {
            float a[4], b0[4], b1[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                b0[j] = Bs0[kk][tx + 16 * j];
                if (GATEUP) b1[j] = Bs1[kk][tx + 16 * j];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
                    if (GATEUP) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t row = row0 + ty + 16 * i;
        if (row >= row_end) continue;
        float wr = 1.f;
        if (!GATEUP && perm != nullptr) {  // no perm: unit weights (a shared expert)
            const int32_t pa = perm[row];
            if (pa < 0 || pa >= nk) {
                raise_flag(status, kFlagBounds, 301);
                wr = 0.f;
            } else {
                wr = topk_w[pa];
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int col = n0 + tx + 16 * j;
            if (col >= N) continue;
            float v = GATEUP ? silu_f32(acc0[i][j]) * acc1[i][j] : wr * acc0[i][j];
            out[row * N + col] = from_f32<T>(v);
            if (GATEUP && gu_keep != nullptr) {  // [g | u] for the backward
                gu_keep[row * 2 * N + col] = from_f32<T>(acc0[i][j]);
                gu_keep[row * 2 * N + N + col] = from_f32<T>(acc1[i][j]);
            }
        }
    }
}

// Upper bound of the m-tiles: sum_e ceil(kept_e / BM) <= max_rows / BM + E.
static inline int64_t simt_mtiles_bound(int64_t max_rows, int E)
{
    return (max_rows + kSBM - 1) / kSBM + E;
}

template <typename T>
static cudaError_t launch_simt(const moe_config& c, int64_t max_rows, const void* x_perm,
                               const int32_t* offsets, const int32_t* perm, const float* topk_w,
                               const void* w_gate, const void* w_up, const void* w_down, void* h,
                               void* y_perm, void* gu_keep, int* status, cudaStream_t s, StageHook mid,
                               void* mid_ctx)
{
    const int64_t mtiles = simt_mtiles_bound(max_rows, c.E);
    const int64_t nk = c.T * c.K;
    dim3 g1((c.F + kSBN - 1) / kSBN, (unsigned)mtiles);
    ffn_simt_kernel<T, true><<<g1, 256, 0, s>>>(
        static_cast<const T*>(x_perm), static_cast<const T*>(w_gate), static_cast<const T*>(w_up),
        static_cast<T*>(h), offsets, perm, topk_w, c.E, c.D, c.F, max_rows, nk, static_cast<T*>(gu_keep),
        status);
    if (mid) mid(mid_ctx, s);
    dim3 g2((c.D + kSBN - 1) / kSBN, (unsigned)mtiles);
    ffn_simt_kernel<T, false><<<g2, 256, 0, s>>>(
        static_cast<const T*>(h), static_cast<const T*>(w_down), nullptr, static_cast<T*>(y_perm),
        offsets, perm, topk_w, c.E, c.F, c.D, max_rows, nk, nullptr, status);
    return cudaGetLastError();
}

cudaError_t launch_ffn_simt_f32(const moe_config& c, int64_t max_rows, const void* x_perm,
                                const int32_t* offsets, const int32_t* perm, const float* topk_w,
                                const void* w_gate, const void* w_up, const void* w_down, void* h,
                                void* y_perm, void* gu_keep, int* status, cudaStream_t s, StageHook mid,
                                void* mid_ctx)
{
    return launch_simt<float>(c, max_rows, x_perm, offsets, perm, topk_w, w_gate, w_up, w_down, h,
                              y_perm, gu_keep, status, s, mid, mid_ctx);
}

}  // namespace moe
