// ffn_simt.cu -- grouped SwiGLU expert FFN in true fp32 on the SIMT pipes
// (no TF32), for layers whose dtype is fp32.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation"
// (SwiGLUExpert: down(silu(gate x) * up x); each expert output scaled by its
// combine weight).  Two launches over each expert's contiguous row block:
//   gate/up: h = silu(x_perm Wg_e) * (x_perm Wu_e)         (rows x F)
//            (the training forward also keeps [g | u], rows x 2F)
//   down:    y_perm = topk_w[perm[row]] * (h Wd_e)         (rows x D)
// Tiles are 32 rows x 64 columns (gate/up: 32 h columns, their gate and up
// columns side by side), on the double-buffered main loop of simt_gemm.cuh;
// the m-tile -> (expert, first row) map is derived on the device from the
// offsets (no host synchronisation).
#include "common.cuh"
#include "internal.h"
#include "simt_gemm.cuh"

namespace moe {

constexpr int kBM = 32, kBN = 64, kBK = 16;

// One BM-row tile of an expert's rows: gate/up (GATEUP: the tile's B columns
// are kBN/2 gate columns then the same kBN/2 up columns, so each thread holds
// g and u of the same h column) or down (kBN output columns, scaled by the
// row's routing weight).  grid (ceil(N / columns per tile), m-tile bound).
template <bool GATEUP>
__global__ void __launch_bounds__(simt::kThreads) ffn_simt_kernel(
    const float* __restrict__ A, const float* __restrict__ B0, const float* __restrict__ B1,
    float* __restrict__ out, const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm,
    const float* __restrict__ topk_w, int E, int Kd, int N, int64_t max_rows, int64_t nk,
    float* __restrict__ gu_keep, int* status)
{
    constexpr int NC = GATEUP ? kBN / 2 : kBN;  // output columns per tile
    constexpr int TM = kBM / 16, TN = kBN / 16;
    __shared__ int s_off[257];
    __shared__ int s_pref[257];
    __shared__ simt::Smem<kBM, kBN, kBK> sm;
    simt::row_tile_prefix<kBM>(offsets, E, max_rows, s_off, s_pref, status, 300);
    int e;
    int64_t row0, row_end;
    if (!simt::row_tile(s_off, s_pref, E, kBM, blockIdx.y, e, row0, row_end)) return;
    const int n0 = blockIdx.x * NC;

    struct LA {
        const float* p;
        int64_t r0, rend;
        int lda;
        MOE_DEVICE float ld(int m, int64_t k) const
        {
            const int64_t row = r0 + m;
            return row < rend ? p[row * lda + k] : 0.f;
        }
    } la{A, row0, row_end, Kd};
    struct LB {
        const float *g, *u;
        int n0, N;
        MOE_DEVICE float ld(int64_t k, int n) const
        {
            const bool up = GATEUP && n >= kBN / 2;
            const int col = n0 + (up ? n - kBN / 2 : n);
            return col < N ? (up ? u : g)[k * N + col] : 0.f;
        }
    } lb{B0 + (size_t)e * Kd * N, GATEUP ? B1 + (size_t)e * Kd * N : nullptr, n0, N};

    float acc[TM][TN];
    simt::mainloop<kBM, kBN, kBK, true, false>(acc, la, lb, 0, Kd, sm);

#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int64_t row = row0 + threadIdx.x / 16 + 16 * i;
        if (row >= row_end) continue;
        float wr = 1.f;
        if (!GATEUP && perm != nullptr) {  // no perm: unit weights (a shared expert, training)
            const int32_t pa = perm[row];
            if (pa < 0 || pa >= nk) {
                raise_flag(status, kFlagBounds, 301);
                wr = 0.f;
            } else {
                wr = topk_w[pa];
            }
        }
#pragma unroll
        for (int j = 0; j < (GATEUP ? TN / 2 : TN); ++j) {
            const int col = n0 + threadIdx.x % 16 + 16 * j;
            if (col >= N) continue;
            if (GATEUP) {
                const float g = acc[i][j], u = acc[i][j + TN / 2];
                out[row * N + col] = silu_f32(g) * u;
                if (gu_keep != nullptr) {  // [g | u] for the backward
                    gu_keep[row * 2 * N + col] = g;
                    gu_keep[row * 2 * N + N + col] = u;
                }
            } else {
                out[row * N + col] = wr * acc[i][j];
            }
        }
    }
}

static cudaError_t launch_simt(const moe_config& c, int64_t max_rows, const void* x_perm,
                               const int32_t* offsets, const int32_t* perm, const float* topk_w,
                               const void* w_gate, const void* w_up, const void* w_down, void* h,
                               void* y_perm, void* gu_keep, int* status, cudaStream_t s, StageHook mid,
                               void* mid_ctx)
{
    const int64_t mtiles = simt::mtiles_bound(max_rows, c.E, kBM);
    const int64_t nk = c.T * c.K;
    dim3 g1((c.F + kBN / 2 - 1) / (kBN / 2), (unsigned)mtiles);
    ffn_simt_kernel<true><<<g1, simt::kThreads, 0, s>>>(
        static_cast<const float*>(x_perm), static_cast<const float*>(w_gate), static_cast<const float*>(w_up),
        static_cast<float*>(h), offsets, perm, topk_w, c.E, c.D, c.F, max_rows, nk,
        static_cast<float*>(gu_keep), status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (mid) mid(mid_ctx, s);
    dim3 g2((c.D + kBN - 1) / kBN, (unsigned)mtiles);
    ffn_simt_kernel<false><<<g2, simt::kThreads, 0, s>>>(
        static_cast<const float*>(h), static_cast<const float*>(w_down), nullptr, static_cast<float*>(y_perm),
        offsets, perm, topk_w, c.E, c.F, c.D, max_rows, nk, nullptr, status);
    return cudaGetLastError();
}

cudaError_t launch_ffn_simt_f32(const moe_config& c, int64_t max_rows, const void* x_perm,
                                const int32_t* offsets, const int32_t* perm, const float* topk_w,
                                const void* w_gate, const void* w_up, const void* w_down, void* h,
                                void* y_perm, void* gu_keep, int* status, cudaStream_t s, StageHook mid,
                                void* mid_ctx)
{
    return launch_simt(c, max_rows, x_perm, offsets, perm, topk_w, w_gate, w_up, w_down, h, y_perm, gu_keep,
                       status, s, mid, mid_ctx);
}

}  // namespace moe
