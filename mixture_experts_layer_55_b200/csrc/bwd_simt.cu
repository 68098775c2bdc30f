// bwd_simt.cu -- the backward's grouped GEMMs in true fp32 on the SIMT pipes
// (no TF32), for layers whose dtype is fp32.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation": the
// expert is down(silu(gate x) * up x), scaled by its combine weight.  With
// dYp = w * dY on every kept row (the rows kernel) and [g | u] kept by the
// training forward, the chain rule through that expression gives
//   dH  = dYp Wd_e^T                          (rows x F)
//   dg  = dH * u * silu'(g),  du = dH * silu(g),  silu'(g) = s + g s (1 - s)
//   dXp = dg Wg_e^T + du Wu_e^T               (rows x D)
//   dWd_e = h^T dYp,  dWg_e = x_perm^T dg,  dWu_e = x_perm^T du
// over each expert's contiguous row block.  The bf16 layer runs the same
// products on the tensor cores (ffn_tc.cu, wgrad_tc.cu); these kernels are
// the plain fp32 form on the double-buffered main loop of simt_gemm.cuh.
#include "common.cuh"
#include "internal.h"
#include "simt_gemm.cuh"

namespace moe {

namespace {

constexpr int kBM = 32, kBN = 64, kBK = 16;  // row-grouped products
constexpr int kWM = 64, kWN = 64;            // weight gradients

// sigmoid and its use in silu and silu' in fp32 (precise exponential and division)
MOE_DEVICE void silu_grad_f32(float g, float& silu, float& dsilu)
{
    const float s = 1.0f / (1.0f + expf(-g));
    silu = g * s;
    dsilu = fmaf(g * s, 1.0f - s, s);
}

enum { kDgradH = 0, kDgradX = 1 };

// Row-grouped products with a transposed weight operand:
//   kDgradH: dH[r, f] = sum_d dyp[r, d] * Wd_e[f, d], written as [dg | du]
//            (ld 2F) using the kept [g | u] (ld 2F);
//   kDgradX: dxp[r, d] = sum_{k < 2F} dgu[r, k] * W(k, d), W(k, d) = Wg_e[d, k]
//            for k < F and Wu_e[d, k - F] after.
// grid (ceil(N / kBN), m-tile bound); N = F for kDgradH, D for kDgradX.
template <int MODE>
__global__ void __launch_bounds__(simt::kThreads) dgrad_simt_kernel(
    const float* __restrict__ A, const float* __restrict__ W0, const float* __restrict__ W1,
    const float* __restrict__ gu, float* __restrict__ out, const int32_t* __restrict__ offsets, int E, int D,
    int F, int64_t max_rows, int* status)
{
    constexpr int TM = kBM / 16, TN = kBN / 16;
    __shared__ int s_off[257];
    __shared__ int s_pref[257];
    __shared__ simt::Smem<kBM, kBN, kBK> sm;
    simt::row_tile_prefix<kBM>(offsets, E, max_rows, s_off, s_pref, status, 800);
    int e;
    int64_t row0, row_end;
    if (!simt::row_tile(s_off, s_pref, E, kBM, blockIdx.y, e, row0, row_end)) return;
    const int n0 = blockIdx.x * kBN;
    const int Kd = MODE == kDgradH ? D : 2 * F;  // contraction length
    const int N = MODE == kDgradH ? F : D;

    struct LA {
        const float* p;
        int64_t r0, rend, lda;
        MOE_DEVICE float ld(int m, int64_t k) const
        {
            const int64_t row = r0 + m;
            return row < rend ? p[row * lda + k] : 0.f;
        }
    } la{A, row0, row_end, Kd};
    // weight rows: Wd_e is F x D, Wg_e and Wu_e are D x F (row n, column k)
    struct LB {
        const float *w0, *w1;
        int n0, N, F, ldw;
        MOE_DEVICE float ld(int64_t k, int n) const
        {
            const int col = n0 + n;
            if (col >= N) return 0.f;
            if (MODE == kDgradH) return w0[(size_t)col * ldw + k];
            return k < F ? w0[(size_t)col * ldw + k] : w1[(size_t)col * ldw + (k - F)];
        }
    } lb{W0 + (size_t)e * D * F, MODE == kDgradX ? W1 + (size_t)e * D * F : nullptr, n0, N, F,
         MODE == kDgradH ? D : F};

    float acc[TM][TN];
    simt::mainloop<kBM, kBN, kBK, true, true>(acc, la, lb, 0, Kd, sm);

#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int64_t row = row0 + threadIdx.x / 16 + 16 * i;
        if (row >= row_end) continue;
#pragma unroll
        for (int j = 0; j < TN; ++j) {
            const int col = n0 + threadIdx.x % 16 + 16 * j;
            if (col >= N) continue;
            if (MODE == kDgradH) {
                const float g = gu[row * 2 * (int64_t)F + col], u = gu[row * 2 * (int64_t)F + F + col];
                float silu, dsilu;
                silu_grad_f32(g, silu, dsilu);
                out[row * 2 * (int64_t)F + col] = acc[i][j] * u * dsilu;
                out[row * 2 * (int64_t)F + F + col] = acc[i][j] * silu;
            } else {
                out[row * (int64_t)N + col] = acc[i][j];
            }
        }
    }
}

// Weight gradients: for expert e = blockIdx.z / halves and half q = blockIdx.z
// % halves, dW_q[e][m, n] = sum over the expert's rows r of A[r, m] * B[r, q*N + n]
// (A rows of lda elements, B rows of ldb), an M x N fp32 matrix per expert.
// An expert without rows gets zeros.  grid (ceil(N / kWN), ceil(M / kWM), E * halves).
__global__ void __launch_bounds__(simt::kThreads) wgrad_simt_kernel(
    const float* __restrict__ A, int64_t lda, const float* __restrict__ Bm, int64_t ldb,
    float* __restrict__ out0, float* __restrict__ out1, const int32_t* __restrict__ offsets, int E, int M,
    int N, int halves, int64_t max_rows, int* status)
{
    constexpr int TM = kWM / 16, TN = kWN / 16;
    __shared__ simt::Smem<kWM, kWN, kBK> sm;
    const int e = blockIdx.z / halves, q = blockIdx.z % halves;
    int64_t r0 = offsets[e], r1 = offsets[e + 1];
    if (r0 < 0 || r1 < r0 || r1 > max_rows) {
        if (threadIdx.x == 0) raise_flag(status, kFlagBounds, 810);
        r0 = r1 = 0;
    }
    const int m0 = blockIdx.y * kWM, n0 = blockIdx.x * kWN;
    struct LA {  // A(m, k = row): m contiguous
        const float* p;
        int64_t lda;
        int m0, M;
        MOE_DEVICE float ld(int m, int64_t k) const { return m0 + m < M ? p[k * lda + m0 + m] : 0.f; }
    } la{A, lda, m0, M};
    struct LB {  // B(k = row, n): n contiguous
        const float* p;
        int64_t ldb;
        int n0, N;
        MOE_DEVICE float ld(int64_t k, int n) const { return n0 + n < N ? p[k * ldb + n0 + n] : 0.f; }
    } lb{Bm + (int64_t)q * N, ldb, n0, N};

    float acc[TM][TN];
    simt::mainloop<kWM, kWN, kBK, false, false>(acc, la, lb, r0, r1, sm);

    float* out = (q == 0 ? out0 : out1) + (size_t)e * M * N;
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int m = m0 + threadIdx.x / 16 + 16 * i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < TN; ++j) {
            const int n = n0 + threadIdx.x % 16 + 16 * j;
            if (n < N) out[(size_t)m * N + n] = acc[i][j];
        }
    }
}

}  // namespace

cudaError_t launch_dgrad_simt_f32(const moe_config& c, int64_t max_rows, const void* dyp, const int32_t* offsets,
                                  const void* gu, const void* w_gate, const void* w_up, const void* w_down,
                                  void* dgu, void* dxp, int* status, cudaStream_t s, StageHook mid, void* mid_ctx)
{
    const unsigned mtiles = (unsigned)simt::mtiles_bound(max_rows, c.E, kBM);
    dim3 g1((c.F + kBN - 1) / kBN, mtiles);
    dgrad_simt_kernel<kDgradH><<<g1, simt::kThreads, 0, s>>>(
        static_cast<const float*>(dyp), static_cast<const float*>(w_down), nullptr, static_cast<const float*>(gu),
        static_cast<float*>(dgu), offsets, c.E, c.D, c.F, max_rows, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (mid) mid(mid_ctx, s);
    dim3 g2((c.D + kBN - 1) / kBN, mtiles);
    dgrad_simt_kernel<kDgradX><<<g2, simt::kThreads, 0, s>>>(
        static_cast<const float*>(dgu), static_cast<const float*>(w_gate), static_cast<const float*>(w_up), nullptr,
        static_cast<float*>(dxp), offsets, c.E, c.D, c.F, max_rows, status);
    return cudaGetLastError();
}

cudaError_t launch_wgrad_simt_f32(int E, int64_t max_rows, const int32_t* offsets, const void* a, int M,
                                  const void* b, int N, int halves, float* out0, float* out1, int* status,
                                  cudaStream_t s)
{
    if (halves < 1 || halves > 2 || M < 1 || N < 1) return cudaErrorInvalidValue;
    dim3 g((N + kWN - 1) / kWN, (M + kWM - 1) / kWM, (unsigned)(E * halves));
    wgrad_simt_kernel<<<g, simt::kThreads, 0, s>>>(static_cast<const float*>(a), M, static_cast<const float*>(b),
                                        (int64_t)N * halves, out0, out1, offsets, E, M, N, halves, max_rows,
                                        status);
    return cudaGetLastError();
}

}  // namespace moe
