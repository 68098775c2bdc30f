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
// the plain fp32 form, 64 x 64 output tiles of 4 x 4 per thread.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16;

// s_pref[e] = number of kBM-row tiles of experts < e; s_pref[E] = total.
MOE_DEVICE void row_tile_prefix(const int32_t* offsets, int E, int64_t max_rows, int* s_off, int* s_pref,
                                int* status)
{
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0, prev = 0;
        for (int e = 0; e < E; ++e) {
            int a = s_off[e], b = s_off[e + 1];
            if (a < prev || b < a || b > max_rows) {  // malformed offsets: treat as empty
                raise_flag(status, kFlagBounds, 800);
                b = a = prev;
            }
            s_off[e] = a;
            s_off[e + 1] = b;
            prev = b;
            s_pref[e] = run;
            run += (b - a + kBM - 1) / kBM;
        }
        s_pref[E] = run;
    }
    __syncthreads();
}

// sigmoid and its use in silu and silu' in fp32 (precise exponential and division)
MOE_DEVICE void silu_grad_f32(float g, float& silu, float& dsilu)
{
    const float s = 1.0f / (1.0f + expf(-g));
    silu = g * s;
    dsilu = fmaf(g * s, 1.0f - s, s);
}

enum { kDgradH = 0, kDgradX = 1 };

// Row-grouped products with a transposed weight operand:
//   kDgradH: out[r, f] from dH[r, f] = sum_d dyp[r, d] * Wd_e[f, d], written as
//            [dg | du] (ld 2F) using gu (ld 2F);
//   kDgradX: dxp[r, d] = sum_{k < 2F} dgu[r, k] * W(k, d), W(k, d) = Wg_e[d, k]
//            for k < F and Wu_e[d, k - F] after.
// grid (ceil(N / 64), m-tile bound); N = F for kDgradH, D for kDgradX.
template <int MODE>
__global__ void __launch_bounds__(256) dgrad_simt_kernel(const float* __restrict__ A, const float* __restrict__ W0,
                                                         const float* __restrict__ W1, const float* __restrict__ gu,
                                                         float* __restrict__ out, const int32_t* __restrict__ offsets,
                                                         int E, int D, int F, int64_t max_rows, int* status)
{
    __shared__ int s_off[257];
    __shared__ int s_pref[257];
    __shared__ float As[kBK][kBM + 4];
    __shared__ float Bs[kBK][kBN + 1];

    row_tile_prefix(offsets, E, max_rows, s_off, s_pref, status);
    const int mt = blockIdx.y;
    if (mt >= s_pref[E]) return;
    int e = 0;
    while (e + 1 < E && s_pref[e + 1] <= mt) ++e;  // experts with no tiles are skipped
    const int64_t row0 = (int64_t)s_off[e] + (int64_t)(mt - s_pref[e]) * kBM;
    const int64_t row_end = s_off[e + 1];
    const int n0 = blockIdx.x * kBN;
    const int Kd = MODE == kDgradH ? D : 2 * F;  // contraction length
    const int N = MODE == kDgradH ? F : D;
    const int64_t lda = MODE == kDgradH ? D : 2 * (int64_t)F;
    // weight rows: Wd_e is F x D (row n, column k); Wg_e, Wu_e are D x F (row n, column k)
    const float* Wa = W0 + (size_t)e * D * F;
    const float* Wb = MODE == kDgradX ? W1 + (size_t)e * D * F : nullptr;
    const int ldw = MODE == kDgradH ? D : F;

    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;  // 4 x 4 outputs: rows ty + 16 i, columns tx + 16 j
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < Kd; k0 += kBK) {
        for (int idx = tid; idx < kBM * kBK; idx += 256) {  // consecutive threads: consecutive k
            const int r = idx / kBK, kk = idx % kBK;
            const int64_t row = row0 + r;
            const int k = k0 + kk;
            As[kk][r] = (row < row_end && k < Kd) ? A[row * lda + k] : 0.f;
        }
        for (int idx = tid; idx < kBN * kBK; idx += 256) {
            const int c = idx / kBK, kk = idx % kBK;
            const int n = n0 + c, k = k0 + kk;
            float v = 0.f;
            if (n < N && k < Kd) {
                if (MODE == kDgradH) v = Wa[(size_t)n * ldw + k];
                else v = k < F ? Wa[(size_t)n * ldw + k] : Wb[(size_t)n * ldw + (k - F)];
            }
            Bs[kk][c] = v;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kBK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t row = row0 + ty + 16 * i;
        if (row >= row_end) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int col = n0 + tx + 16 * j;
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
// An expert without rows gets zeros.  grid (ceil(N / 64), ceil(M / 64), E * halves).
__global__ void __launch_bounds__(256) wgrad_simt_kernel(const float* __restrict__ A, int64_t lda,
                                                         const float* __restrict__ Bm, int64_t ldb,
                                                         float* __restrict__ out0, float* __restrict__ out1,
                                                         const int32_t* __restrict__ offsets, int E, int M,
                                                         int N, int halves, int64_t max_rows, int* status)
{
    __shared__ float As[kBK][kBM];
    __shared__ float Bs[kBK][kBN];
    const int e = blockIdx.z / halves, q = blockIdx.z % halves;
    int64_t r0 = offsets[e], r1 = offsets[e + 1];
    if (r0 < 0 || r1 < r0 || r1 > max_rows) {
        if (threadIdx.x == 0) raise_flag(status, kFlagBounds, 810);
        r0 = r1 = 0;
    }
    const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
    const float* Bq = Bm + (int64_t)q * N;
    float* out = (q == 0 ? out0 : out1) + (size_t)e * M * N;
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int64_t k0 = r0; k0 < r1; k0 += kBK) {
        for (int idx = tid; idx < kBK * kBM; idx += 256) {  // consecutive threads: consecutive m
            const int kk = idx / kBM, c = idx % kBM;
            const int64_t r = k0 + kk;
            As[kk][c] = (r < r1 && m0 + c < M) ? A[r * lda + m0 + c] : 0.f;
            Bs[kk][c] = (r < r1 && n0 + c < N) ? Bq[r * ldb + n0 + c] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kBK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty + 16 * i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx + 16 * j;
            if (n < N) out[(size_t)m * N + n] = acc[i][j];
        }
    }
}

}  // namespace

cudaError_t launch_dgrad_simt_f32(const moe_config& c, int64_t max_rows, const void* dyp, const int32_t* offsets,
                                  const void* gu, const void* w_gate, const void* w_up, const void* w_down,
                                  void* dgu, void* dxp, int* status, cudaStream_t s, StageHook mid, void* mid_ctx)
{
    const unsigned mtiles = (unsigned)((max_rows + kBM - 1) / kBM + c.E);
    dim3 g1((c.F + kBN - 1) / kBN, mtiles);
    dgrad_simt_kernel<kDgradH><<<g1, 256, 0, s>>>(static_cast<const float*>(dyp), static_cast<const float*>(w_down),
                                                  nullptr, static_cast<const float*>(gu), static_cast<float*>(dgu),
                                                  offsets, c.E, c.D, c.F, max_rows, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (mid) mid(mid_ctx, s);
    dim3 g2((c.D + kBN - 1) / kBN, mtiles);
    dgrad_simt_kernel<kDgradX><<<g2, 256, 0, s>>>(static_cast<const float*>(dgu), static_cast<const float*>(w_gate),
                                                  static_cast<const float*>(w_up), nullptr, static_cast<float*>(dxp),
                                                  offsets, c.E, c.D, c.F, max_rows, status);
    return cudaGetLastError();
}

cudaError_t launch_wgrad_simt_f32(int E, int64_t max_rows, const int32_t* offsets, const void* a, int M,
                                  const void* b, int N, int halves, float* out0, float* out1, int* status,
                                  cudaStream_t s)
{
    if (halves < 1 || halves > 2 || M < 1 || N < 1) return cudaErrorInvalidValue;
    dim3 g((N + kBN - 1) / kBN, (M + kBM - 1) / kBM, (unsigned)(E * halves));
    wgrad_simt_kernel<<<g, 256, 0, s>>>(static_cast<const float*>(a), M, static_cast<const float*>(b),
                                        (int64_t)N * halves, out0, out1, offsets, E, M, N, halves, max_rows,
                                        status);
    return cudaGetLastError();
}

}  // namespace moe
