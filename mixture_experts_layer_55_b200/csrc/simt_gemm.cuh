// simt_gemm.cuh -- the main loop of the fp32 (true fp32 FMA, no TF32) tiled
// GEMMs of fp32 layers: acc[BM x BN] += A(m, k) * B(k, n) over one K range.
//
// 256 threads as a 16 x 16 grid, each owning (BM/16) x (BN/16) outputs (rows
// ty + 16 i, columns tx + 16 j: conflict-free shared-memory reads).  Tiles of
// BK along K are double-buffered in shared memory through registers: the
// next tile's global loads are issued before the current tile's FMAs, so
// their latency overlaps the arithmetic, with one barrier per tile.
//
// Operands are read through accessors: a.ld(m, k) / b.ld(k, n) return the
// element or 0 outside the problem.  A_KFAST / B_KFAST say which index is
// contiguous in memory, so consecutive threads load consecutive addresses.
#pragma once
#include "common.cuh"

namespace moe {
namespace simt {

constexpr int kThreads = 256;

template <int BM, int BN, int BK>
struct Smem {
    float a[2][BK][BM + 4];
    float b[2][BK][BN + 4];
};

template <int BM, int BN, int BK, bool A_KFAST, bool B_KFAST, class LA, class LB>
MOE_DEVICE void mainloop(float (&acc)[BM / 16][BN / 16], const LA& la, const LB& lb, int64_t k_begin,
                         int64_t k_end, Smem<BM, BN, BK>& sm)
{
    constexpr int TM = BM / 16, TN = BN / 16;
    constexpr int NA = BM * BK / kThreads, NB = BK * BN / kThreads;  // elements per thread
    static_assert(NA >= 1 && NB >= 1 && BM * BK % kThreads == 0 && BK * BN % kThreads == 0, "tile");
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
    if (k_end <= k_begin) return;

    float ra[NA], rb[NB];
    auto load = [&](int64_t k0) {
#pragma unroll
        for (int q = 0; q < NA; ++q) {
            const int idx = tid + q * kThreads;
            const int m = A_KFAST ? idx / BK : idx % BM, kk = A_KFAST ? idx % BK : idx / BM;
            const int64_t k = k0 + kk;
            ra[q] = k < k_end ? la.ld(m, k) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            const int idx = tid + q * kThreads;
            const int n = B_KFAST ? idx / BK : idx % BN, kk = B_KFAST ? idx % BK : idx / BN;
            const int64_t k = k0 + kk;
            rb[q] = k < k_end ? lb.ld(k, n) : 0.f;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int q = 0; q < NA; ++q) {
            const int idx = tid + q * kThreads;
            const int m = A_KFAST ? idx / BK : idx % BM, kk = A_KFAST ? idx % BK : idx / BM;
            sm.a[buf][kk][m] = ra[q];
        }
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            const int idx = tid + q * kThreads;
            const int n = B_KFAST ? idx / BK : idx % BN, kk = B_KFAST ? idx % BK : idx / BN;
            sm.b[buf][kk][n] = rb[q];
        }
    };

    load(k_begin);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int64_t k0 = k_begin; k0 < k_end; k0 += BK) {
        const bool more = k0 + BK < k_end;
        if (more) load(k0 + BK);  // in flight during the FMAs below
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[TM], b[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) a[i] = sm.a[buf][kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < TN; ++j) b[j] = sm.b[buf][kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (more) store(buf ^ 1);  // that buffer's last reads finished before the last barrier
        __syncthreads();
        buf ^= 1;
    }
}

// m-tile prefix of a row-grouped problem: s_pref[e] = number of BM-row tiles of
// experts < e, s_pref[E] = total; malformed offsets become empty experts and
// raise the bounds flag.  Whole block; s_off / s_pref hold E + 1 entries.
template <int BM>
MOE_DEVICE void row_tile_prefix(const int32_t* offsets, int E, int64_t max_rows, int* s_off, int* s_pref,
                                int* status, int where)
{
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0, prev = 0;
        for (int e = 0; e < E; ++e) {
            int a = s_off[e], b = s_off[e + 1];
            if (a < prev || b < a || b > max_rows) {
                raise_flag(status, kFlagBounds, where);
                b = a = prev;
            }
            s_off[e] = a;
            s_off[e + 1] = b;
            prev = b;
            s_pref[e] = run;
            run += (b - a + BM - 1) / BM;
        }
        s_pref[E] = run;
    }
    __syncthreads();
}

// Expert and first row of m-tile mt, or false when mt is past the last tile.
MOE_DEVICE bool row_tile(const int* s_off, const int* s_pref, int E, int BM, int mt, int& e, int64_t& row0,
                         int64_t& row_end)
{
    if (mt >= s_pref[E]) return false;
    e = 0;
    while (e + 1 < E && s_pref[e + 1] <= mt) ++e;  // experts with no tiles are skipped
    row0 = (int64_t)s_off[e] + (int64_t)(mt - s_pref[e]) * BM;
    row_end = s_off[e + 1];
    return true;
}

// Upper bound of the m-tiles of a row-grouped problem: sum_e ceil(rows_e / BM)
// <= max_rows / BM + E.
inline int64_t mtiles_bound(int64_t max_rows, int E, int BM) { return (max_rows + BM - 1) / BM + E; }

}  // namespace simt
}  // namespace moe
