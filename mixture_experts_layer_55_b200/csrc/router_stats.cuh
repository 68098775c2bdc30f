// router_stats.cuh -- the last step of the router statistics, run by the
// block of a router kernel that finishes last.
//
// "Lab: build a tiny MoE in PyTorch", section "Full implementation": the
// balance loss E * sum_e f_e P_e with f_e = count_e / (T K) and P_e the mean
// router probability of expert e, and the z-loss mean_t logsumexp_t^2; its
// stats also report the mean router entropy.  Each block of a router kernel
// leaves per-block partials (probability sums per expert, counts per expert,
// sums of lse^2 and of the entropy); the block that increments the counter
// last adds them up in a fixed order (so results are bitwise reproducible,
// whichever block is last), writes mean_prob and losses, and resets the
// counter to zero for the next launch.
#pragma once

#include "common.cuh"

namespace moe {

// Word of the workspace status region that counts finished router blocks.
constexpr int kRouterCounterWord = 16;

// Shared scratch of finish_router_stats: kStatD doubles, kStatC long longs.
constexpr int kStatD = 768;
constexpr int kStatC = 512;

// Called by all `nthreads` threads (tid = 0 .. nthreads-1) of the last block,
// after a block-wide barrier; `sync` is that block's barrier.  E <= 256.
template <typename Sync>
MOE_DEVICE void finish_router_stats(const float* blk_mp, const float* blk_z, const float* blk_ent,
                                    const int32_t* blk_cnt, int nb, int64_t T, int E, int K,
                                    float* mean_prob, float* losses, double* sd, long long* sc,
                                    int nthreads, int tid, Sync sync)
{
    const int ncol = E + 2;  // E probability sums (and counts), the z sum, the entropy sum
    int cc = nthreads / ncol;
    if (cc < 1) cc = 1;
    // chunk sums over a fixed range of blocks each: the loads of 16 blocks are
    // issued together (unconditionally, at clamped indices, so that none waits
    // for another), then the ones in range are added in block order
    for (int j = tid; j < ncol * cc; j += nthreads) {
        const int col = j % ncol, ch = j / ncol;
        const int b0 = (int)((int64_t)nb * ch / cc), b1 = (int)((int64_t)nb * (ch + 1) / cc);
        const float* src = col < E ? blk_mp + col : (col == E ? blk_z : blk_ent);
        const size_t stride = col < E ? (size_t)E : 1;
        const int32_t* csrc = blk_cnt + (col < E ? col : 0);
        const size_t cstride = (size_t)E;
        double a = 0.0;
        long long c = 0;
        for (int b = b0; b < b1; b += 16) {
            float v[16];
            int32_t n[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int bb = min(b + u, b1 - 1);
                v[u] = __ldcg(src + (size_t)bb * stride);
                n[u] = __ldcg(csrc + (size_t)bb * cstride);
            }
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (b + u < b1) {
                    a += (double)v[u];
                    c += col < E ? n[u] : 0;
                }
        }
        sd[j] = a;
        sc[j] = c;
    }
    sync();
    // each column: its chunks in order
    for (int col = tid; col < ncol; col += nthreads) {
        double a = 0.0;
        long long c = 0;
        for (int ch = 0; ch < cc; ++ch) {
            a += sd[ch * ncol + col];
            c += sc[ch * ncol + col];
        }
        sd[col] = a;
        sc[col] = c;
    }
    sync();
    // mean probabilities, and the balance-loss terms summed by a fixed tree
    double* term = sd + 512;
    for (int e = tid; e < 256; e += nthreads) {
        double v = 0.0;
        if (e < E) {
            const double mp = sd[e] / (double)T;
            if (mean_prob) mean_prob[e] = (float)mp;
            v = ((double)sc[e] / ((double)T * (double)K)) * mp;
        }
        term[e] = v;
    }
    sync();
    for (int off = 128; off > 0; off >>= 1) {
        for (int e = tid; e < off; e += nthreads) term[e] += term[e + off];
        sync();
    }
    if (tid == 0 && losses) {
        losses[0] = (float)(sd[E] / (double)T);
        losses[1] = (float)((double)E * term[0]);
        losses[2] = (float)(sd[E + 1] / (double)T);
    }
}

}  // namespace moe
