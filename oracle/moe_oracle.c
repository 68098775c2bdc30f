/*
 * moe_oracle.c -- plain CPU fp64 oracle of the token-choice top-k
 * Mixture-of-Experts layer: forward, and the backward of its training loss.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker that the CUDA library is
 * compared against.  It shares no code, header, table or helper with the CUDA
 * path and must never be linked into it.  Only the tests, the smoke check and
 * the CPU-baseline leg of the benchmark load it.
 *
 * Every step is written as plain nested loops in double precision, in the order
 * the sources give it; OpenMP only splits independent tokens (or rows) across
 * threads and never changes the order of any sum.
 *
 * Sources (web pages; cited by page title and section):
 *   [TinyMoE]  "Lab: build a tiny MoE in PyTorch" (open-llm-engineering),
 *              sections "Full implementation", "Add a capacity limit",
 *              "Trace one token by hand", "Required correctness tests".
 *   [LLMBook]  "2.9 Mixture-of-Experts (MoE) Architectures" (llm-stack-book),
 *              sections "The Router: Gating, Top-k, and the Softmax-Then-Select
 *              Question", "A Toy MoE Layer From Scratch", "The auxiliary
 *              load-balancing loss", "Capacity Factor, Token Dropping, and the
 *              Worked Numbers".
 *   Backward:  [TinyMoE] "Smoke test and backward pass" (the training loss is
 *              main + c_bal * balance + c_z * z, differentiated by autograd) and
 *              [LLMBook] "The Router" (the top-k index decision is a stop-
 *              gradient; gradient reaches the router only through the kept gate
 *              weights and the auxiliary losses; an expert that was not chosen
 *              gets none from that token).
 *
 * Element types of inputs: 0 = IEEE fp32, 1 = bf16 given as raw 16-bit words.
 * Both convert exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1

static double elem(const void *p, int32_t dtype, int64_t i)
{
    if (dtype == ORC_F32)
        return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Router logits, [TinyMoE] "Full implementation" (router = bias-free linear
 * layer evaluated in fp32; here in fp64) and [LLMBook] "The Router" (one
 * logit per expert from a single linear map):
 *     L[t,e] = sum_d x[t,d] * W_r[d,e]  (+ bias[e])  (+ noise[t,e])
 * W_r is (D, E) row-major.  bias (E) and noise (T, E) may be NULL.  The bias
 * is a plain linear bias; the noise is noisy top-k gating's additive logit
 * noise ([LLMBook] "Noisy / top-k gating"), drawn by the caller.
 */
void oracle_router_logits(int64_t T, int32_t D, int32_t E, const void *x, int32_t x_dtype,
                          const float *w_r, const float *bias, const float *noise,
                          double *logits)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int32_t d = 0; d < D; ++d)
                acc += elem(x, x_dtype, t * D + d) * (double)w_r[(int64_t)d * E + e];
            if (bias)
                acc += (double)bias[e];
            if (noise)
                acc += (double)noise[t * E + e];
            logits[t * E + e] = acc;
        }
    }
}

/*
 * Routing of one token from its logits.  Sources: [TinyMoE] "Full
 * implementation" (softmax, top-k, weights divided by the sum of the
 * selected); [LLMBook] "The Router" (softmax-then-top-k keeps the selected
 * probabilities as they are, without renormalisation) and "Exercises" 6
 * (DeepSeek-V3 selection-only bias: top-k on h + b, gate weights from the
 * unbiased logits over the chosen set); [TinyMoE] "Lab extensions" (sigmoid
 * top-k, group-limited routing).
 *
 *   scores      softmax: p_e = exp(L_e - m) / sum_e' exp(L_e' - m)
 *               sigmoid: s_e = 1 / (1 + exp(-L_e))
 *   selection   u_e = L_e + sel_bias[e] (sel_bias may be NULL: u = L).
 *               With n_groups > 1 the experts form n_groups contiguous
 *               groups; a group's score is the largest u in it; the
 *               topk_groups groups of largest score (ties: lower group id)
 *               stay eligible, the others are excluded.  Then the K eligible
 *               experts ordered by (u desc, id asc) fill slots 0..K-1.
 *   weights     w_k = score[id_k] / sum_j score[id_j] when renormalize, else
 *               score[id_k]; then times route_scale.
 *   norm_scores (T, E): the scores normalised per token to sum to one (the
 *               softmax probabilities themselves; sigmoid scores / their sum);
 *               they feed the mean probability of the balance loss.
 *   lse         m + log sum_e exp(L_e - m)            (the z-loss term)
 *   entropy     -sum_e p_e log max(p_e, 1e-9) of the softmax probabilities
 *
 * norm_scores and entropy may be NULL.  Returns 0, or -1 if a logit is not
 * finite.
 */
int32_t oracle_route(int64_t T, int32_t E, int32_t K, const double *logits, int32_t score_func,
                     int32_t renormalize, const double *sel_bias, int32_t n_groups,
                     int32_t topk_groups, double route_scale, int32_t *ids, double *weights,
                     double *norm_scores, double *lse, double *entropy)
{
    int32_t bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t t = 0; t < T; ++t) {
        const double *L = logits + t * E;
        double *score = (double *)malloc(sizeof(double) * (size_t)E);
        double *u = (double *)malloc(sizeof(double) * (size_t)E);
        unsigned char *eligible = (unsigned char *)malloc((size_t)E);
        double m = L[0];
        for (int32_t e = 0; e < E; ++e) {
            if (!isfinite(L[e]))
                bad = 1;
            if (L[e] > m)
                m = L[e];
        }
        double s = 0.0;
        for (int32_t e = 0; e < E; ++e)
            s += exp(L[e] - m);
        if (lse)
            lse[t] = m + log(s);
        if (entropy) {
            double h = 0.0;
            for (int32_t e = 0; e < E; ++e) {
                double p = exp(L[e] - m) / s;
                h -= p * log(p > 1e-9 ? p : 1e-9);
            }
            entropy[t] = h;
        }
        for (int32_t e = 0; e < E; ++e) {
            score[e] = score_func == 1 ? 1.0 / (1.0 + exp(-L[e])) : exp(L[e] - m) / s;
            u[e] = L[e] + (sel_bias ? sel_bias[e] : 0.0);
            eligible[e] = 1;
        }
        if (norm_scores) {
            double ss = 0.0;
            for (int32_t e = 0; e < E; ++e)
                ss += score[e];
            for (int32_t e = 0; e < E; ++e)
                norm_scores[t * E + e] = score[e] / ss;
        }
        if (n_groups > 1) {
            int32_t gsize = E / n_groups;
            unsigned char *keep = (unsigned char *)calloc((size_t)n_groups, 1);
            for (int32_t r = 0; r < topk_groups; ++r) {
                int32_t best = -1;
                double bestv = 0.0;
                for (int32_t g = 0; g < n_groups; ++g) {
                    if (keep[g])
                        continue;
                    double gm = u[g * gsize];
                    for (int32_t e = g * gsize; e < (g + 1) * gsize; ++e)
                        if (u[e] > gm)
                            gm = u[e];
                    if (best < 0 || gm > bestv) { /* strict: lower group id on ties */
                        best = g;
                        bestv = gm;
                    }
                }
                keep[best] = 1;
            }
            for (int32_t e = 0; e < E; ++e)
                eligible[e] = keep[e / gsize];
            free(keep);
        }
        /* K passes, each picking the best eligible expert not yet taken. */
        for (int32_t k = 0; k < K; ++k) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (!eligible[e])
                    continue;
                int32_t taken = 0;
                for (int32_t j = 0; j < k; ++j)
                    if (ids[t * K + j] == e)
                        taken = 1;
                if (taken)
                    continue;
                if (best < 0 || u[e] > u[best])
                    best = e; /* strict '>' keeps the lower id on ties */
            }
            ids[t * K + k] = best;
        }
        double sel = 0.0;
        for (int32_t k = 0; k < K; ++k)
            sel += score[ids[t * K + k]];
        for (int32_t k = 0; k < K; ++k) {
            double w = score[ids[t * K + k]];
            if (renormalize)
                w = w / sel;
            weights[t * K + k] = w * route_scale;
        }
        free(score);
        free(u);
        free(eligible);
    }
    return bad ? -1 : 0;
}

/*
 * DeepSeek-V3 auxiliary-loss-free balancing, [LLMBook] "Exercises" 6
 * (update_bias): b_e += gamma * sign(mean_e'(counts) - counts_e): overloaded
 * experts get their selection bias lowered, underloaded ones raised, experts
 * exactly at the mean keep theirs.
 */
void oracle_update_bias(int32_t E, const int64_t *counts, double gamma, double *bias)
{
    double mean = 0.0;
    for (int32_t e = 0; e < E; ++e)
        mean += (double)counts[e];
    mean /= (double)E;
    for (int32_t e = 0; e < E; ++e) {
        double d = mean - (double)counts[e];
        double sg = d > 0.0 ? 1.0 : (d < 0.0 ? -1.0 : 0.0);
        bias[e] += gamma * sg;
    }
}

/*
 * Router statistics, [TinyMoE] "Full implementation" (Switch-style top-k
 * balance loss and ST-MoE z-loss) and [LLMBook] "The auxiliary load-balancing
 * loss":
 *     counts_e = #{(t,k) : ids[t,k] = e}          (before any capacity drop)
 *     f_e      = counts_e / (T*K)
 *     P_e      = (1/T) sum_t p[t,e]   (p: the per-token normalised scores)
 *     balance  = E * sum_e f_e * P_e
 *     z        = (1/T) sum_t lse_t^2
 * The raw, unweighted values (the loss coefficients are the caller's).
 */
void oracle_router_stats(int64_t T, int32_t E, int32_t K, const int32_t *ids, const double *probs,
                         const double *lse, int64_t *counts, double *mean_prob, double *z_loss,
                         double *balance_loss)
{
    for (int32_t e = 0; e < E; ++e) {
        counts[e] = 0;
        mean_prob[e] = 0.0;
    }
    for (int64_t i = 0; i < T * K; ++i)
        counts[ids[i]] += 1;
    for (int32_t e = 0; e < E; ++e) {
        double s = 0.0;
        for (int64_t t = 0; t < T; ++t)
            s += probs[t * E + e];
        mean_prob[e] = s / (double)T;
    }
    double bal = 0.0;
    for (int32_t e = 0; e < E; ++e)
        bal += ((double)counts[e] / (double)(T * K)) * mean_prob[e];
    *balance_loss = (double)E * bal;
    double z = 0.0;
    for (int64_t t = 0; t < T; ++t)
        z += lse[t] * lse[t];
    *z_loss = z / (double)T;
}

/*
 * Expert capacity, [TinyMoE] "Add a capacity limit" and [LLMBook] "A Toy MoE
 * Layer From Scratch": C = max(1, ceil(cf * T * K / E)), evaluated in double.
 * cf <= 0 means dropless; then C = T*K, which no expert can exceed.
 */
int64_t oracle_capacity(int64_t T, int32_t K, int32_t E, double cf)
{
    if (!(cf > 0.0))
        return T * (int64_t)K;
    double c = ceil(cf * (double)T * (double)K / (double)E);
    if (c < 1.0)
        c = 1.0;
    return (int64_t)c;
}

/*
 * Dispatch layout, [TinyMoE] "Add a capacity limit" (first-come keep mask:
 * walk tokens in order and their slots in order; an assignment is kept while
 * its expert has used fewer than C places) and "From local loop to expert
 * parallelism" (group rows by expert).
 *
 *   counts[e]  assignments that chose e (before drops)
 *   kept[e]    assignments of e that were kept
 *   offsets    exclusive prefix sum of kept, E+1 entries
 *   perm[row]  = t*K + k for the assignment stored at that row; the rows of
 *              expert e are offsets[e] .. offsets[e+1]-1 and hold its kept
 *              assignments in increasing token order
 *   row_of[t*K+k] = its row, or -1 when the assignment was dropped
 */
void oracle_dispatch(int64_t T, int32_t K, int32_t E, const int32_t *ids, int64_t C,
                     int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *perm,
                     int32_t *row_of)
{
    int64_t *used = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    unsigned char *keep = (unsigned char *)calloc((size_t)(T * K), 1);
    for (int32_t e = 0; e < E; ++e) {
        counts[e] = 0;
        kept[e] = 0;
    }
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int32_t e = ids[t * K + k];
            counts[e] += 1;
            if (used[e] < C) {
                keep[t * K + k] = 1;
                used[e] += 1;
            }
        }
    }
    for (int32_t e = 0; e < E; ++e)
        kept[e] = (int32_t)used[e];
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + kept[e];
    int64_t *cursor = used; /* reuse: next free row of each expert */
    for (int32_t e = 0; e < E; ++e)
        cursor[e] = offsets[e];
    for (int64_t i = 0; i < T * K; ++i) {
        if (keep[i]) {
            int32_t e = ids[i];
            int64_t row = cursor[e]++;
            perm[row] = (int32_t)i;
            row_of[i] = (int32_t)row;
        } else {
            row_of[i] = -1;
        }
    }
    free(keep);
    free(used);
}

/*
 * Gather each expert's token rows, [TinyMoE] "Full implementation"
 * (flat[token_index]): x_perm[row, :] = x[perm[row] / K, :].
 */
void oracle_gather(int64_t R, int32_t D, int32_t K, const void *x, int32_t x_dtype,
                   const int32_t *perm, double *x_perm)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        int64_t t = perm[r] / K;
        for (int32_t d = 0; d < D; ++d)
            x_perm[r * D + d] = elem(x, x_dtype, t * D + d);
    }
}

/*
 * One SwiGLU expert on a block of rows, [TinyMoE] "Full implementation"
 * (SwiGLUExpert: down(silu(gate(x)) * up(x)), no biases):
 *     g_f = sum_d x_d Wg[d,f],  u_f = sum_d x_d Wu[d,f]
 *     h_f = g_f / (1 + exp(-g_f)) * u_f
 *     o_j = sum_f h_f Wd[f,j]
 * wg, wu point at this expert's (D, F) matrices, wd at its (F, D) matrix, all
 * row-major, element type w_dtype.  rows_in (n, D), rows_out (n, D).
 */
void oracle_expert_rows(int64_t n, int32_t D, int32_t F, const double *rows_in, const void *wg,
                        const void *wu, const void *wd, int32_t w_dtype, double *rows_out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
        double *g = (double *)malloc(sizeof(double) * (size_t)F);
        double *u = (double *)malloc(sizeof(double) * (size_t)F);
        const double *xr = rows_in + r * D;
        for (int32_t f = 0; f < F; ++f) {
            g[f] = 0.0;
            u[f] = 0.0;
        }
        for (int32_t d = 0; d < D; ++d) {
            double xd = xr[d];
            for (int32_t f = 0; f < F; ++f) {
                g[f] += xd * elem(wg, w_dtype, (int64_t)d * F + f);
                u[f] += xd * elem(wu, w_dtype, (int64_t)d * F + f);
            }
        }
        for (int32_t f = 0; f < F; ++f)
            g[f] = g[f] / (1.0 + exp(-g[f])) * u[f]; /* h_f */
        double *o = rows_out + r * D;
        for (int32_t j = 0; j < D; ++j)
            o[j] = 0.0;
        for (int32_t f = 0; f < F; ++f) {
            double hf = g[f];
            for (int32_t j = 0; j < D; ++j)
                o[j] += hf * elem(wd, w_dtype, (int64_t)f * D + j);
        }
        free(g);
        free(u);
    }
}

/*
 * Weighted combine back to token order, [TinyMoE] "Full implementation"
 * (index_add_ of weight * expert output) and "Add a capacity limit" (a dropped
 * assignment adds nothing; an all-dropped token gets zero):
 *     y[t, :] = sum over kept slots k, in slot order, of w[t,k] * o[row_of[t*K+k], :]
 * o holds the unweighted expert outputs in row order (R, D).
 */
void oracle_combine(int64_t T, int32_t K, int32_t D, const double *o, const int32_t *row_of,
                    const double *weights, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double *yt = y + t * D;
        for (int32_t j = 0; j < D; ++j)
            yt[j] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            int32_t row = row_of[t * K + k];
            if (row < 0)
                continue;
            double w = weights[t * K + k];
            for (int32_t j = 0; j < D; ++j)
                yt[j] += w * o[(int64_t)row * D + j];
        }
    }
}

/* ------------------------------------------------------------------ backward
 *
 * The gradient of  loss = sum_t <dY_t, y_t> + c_bal * balance + c_z * z,
 * i.e. the backward of the forward above for an upstream gradient dY of y and
 * the loss coefficients c_bal, c_z ([TinyMoE] "Smoke test and backward pass":
 * loss = main + 0.01 * balance + 0.001 * z).  Stop-gradients, as autograd
 * applies them to the forward: the chosen ids (top-k, the group limit, the
 * selection bias) and the counts f_e of the balance loss (an integer count)
 * carry no gradient; the capacity keep mask is a function of the ids only.
 * Everything else -- the gate weights, the normalised scores of the balance
 * loss, the logsumexp of the z-loss, the router's linear map and the experts --
 * is differentiated by the chain rule, written out below step by step.
 */

/*
 * Gradient of the router logits for each token, from the gradients of its K
 * gate weights (dw, T x K; a dropped slot never reached y, so its dw is 0),
 * and of the two auxiliary losses.  With S the chosen scores' sum and
 * rs = route_scale:
 *   gate weights   w_k = rs * score[id_k] / S   (renormalize) or rs * score[id_k]
 *                  d score[id_j] += rs/S * (dw_j - sum_k dw_k * score[id_k] / S)
 *                             or += rs * dw_j
 *   balance        balance = E * sum_e f_e * P_e,  P_e = (1/T) sum_t n[t,e], where
 *                  n = score / sum_e score (softmax: n = p), f_e = counts_e/(T*K):
 *                  d n[t,e] = c_bal * E * f_e / T;  for sigmoid scores
 *                  d score_j += (d n_j - sum_e d n_e * n_e) / sum_e score_e
 *   scores         softmax: dL_j = p_j * (d p_j - sum_i p_i * d p_i)
 *                  sigmoid: dL_j = d s_j * s_j * (1 - s_j)
 *   z-loss         z = (1/T) sum_t lse_t^2:  dL_j += c_z * 2 * lse_t / T * softmax(L)_j
 * logits (T, E) are the logits the forward routed on.  dlogits (T, E).
 */
void oracle_router_backward(int64_t T, int32_t E, int32_t K, const double *logits,
                            const int32_t *ids, const double *dw, const int64_t *counts,
                            int32_t score_func, int32_t renormalize, double route_scale,
                            double c_bal, double c_z, double *dlogits)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *L = logits + t * E;
        double *dL = dlogits + t * E;
        double *p = (double *)malloc(sizeof(double) * (size_t)E);     /* softmax(L) */
        double *score = (double *)malloc(sizeof(double) * (size_t)E);
        double *dscore = (double *)malloc(sizeof(double) * (size_t)E);
        double m = L[0];
        for (int32_t e = 0; e < E; ++e)
            if (L[e] > m)
                m = L[e];
        double se = 0.0;
        for (int32_t e = 0; e < E; ++e)
            se += exp(L[e] - m);
        const double lse = m + log(se);
        for (int32_t e = 0; e < E; ++e) {
            p[e] = exp(L[e] - m) / se;
            score[e] = score_func == 1 ? 1.0 / (1.0 + exp(-L[e])) : p[e];
            dscore[e] = 0.0;
        }
        /* the gate weights */
        double S = 0.0, sdw = 0.0;
        for (int32_t k = 0; k < K; ++k)
            S += score[ids[t * K + k]];
        for (int32_t k = 0; k < K; ++k)
            sdw += dw[t * K + k] * score[ids[t * K + k]] / S;
        for (int32_t k = 0; k < K; ++k) {
            int32_t j = ids[t * K + k];
            if (renormalize)
                dscore[j] += route_scale / S * (dw[t * K + k] - sdw);
            else
                dscore[j] += route_scale * dw[t * K + k];
        }
        /* the balance loss, through the normalised scores */
        double ss = 0.0;
        for (int32_t e = 0; e < E; ++e)
            ss += score[e];
        if (score_func == 1) {
            double dot = 0.0;
            for (int32_t e = 0; e < E; ++e)
                dot += c_bal * (double)E * ((double)counts[e] / (double)(T * K)) / (double)T *
                       (score[e] / ss);
            for (int32_t e = 0; e < E; ++e) {
                double dn = c_bal * (double)E * ((double)counts[e] / (double)(T * K)) / (double)T;
                dscore[e] += (dn - dot) / ss;
            }
        } else {
            for (int32_t e = 0; e < E; ++e)
                dscore[e] += c_bal * (double)E * ((double)counts[e] / (double)(T * K)) / (double)T;
        }
        /* the scores, from the logits */
        if (score_func == 1) {
            for (int32_t e = 0; e < E; ++e)
                dL[e] = dscore[e] * score[e] * (1.0 - score[e]);
        } else {
            double dot = 0.0;
            for (int32_t e = 0; e < E; ++e)
                dot += p[e] * dscore[e];
            for (int32_t e = 0; e < E; ++e)
                dL[e] = p[e] * (dscore[e] - dot);
        }
        /* the z-loss */
        for (int32_t e = 0; e < E; ++e)
            dL[e] += c_z * 2.0 * lse / (double)T * p[e];
        free(p);
        free(score);
        free(dscore);
    }
}

/*
 * Gradients of the router's linear map L = x W_r + b (+ noise), from dlogits:
 *     dW_r[d,e] = sum_t x[t,d] * dL[t,e]      (tokens in order)
 *     db[e]     = sum_t dL[t,e]
 *     dx_r[t,d] = sum_e dL[t,e] * W_r[d,e]
 * The noise is an input, not a parameter.  db and dx_r may be NULL.
 */
void oracle_router_linear_backward(int64_t T, int32_t D, int32_t E, const void *x, int32_t x_dtype,
                                   const float *w_r, const double *dlogits, double *dw_r,
                                   double *db, double *dx_r)
{
#pragma omp parallel for schedule(static)
    for (int32_t d = 0; d < D; ++d) {
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t)
                acc += elem(x, x_dtype, t * D + d) * dlogits[t * E + e];
            dw_r[(int64_t)d * E + e] = acc;
        }
    }
    if (db) {
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t)
                acc += dlogits[t * E + e];
            db[e] = acc;
        }
    }
    if (dx_r) {
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t)
            for (int32_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int32_t e = 0; e < E; ++e)
                    acc += dlogits[t * E + e] * (double)w_r[(int64_t)d * E + e];
                dx_r[t * D + d] = acc;
            }
    }
}

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* d silu / d g = s + g * s * (1 - s), s = 1 / (1 + exp(-g)) */
static double dsilu(double g)
{
    double sg = 1.0 / (1.0 + exp(-g));
    return sg + g * sg * (1.0 - sg);
}

/*
 * Backward of the expert FFN for a list of rows (token tok[r] through expert
 * ex[r] with gate weight wt[r]).  For one row, with x its token's input and
 * dYp = wt * dY[tok] (the gradient reaching this expert's output):
 *     g = x Wg,  u = x Wu,  h = silu(g) * u,  o = h Wd   (the forward, recomputed)
 *     dw     = <dY[tok], o>                 (gradient of the gate weight)
 *     dh_f   = sum_j dYp_j Wd[f,j]
 *     dg_f   = dh_f * u_f * silu'(g_f),   du_f = dh_f * silu(g_f)
 *     dx_d   = sum_f dg_f Wg[d,f] + du_f Wu[d,f]
 * Weights are (E, D, F) gate/up and (E, F, D) down, row-major, w_dtype.
 * dy is (T, D).  Outputs: dw (n), dx (n, D); h, dg, du (n, F) may be NULL.
 */
void oracle_expert_backward_rows(int64_t n, const int32_t *tok, const int32_t *ex,
                                 const double *wt, int32_t D, int32_t F, const void *x,
                                 int32_t x_dtype, const double *dy, const void *w_gate,
                                 const void *w_up, const void *w_down, int32_t w_dtype,
                                 double *dw, double *dx, double *h_out, double *dg_out,
                                 double *du_out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
        const int64_t t = tok[r];
        const int64_t wo = (int64_t)ex[r] * D * F; /* this expert's matrices */
        double *g = (double *)malloc(sizeof(double) * (size_t)F);
        double *u = (double *)malloc(sizeof(double) * (size_t)F);
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        double *dh = (double *)malloc(sizeof(double) * (size_t)F);
        double *xr = (double *)malloc(sizeof(double) * (size_t)D);
        for (int32_t d = 0; d < D; ++d)
            xr[d] = elem(x, x_dtype, t * D + d);
        for (int32_t f = 0; f < F; ++f) {
            double ga = 0.0, ua = 0.0;
            for (int32_t d = 0; d < D; ++d) {
                ga += xr[d] * elem(w_gate, w_dtype, wo + (int64_t)d * F + f);
                ua += xr[d] * elem(w_up, w_dtype, wo + (int64_t)d * F + f);
            }
            g[f] = ga;
            u[f] = ua;
            h[f] = silu(ga) * ua;
        }
        /* dw = <dY, o> with o = h Wd; dh = dYp Wd^T */
        double dwr = 0.0;
        for (int32_t j = 0; j < D; ++j) {
            double o = 0.0;
            for (int32_t f = 0; f < F; ++f)
                o += h[f] * elem(w_down, w_dtype, wo + (int64_t)f * D + j);
            dwr += dy[t * D + j] * o;
        }
        dw[r] = dwr;
        for (int32_t f = 0; f < F; ++f) {
            double acc = 0.0;
            for (int32_t j = 0; j < D; ++j)
                acc += wt[r] * dy[t * D + j] * elem(w_down, w_dtype, wo + (int64_t)f * D + j);
            dh[f] = acc;
        }
        /* through SwiGLU: reuse g for dg and u for du */
        for (int32_t f = 0; f < F; ++f) {
            double dgf = dh[f] * u[f] * dsilu(g[f]);
            double duf = dh[f] * silu(g[f]);
            if (h_out)
                h_out[r * F + f] = h[f];
            g[f] = dgf;
            u[f] = duf;
            if (dg_out)
                dg_out[r * F + f] = dgf;
            if (du_out)
                du_out[r * F + f] = duf;
        }
        for (int32_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int32_t f = 0; f < F; ++f)
                acc += g[f] * elem(w_gate, w_dtype, wo + (int64_t)d * F + f) +
                       u[f] * elem(w_up, w_dtype, wo + (int64_t)d * F + f);
            dx[r * D + d] = acc;
        }
        free(g);
        free(u);
        free(h);
        free(dh);
        free(xr);
    }
}

/*
 * The same per-row quantities restricted to a list of hidden columns
 * fcols (nf of them): for each row r and column f = fcols[i]
 *     g_f = x Wg[:,f],  u_f = x Wu[:,f],  h_f = silu(g_f) u_f,
 *     dh_f = sum_j wt_r dY[tok_r, j] Wd[f, j],
 *     dg_f = dh_f u_f silu'(g_f),  du_f = dh_f silu(g_f)
 * written to h, dg, du (n, nf).  With them, oracle_expert_wgrad (F := nf)
 * gives the weight gradients' columns fcols of dWg, dWu and rows fcols of dWd
 * at a cost of n * 3 * D per column.
 */
void oracle_expert_backward_cols(int64_t n, const int32_t *tok, const int32_t *ex,
                                 const double *wt, int32_t D, int32_t F, int32_t nf,
                                 const int32_t *fcols, const void *x, int32_t x_dtype,
                                 const double *dy, const void *w_gate, const void *w_up,
                                 const void *w_down, int32_t w_dtype, double *h, double *dg,
                                 double *du)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        const int64_t t = tok[r];
        const int64_t wo = (int64_t)ex[r] * D * F;
        for (int32_t i = 0; i < nf; ++i) {
            const int64_t f = fcols[i];
            double g = 0.0, u = 0.0, dh = 0.0;
            for (int32_t d = 0; d < D; ++d) {
                double xd = elem(x, x_dtype, t * D + d);
                g += xd * elem(w_gate, w_dtype, wo + (int64_t)d * F + f);
                u += xd * elem(w_up, w_dtype, wo + (int64_t)d * F + f);
                dh += wt[r] * dy[t * D + d] * elem(w_down, w_dtype, wo + f * D + d);
            }
            h[r * nf + i] = silu(g) * u;
            dg[r * nf + i] = dh * u * dsilu(g);
            du[r * nf + i] = dh * silu(g);
        }
    }
}

/*
 * Weight gradients of one expert from its rows (in row order), given each
 * row's h, dg, du (n, F) from oracle_expert_backward_rows:
 *     dWg[d,f] = sum_r x[tok_r, d] * dg_r[f]
 *     dWu[d,f] = sum_r x[tok_r, d] * du_r[f]
 *     dWd[f,j] = sum_r h_r[f] * wt_r * dY[tok_r, j]
 * dWg, dWu (D, F) and dWd (F, D), row-major.  n = 0 gives zeros.
 */
void oracle_expert_wgrad(int64_t n, const int32_t *tok, const double *wt, int32_t D, int32_t F,
                         const void *x, int32_t x_dtype, const double *dy, const double *h,
                         const double *dg, const double *du, double *dWg, double *dWu,
                         double *dWd)
{
#pragma omp parallel for schedule(static)
    for (int32_t d = 0; d < D; ++d) {
        for (int32_t f = 0; f < F; ++f) {
            double ag = 0.0, au = 0.0;
            for (int64_t r = 0; r < n; ++r) {
                double xd = elem(x, x_dtype, (int64_t)tok[r] * D + d);
                ag += xd * dg[r * F + f];
                au += xd * du[r * F + f];
            }
            dWg[(int64_t)d * F + f] = ag;
            dWu[(int64_t)d * F + f] = au;
        }
    }
#pragma omp parallel for schedule(static)
    for (int32_t f = 0; f < F; ++f) {
        for (int32_t j = 0; j < D; ++j) {
            double a = 0.0;
            for (int64_t r = 0; r < n; ++r)
                a += h[r * F + f] * wt[r] * dy[(int64_t)tok[r] * D + j];
            dWd[(int64_t)f * D + j] = a;
        }
    }
}

/* Threads OpenMP will use (1 when built without OpenMP). */
int32_t oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return (int32_t)omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the following parallel loops (no effect without OpenMP).  The
   results do not depend on it: every parallel loop owns disjoint outputs. */
void oracle_set_num_threads(int32_t n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n < 1 ? 1 : (int)n);
#else
    (void)n;
#endif
}
