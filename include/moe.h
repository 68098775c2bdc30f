/*
 * moe.h -- C ABI of libmoe_b200.so: the forward pass of a token-choice top-k
 * Mixture-of-Experts layer on NVIDIA B200 (sm_100a), and its backward.
 *
 * The layer (sources cited by page title and section):
 *   "Lab: build a tiny MoE in PyTorch" (open-llm-engineering), sections
 *   "The contract", "Full implementation", "Add a capacity limit";
 *   "2.9 Mixture-of-Experts (MoE) Architectures" (llm-stack-book), sections
 *   "The Router", "A Toy MoE Layer From Scratch", "Capacity Factor, Token
 *   Dropping, and the Worked Numbers".
 *
 *   y = sum over the K experts a token selects of w_k * Expert_{id_k}(x),
 *   Expert_e(x) = (silu(x Wg_e) * (x Wu_e)) Wd_e,
 *   ids = top-K of the router logits x W_r (+ bias) (+ noise), ties to the
 *   lower expert id; w = softmax probabilities of the selected experts,
 *   renormalised to sum to one; with a capacity factor, each expert keeps its
 *   first C assignments in token order and the rest contribute zero.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument named as a buffer is a DEVICE pointer unless
 *     stated otherwise; the caller allocates and owns every buffer.  The
 *     library allocates no device or host memory and never synchronises the
 *     host, except moe_get_device_status.
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work is enqueued on it, asynchronously.
 *   - Layouts are row-major and dense:
 *       x (T, D), y (T, D), w_router (D, E) fp32, router_bias (E) fp32,
 *       logit_noise (T, E) fp32, w_gate / w_up (E, D, F), w_down (E, F, D),
 *       x_perm / y_perm (max_rows, D), h (max_rows, F),
 *       topk_ids (T, K) int32, topk_w (T, K) fp32, probs (T, E) fp32.
 *     dtype (moe_config.dtype) is the element type of x, y, the expert
 *     weights, x_perm, h and y_perm; router arithmetic is always fp32.
 *   - Alignment: D and F must be multiples of 8, and every buffer must start
 *     on a 16-byte boundary (MOE_ERR_ALIGN otherwise).
 *   - Errors in the arguments are reported before anything is enqueued, and
 *     nothing is enqueued then.  A failure in the CUDA runtime returns
 *     MOE_ERR_CUDA.  Faults found on the device (an index out of range, a
 *     wait that gave up) are recorded in the workspace status word and read
 *     with moe_get_device_status.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_ARG = -1,            /* K outside [1, min(E, 8)], E > 256, a NULL required pointer, a bad enum */
    MOE_ERR_SHAPE = -2,          /* T, D, F or E below 1, or T*K beyond 2^31 - 1 */
    MOE_ERR_UNSUPPORTED = -3,    /* an option this library does not implement */
    MOE_ERR_ALIGN = -4,          /* D or F not a multiple of 8, or a buffer not 16-byte aligned */
    MOE_ERR_CUDA = -5,           /* a CUDA runtime call failed */
    MOE_ERR_DEVICE_TIMEOUT = -6, /* a kernel gave up a bounded wait (device status) */
    MOE_ERR_DEVICE_BOUNDS = -7,  /* a kernel met an index out of range (device status) */
    MOE_ERR_WORKSPACE = -8       /* workspace NULL or smaller than the size query returned */
} moe_status;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/*
 * Router score function: softmax over the experts ("Lab: build a tiny MoE in
 * PyTorch", "Full implementation") or a per-expert sigmoid (the lab's
 * extension "sigmoid top-k"; the NeMo Gate's score_func).  Either way the
 * experts are selected on the logits (plus the selection bias), and the
 * weights are the scores of the selected experts.
 */
typedef enum moe_score_func { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_func;

/* Device status flags (bit set), as read by moe_get_device_status. */
#define MOE_DEVFLAG_TIMEOUT 0x1
#define MOE_DEVFLAG_BOUNDS 0x2

typedef struct moe_config {
    int64_t T;             /* tokens = batch * sequence, >= 1 */
    int32_t D;             /* d_model, multiple of 8 */
    int32_t F;             /* expert hidden size d_hidden, multiple of 8 */
    int32_t E;             /* number of experts, 1..256 */
    int32_t K;             /* experts per token (top-k), 1..min(E, 8) */
    float capacity_factor; /* <= 0: dropless; > 0: C = max(1, ceil(cf * T * K / E)) */
    int32_t score_func;    /* moe_score_func */
    int32_t renormalize;   /* 1: selected scores renormalised to sum to one (Mixtral);
                              0: kept as they are (GShard / Switch softmax-then-top-k) */
    int32_t dtype;         /* moe_dtype */
    int32_t n_groups;      /* 0 or 1: no group limit; else the experts form n_groups
                              contiguous groups (E divisible by n_groups, <= 32) */
    int32_t topk_groups;   /* groups a token may use, 1..n_groups, with
                              topk_groups * E / n_groups >= K (ignored without groups) */
    float route_scale;     /* multiplies every routing weight; > 0 (1 = none) */
    int32_t F_shared;      /* hidden size of a shared expert that every token passes
                              through (0: none), multiple of 8 */
} moe_config;

/* Returns a static, NUL-terminated description of a status code. */
MOE_API const char *moe_status_string(int32_t status);

/* Library version as 10000*major + 100*minor + patch. */
MOE_API int32_t moe_version(void);

/* Validates a configuration (no device work).  MOE_OK or the error code. */
MOE_API moe_status moe_check_config(const moe_config *cfg);

/*
 * Expert capacity C ("Lab: build a tiny MoE in PyTorch", section "Add a
 * capacity limit"): max(1, ceil(cf * T * K / E)) computed in double; T*K when
 * dropless.  Host-only.
 */
MOE_API moe_status moe_capacity(const moe_config *cfg, int64_t *capacity);

/*
 * Upper bound on the kept assignments R: T*K dropless, else min(T*K, E*C).
 * Rows of x_perm, h and y_perm must be allocated for this many.  Host-only.
 */
MOE_API moe_status moe_max_rows(const moe_config *cfg, int64_t *rows);

/*
 * Bytes of device workspace that moe_route, moe_dispatch and moe_expert_ffn
 * need (the same buffer serves all three; it holds the device status word and
 * per-block partials).  The workspace must be 256-byte aligned and zeroed
 * once before first use (the status word must start at zero).
 */
MOE_API moe_status moe_workspace_size(const moe_config *cfg, size_t *bytes);

/*
 * Bytes of device workspace moe_forward needs: the above plus every
 * intermediate of the layer (routing, dispatch layout, x_perm, h, y_perm).
 */
MOE_API moe_status moe_forward_workspace_size(const moe_config *cfg, size_t *bytes);

/*
 * The router weight prepared for the tensor-core router of bf16 layers
 * ("Lab: build a tiny MoE in PyTorch", "Full implementation": the router
 * logits are fp32).  Each fp32 weight W_r[d, e] is split exactly into three
 * bf16 terms, hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
 * (round to nearest even), so that x * hi + x * mid + x * lo, accumulated in
 * fp32 on the tensor cores, is the fp32 product.  Layout: bf16
 * terms[p][e][d] for p = 0 (hi), 1 (mid), 2 (lo), e < E16 and d < D, where
 * E16 is E rounded up to 16, 32, 64 or 128; the rows e >= E are zero.
 *
 * moe_router_terms_size: 3 * E16 * D * 2 bytes for bf16 layers with E <= 128
 * (the layers whose router can run on the tensor cores), 0 for the others.
 * moe_router_prepare writes the terms of w_router (D, E) fp32 into
 * w_router_terms (16-byte aligned, moe_router_terms_size bytes) on the
 * stream; MOE_ERR_UNSUPPORTED where the size is 0.  The terms depend on the
 * weight only: prepare them once per weight value (again after every update
 * of W_r) and pass them to moe_route / moe_forward, which then skip the split.
 */
MOE_API moe_status moe_router_terms_size(const moe_config *cfg, size_t *bytes);
MOE_API moe_status moe_router_prepare(const moe_config *cfg, const float *w_router,
                                      void *w_router_terms, void *stream);

/*
 * Router: "Lab: build a tiny MoE in PyTorch", section "Full implementation"
 * (fp32 router logits, softmax, top-k, renormalised weights, balance loss and
 * router z-loss) and "2.9 Mixture-of-Experts (MoE) Architectures", section
 * "The Router" (noisy top-k gating adds noise to the logits before top-k).
 *
 *   L[t,e]  = sum_d x[t,d] W_r[d,e] + router_bias[e] + logit_noise[t,e]   (fp32)
 *   s[t,e]  = softmax(L[t,:])_e, or sigmoid(L[t,e]) (score_func)
 *   u[t,e]  = L[t,e] + selection_bias[e]   (selection only: DeepSeek-V3's
 *             auxiliary-loss-free balancing, "2.9 Mixture-of-Experts (MoE)
 *             Architectures", "Exercises" 6)
 *   groups  with n_groups > 1: a group's score is its largest u; only the
 *           topk_groups groups of largest score (ties: lower group id) are
 *           eligible
 *   ids[t,:]= the K eligible experts of largest u, ties to the lower id, in
 *             descending order
 *   w[t,k]  = route_scale * s[t,ids[t,k]] (/ sum_j s[t,ids[t,j]] when renormalize)
 *   p[t,e]  = s[t,e] / sum_e' s[t,e']  (the softmax itself, or the normalised
 *             sigmoid scores)
 *   mean_prob[e] = (1/T) sum_t p[t,e]
 *   losses[0] = z-loss = (1/T) sum_t (logsumexp_e L[t,e])^2
 *   losses[1] = balance = E * sum_e (counts_e / (T*K)) * mean_prob[e],
 *               counts_e = assignments to e before any capacity drop
 *   losses[2] = router entropy = (1/T) sum_t -sum_e q log max(q, 1e-9),
 *               q = softmax(L[t,:])  ("Full implementation", stats)
 *
 * x (T, D) dtype; w_router (D, E) fp32.  w_router_terms may be NULL or the
 * terms moe_router_prepare wrote for this w_router (same D and E): the
 * tensor-core router (bf16 layers, E <= 128, T >= 2048) then reads them
 * instead of splitting w_router itself, one kernel fewer; the other routers
 * ignore them.  router_bias (E), selection_bias (E)
 * and logit_noise (T, E) may be NULL.  logits_in (T, E), if not NULL, are
 * taken as the complete routing logits L: x, w_router, router_bias and noise
 * are then not read and may be NULL (selection_bias still applies).
 * logits_out (T, E) and probs_out (T, E, the p above) may be NULL.
 * topk_ids (T, K) and topk_w (T, K) are required.  mean_prob (E) and
 * losses (3) may be NULL; the statistics are then skipped.
 * The reductions behind mean_prob and losses run in a fixed order
 * (deterministic run to run), finished on the device by the router kernel's
 * block that completes last (workspace status word 16 counts the blocks and
 * is left at zero).
 */
MOE_API moe_status moe_route(const moe_config *cfg, const void *x, const float *w_router,
                     const void *w_router_terms, const float *router_bias, const float *selection_bias,
                     const float *logit_noise, const float *logits_in,
                     float *logits_out, float *probs_out, int32_t *topk_ids, float *topk_w,
                     float *mean_prob, float *losses, void *workspace, size_t workspace_bytes,
                     void *stream);

/*
 * DeepSeek-V3 auxiliary-loss-free balancing step, "2.9 Mixture-of-Experts
 * (MoE) Architectures", "Exercises" 6 (update_bias):
 *   selection_bias[e] += gamma * sign(mean_e'(counts) - counts[e])
 * so overloaded experts become less likely to be selected and underloaded
 * ones more; an expert exactly at the mean keeps its bias.  counts (E, int32,
 * e.g. from moe_dispatch or moe_forward) and selection_bias (E, fp32) are
 * device arrays; updated in place on the stream.
 */
MOE_API moe_status moe_update_selection_bias(const moe_config *cfg, const int32_t *counts,
                                             float gamma, float *selection_bias, void *stream);

/*
 * Dispatch: per-expert histogram, capacity drop, exclusive-scan offsets and a
 * stable expert-major permutation, then the gather of token rows.
 * "Lab: build a tiny MoE in PyTorch", sections "Full implementation" (bincount,
 * gather flat[token_index]) and "Add a capacity limit" (first C assignments of
 * each expert in token order are kept).
 *
 *   counts[e]  = #{(t,k) : topk_ids[t,k] = e}                    (E)
 *   kept[e]    = min(counts[e], C)                                (E)
 *   offsets    = exclusive prefix sum of kept, offsets[E] = R     (E+1)
 *   perm[row]  = t*K + k of the assignment stored at row; the rows of expert e
 *                are offsets[e] .. offsets[e+1]-1, in increasing t  (max_rows)
 *   row_of[t*K+k] = its row, or -1 if dropped                     (T*K)
 *   x_perm[row, :] = x[perm[row] / K, :]                          (max_rows, D)
 *
 * Every output is fully determined (bit-exact run to run).  x and x_perm may
 * both be NULL: only the index arrays are then produced.  Entries of perm and
 * rows of x_perm at and beyond R are left untouched.
 */
MOE_API moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *topk_ids,
                        int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *perm,
                        int32_t *row_of, void *x_perm, void *workspace, size_t workspace_bytes,
                        void *stream);

/*
 * Grouped SwiGLU experts over each expert's contiguous row block, with the
 * routing weight applied to the output.  "Lab: build a tiny MoE in PyTorch",
 * section "Full implementation" (SwiGLUExpert: down(silu(gate x) * up x), no
 * biases; each expert output scaled by its combine weight).
 *
 * For every row r < offsets[E] of expert e (offsets[e] <= r < offsets[e+1]):
 *   h[r, :]      = silu(x_perm[r] Wg_e) * (x_perm[r] Wu_e)        (dtype)
 *   y_perm[r, :] = topk_w[perm[r]] * (h[r] Wd_e)                  (dtype)
 * with fp32 accumulation, silu(z) = z / (1 + exp(-z)).  bf16 runs on tcgen05
 * tensor cores; fp32 runs in true fp32 (no TF32).
 * h is a caller-provided intermediate of max_rows x F elements.  offsets,
 * perm and topk_w are device arrays as produced by moe_dispatch / moe_route.
 * perm and topk_w may both be NULL: every row then gets weight 1 (a shared
 * expert: cfg with E = 1, K = 1, F = F_shared, x_perm = x, offsets = {0, T}).
 */
MOE_API moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                          const int32_t *perm, const float *topk_w, const void *w_gate,
                          const void *w_up, const void *w_down, void *h, void *y_perm,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * Combine back to token order.  "Lab: build a tiny MoE in PyTorch", sections
 * "Full implementation" (index_add_ of weighted expert outputs) and "Add a
 * capacity limit" (an all-dropped token returns zero).
 *
 *   y[t, :] = y_add[t, :] + sum over k = 0..K-1 with row_of[t*K+k] >= 0 of
 *             y_perm[row_of[t*K+k], :]
 * summed in fp32 (y_add first, then the slots in order) and rounded once to
 * dtype (deterministic; the routing weight was applied by moe_expert_ffn).
 * y_add (T, D) dtype may be NULL; it carries a shared expert's output ("Lab:
 * build a tiny MoE in PyTorch", "Add a shared expert": routed + shared).
 */
MOE_API moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *row_of,
                               const void *y_add, void *y, void *stream);

/*
 * The whole layer ("Lab: build a tiny MoE in PyTorch", "Full implementation";
 * "2.9 Mixture-of-Experts (MoE) Architectures", "A Toy MoE Layer From
 * Scratch"): moe_route -> moe_dispatch -> moe_expert_ffn -> (shared expert)
 * -> moe_combine on one stream, every intermediate in the workspace
 * (moe_forward_workspace_size bytes).  w_router_terms as for moe_route
 * (NULL: the router splits w_router itself).  With cfg->F_shared > 0,
 * w_gate_shared / w_up_shared (D, F_shared) and w_down_shared (F_shared, D)
 * are required and the shared SwiGLU expert's output over all tokens is
 * added in the combine; otherwise they are ignored (may be NULL).  y (T, D)
 * dtype is required; losses (3),
 * mean_prob (E), counts (E, before drops), topk_ids (T, K) and topk_w (T, K)
 * are optional copies of the routing results (NULL to skip).
 */
MOE_API moe_status moe_forward(const moe_config *cfg, const void *x, const float *w_router,
                       const void *w_router_terms, const float *router_bias, const float *selection_bias,
                       const float *logit_noise, const void *w_gate,
                       const void *w_up, const void *w_down, const void *w_gate_shared,
                       const void *w_up_shared, const void *w_down_shared, void *y, float *losses,
                       float *mean_prob, int32_t *counts, int32_t *topk_ids, float *topk_w,
                       void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------ training
 *
 * The backward of the layer's training loss ("Lab: build a tiny MoE in
 * PyTorch", "Smoke test and backward pass": loss = main + c_bal * balance +
 * c_z * z, differentiated by autograd; "2.9 Mixture-of-Experts (MoE)
 * Architectures", "The Router": the top-k index decision is a stop-gradient,
 * gradient reaches the router only through the kept gate weights and the
 * auxiliary losses, and an expert a token did not choose gets nothing from
 * it).  The stop-gradients, as autograd applies them to the forward: the chosen
 * ids (with the group limit and the selection bias), the capacity keep mask
 * and the balance loss's counts f_e.  Logit noise is an input.  bf16 layers
 * run the backward's GEMMs on the tensor cores; fp32 layers in true fp32 on
 * the SIMT pipes (no TF32).
 */

/*
 * Bytes of the state moe_forward_train keeps for moe_backward:
 * moe_forward_workspace_size plus the routed logits (T, E) fp32, the gate/up
 * pre-activations (max_rows, 2F) and, with a shared expert, its (T, 2 F_shared).
 */
MOE_API moe_status moe_train_state_size(const moe_config *cfg, size_t *bytes);

/*
 * moe_forward for training ("Lab: build a tiny MoE in PyTorch", "Smoke test
 * and backward pass"): the same arguments and results, with the
 * workspace replaced by `state` (moe_train_state_size bytes, 256-byte
 * aligned), which keeps what moe_backward reads: the routing results, the
 * dispatch layout, x_perm, [g | u] = the gate/up pre-activations in the
 * layer dtype, h, the unweighted expert outputs and the logits.  The state must not
 * be written between this call and moe_backward.  y equals moe_forward's up
 * to rounding order: the routing weight multiplies each expert output in the
 * combine (fp32) instead of in the down projection's epilogue.
 */
MOE_API moe_status moe_forward_train(const moe_config *cfg, const void *x, const float *w_router,
                                     const float *router_bias, const float *selection_bias,
                                     const float *logit_noise, const void *w_gate, const void *w_up,
                                     const void *w_down, const void *w_gate_shared,
                                     const void *w_up_shared, const void *w_down_shared, void *y,
                                     float *losses, float *mean_prob, int32_t *counts,
                                     int32_t *topk_ids, float *topk_w, void *state,
                                     size_t state_bytes, void *stream);

/* Bytes of device scratch moe_backward needs (its status word first). */
MOE_API moe_status moe_backward_workspace_size(const moe_config *cfg, size_t *bytes);

/*
 * Gradients of  loss = sum_{t,d} dy[t,d] * y[t,d] + c_balance * balance + c_z * z
 * for the forward recorded in `state` by moe_forward_train (pass the same x
 * and weights).  dy (T, D) in the layer dtype is the upstream gradient of y; c_balance and
 * c_z are the loss coefficients (the lab's 0.01 and 0.001), host values.
 *
 *   gate weights  dw[t,k] = <dy[t], o_k(x_t)> for a kept slot, 0 for a dropped
 *                 one; through the renormalisation (or not) and route_scale
 *   router        dL[t] = softmax / sigmoid backward of the gate weights' and
 *                 the balance loss's score gradients, plus c_z * 2 lse_t / T * p_t
 *   experts       dH = (w dy) Wd^T, [dg | du] = dH * [u silu'(g) | silu(g)],
 *                 dx_e = dg Wg^T + du Wu^T; weight gradients summed over each
 *                 expert's rows
 *   input         dx = dL W_r^T + sum over kept slots of dx_e (+ shared expert)
 *
 * Outputs, all overwritten: dx (T, D) in the layer dtype; dw_router (D, E) fp32;
 * db_router (E) fp32 or NULL; dw_gate, dw_up (E, D, F) fp32; dw_down
 * (E, F, D) fp32; with a shared expert dw_gate_shared, dw_up_shared
 * (D, F_shared) and dw_down_shared (F_shared, D) fp32 (ignored otherwise).
 * Rounding (bf16 layers): dy * w, [dg | du] and each expert's dx rows are
 * rounded to bf16 before the next contraction; every sum is fp32 (fp32 layers
 * keep every value in fp32).  Deterministic.
 * workspace: moe_backward_workspace_size bytes, 256-byte aligned; device
 * faults are reported in its status word (moe_get_device_status(workspace)).
 */
MOE_API moe_status moe_backward(const moe_config *cfg, const void *x, const float *w_router,
                                const void *w_gate, const void *w_up, const void *w_down,
                                const void *w_gate_shared, const void *w_up_shared,
                                const void *w_down_shared, const void *state, size_t state_bytes,
                                const void *dy, float c_balance, float c_z, void *dx,
                                float *dw_router, float *db_router, float *dw_gate, float *dw_up,
                                float *dw_down, float *dw_gate_shared, float *dw_up_shared,
                                float *dw_down_shared, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * Number of kernels one moe_backward call launches for this configuration
 * (0 for an invalid or unsupported one).
 */
MOE_API int32_t moe_backward_kernel_count(const moe_config *cfg);

/* ------------------------------------------------------- expert parallelism
 *
 * "Lab: build a tiny MoE in PyTorch", "From local loop to expert
 * parallelism": sort by owner -> exchange counts -> all-to-all dispatch ->
 * grouped local experts -> reverse all-to-all -> scatter-add, with the same
 * mathematical output as the local layer.  Rank r of W owns the contiguous
 * experts r*EL .. r*EL + EL - 1 (EL = E / W).  moe_dispatch's expert-major rows
 * are already sorted by owner; the exchanges themselves are collectives of the
 * caller's communication library.  These entry points are the layer's own
 * steps around them.
 */

/* Bytes of device scratch moe_ep_layout needs (status word first). */
MOE_API moe_status moe_ep_workspace_size(int32_t world, int32_t experts_per_rank, size_t *bytes);

/*
 * Receive layout of one rank's experts.  recv_counts (world, EL) int32: rows
 * that arrive from source rank s for local expert e, in the order they arrive
 * (source-major: all of source 0's rows, its expert 0 first, then source 1's).
 * Writes offsets (EL + 1) int32, the expert-major row offsets of the local
 * experts (expert e's rows are its segments from sources 0..W-1 in order);
 * dst_of (rows) int32, the expert-major row of each arrived row; src_of
 * (rows) int32, the inverse.  rows = sum of recv_counts <= max_rows; world *
 * EL <= 256.  All device pointers; workspace = moe_ep_workspace_size bytes.
 */
MOE_API moe_status moe_ep_layout(int32_t world, int32_t experts_per_rank, const int32_t *recv_counts,
                                 int64_t max_rows, int32_t *offsets, int32_t *dst_of, int32_t *src_of,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * out[i, :] = in[idx[i], :] for i < n: rows of row_bytes (a multiple of 16)
 * bytes; in has in_rows rows; an idx outside [0, in_rows) sets the bounds flag
 * of `workspace`'s status word and leaves that row unwritten.  Device pointers.
 */
MOE_API moe_status moe_permute_rows(const void *in, int64_t in_rows, const int32_t *idx, int64_t n,
                                    int64_t row_bytes, void *out, void *workspace, void *stream);

/*
 * moe_combine with the routing weight applied here (the combine's weighted
 * index_add_ of "Full implementation"): y[t] = y_add[t] + sum over
 * kept slots of topk_w[t, k] * y_perm[row_of[t, k]], fp32, rounded once.  For
 * unweighted expert outputs (the rows that come back from the experts' owners).
 */
MOE_API moe_status moe_combine_weighted(const moe_config *cfg, const void *y_perm,
                                        const int32_t *row_of, const float *topk_w,
                                        const void *y_add, void *y, void *stream);

/* ------------------------------------------ expert parallelism over peer memory
 *
 * The same layer with the two exchanges done by this library's kernels
 * instead of all-to-all collectives: every rank's receive buffers are mapped
 * into every rank's address space (CUDA IPC; NVLink between the GPUs of one
 * node), the dispatch kernel stores each kept token row straight into its
 * owner's receive buffer at its expert-major row, the owner runs moe_expert_ffn
 * on that buffer, and the combine kernel loads each kept slot's result from
 * its owner's output buffer.  The caller's communication library supplies an
 * all-gather of the kept counts (world x E int32, each rank's moe_dispatch
 * `kept`) before moe_ep_peer_dispatch, and two stream-ordered barriers: after
 * moe_ep_peer_dispatch on every rank (all rows have arrived) and after every
 * owner's moe_expert_ffn (all results are ready).  No host synchronisation.
 *
 * Receive layout.  Rank o's buffer holds its experts e = o*EL .. o*EL+EL-1
 * (EL = E / world) in order; expert e's block holds the kept rows of sources
 * 0 .. world-1 in order, each source's rows in its own expert-major order.
 * The slot (t, k) of source `rank`, routed to expert e and kept at local row
 * r = row_of[t, k], lands at
 *   sum_{o*EL <= e' < e} sum_s kept_all[s][e'] + sum_{s < rank} kept_all[s][e]
 *     + (r - offsets[e])
 * of its owner's buffer -- the expert-major order of the all-to-all path's
 * moe_ep_layout.
 */

/* Bytes of one peer-exchange handle (a cudaIpcMemHandle_t). */
#define MOE_IPC_HANDLE_BYTES 64

/*
 * Setup-time entry points for the peer-mapped buffers (not for the per-step
 * path: they allocate, and opening a mapping synchronises).  moe_ipc_alloc:
 * `bytes` of device memory on the current device (*ptr) and its exchange
 * handle (MOE_IPC_HANDLE_BYTES host bytes, written to `handle`), to be sent
 * to the other ranks.  moe_ipc_open: map another process's buffer from its
 * handle into this process (*ptr; a handle of this process's own buffer is
 * refused by CUDA: use the pointer itself).  moe_ipc_close unmaps, moe_ipc_free
 * frees the owner's buffer (after every peer has closed it).  MOE_ERR_CUDA on
 * any CUDA error; *ptr is NULL then.
 */
MOE_API moe_status moe_ipc_alloc(size_t bytes, void **ptr, void *handle);
MOE_API moe_status moe_ipc_open(const void *handle, void **ptr);
MOE_API moe_status moe_ipc_close(void *ptr);
MOE_API moe_status moe_ipc_free(void *ptr);

/*
 * Dispatch of this rank's tokens into the owners' receive buffers (the
 * all-to-all dispatch of "From local loop to expert parallelism", done by
 * stores into the owners' memory).
 *   cfg            this rank's layer: T tokens, all E experts (E % world == 0)
 *   rank, world    this rank and the number of ranks (1 <= world <= 64)
 *   kept_all       (world, E) int32, device: every rank's kept counts
 *   x              (T, D) activations, device, 16-byte aligned
 *   topk_ids, row_of, offsets
 *                  this rank's moe_route ids (T, K) and moe_dispatch row_of
 *                  (T, K) and offsets (E + 1), device (moe_dispatch may be
 *                  called with x = x_perm = NULL: no local gather is needed)
 *   recv_bufs      device array of `world` device pointers: rank o's receive
 *                  buffer (its own pointer at index `rank`, peers' from
 *                  moe_ipc_open), each recv_rows rows of D elements
 *   local_offsets  out, device (EL + 1) int32: this rank's receive layout,
 *                  the offsets moe_expert_ffn takes (cfg.T = recv_rows, E = EL,
 *                  K = 1)
 *   remote_row     out, device (T, K) int32: the slot's row in its owner's
 *                  buffer, -1 for a dropped slot (moe_ep_peer_combine's map)
 *   workspace      moe_ep_workspace_size(world, EL) bytes
 * A count, id, row or destination out of range raises the bounds flag of
 * the workspace's status word (moe_get_device_status) and skips the slot.
 */
MOE_API moe_status moe_ep_peer_dispatch(const moe_config *cfg, int32_t rank, int32_t world,
                                        const int32_t *kept_all, const void *x,
                                        const int32_t *topk_ids, const int32_t *row_of,
                                        const int32_t *offsets, void *const *recv_bufs,
                                        int64_t recv_rows, int32_t *local_offsets,
                                        int32_t *remote_row, void *workspace,
                                        size_t workspace_bytes, void *stream);

/*
 * Weighted combine from the owners' output buffers (the reverse all-to-all and
 * scatter-add of "From local loop to expert parallelism", done by loads from
 * the owners' memory): y[t] = y_add[t] + sum over
 * kept slots, in slot order, of topk_w[t, k] * y_bufs[owner][remote_row[t, k]],
 * fp32 sums rounded once to cfg.dtype.  y_bufs: device array of `world`
 * device pointers to the owners' moe_expert_ffn outputs (unweighted:
 * perm = topk_w = NULL there), recv_rows rows each.  y_add (T, D) or NULL.
 */
MOE_API moe_status moe_ep_peer_combine(const moe_config *cfg, int32_t world, const int32_t *topk_ids,
                                       const int32_t *remote_row, const float *topk_w,
                                       const void *const *y_bufs, int64_t recv_rows,
                                       const void *y_add, void *y, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * moe_dispatch without a workspace, for callers that cannot allocate device
 * memory: code handed only its input and output buffers by a host framework
 * (a plugin in an inference engine, a fixed-budget C program) has no
 * workspace to pass, and cudaMalloc is not open to it because the call can
 * synchronise the device and lies outside the memory it was budgeted.  The
 * sources have no counterpart of this entry point; it is a deployment aid.
 *
 * Same arguments and results as moe_dispatch, minus the workspace.  Its
 * scratch (status word, per-chunk counts and rank bases) lives in a static
 * device array of 256 KiB inside the library, which every GPU that loads the
 * library holds until the process exits.  A problem whose scratch would not
 * fit (2 * ceil(T*K / 2048) * E int32 words plus 256 bytes) is rejected with
 * MOE_ERR_WORKSPACE before anything is enqueued.  Allocates nothing.
 *   - Every call looks up the array's device address on the current device
 *     (a table read; nothing is cached, so the address stays right after a
 *     cudaDeviceReset).  The first call on a device may load the library's
 *     device code there: make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; each call clears what must start at zero.  Calls whose work
 *     overlaps on the GPU (other streams, other threads) race on the array:
 *     order them on one stream.
 *   - Device-side range checks still guard every write; their flags go to a
 *     status word in the shared array, cleared at the start of every call and
 *     read back by moe_dispatch_noalloc_status.
 */
MOE_API moe_status moe_dispatch_noalloc(const moe_config *cfg, const void *x,
                                        const int32_t *topk_ids, int32_t *counts, int32_t *kept,
                                        int32_t *offsets, int32_t *perm, int32_t *row_of,
                                        void *x_perm, void *stream);

/*
 * The device status of the last moe_dispatch_noalloc on the current device
 * (the MOE_DEVFLAG_* bits of its static array's status word, read like
 * moe_get_device_status reads a workspace's): synchronises the stream, stores
 * the flags in *flags and returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT or
 * MOE_ERR_DEVICE_BOUNDS.  Allocates nothing.
 */
MOE_API moe_status moe_dispatch_noalloc_status(void *stream, int32_t *flags);

/*
 * Device status of a workspace: synchronises the stream, then reads the
 * status word.  *flags receives MOE_DEVFLAG_* bits (0 when clean).  Returns
 * MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_BOUNDS when a flag is set, MOE_OK
 * otherwise.  moe_clear_device_status enqueues a reset of the word.
 */
MOE_API moe_status moe_get_device_status(const void *workspace, void *stream, int32_t *flags);
MOE_API moe_status moe_clear_device_status(void *workspace, void *stream);

/*
 * Self-test of the device-side failure path.  Launches one kernel whose only
 * thread waits, with the library's bounded mbarrier wait and a limit of
 * limit_ns (1 us .. 1 s), on a barrier that nothing arrives at.  The wait gives
 * up, sets MOE_DEVFLAG_TIMEOUT (location code 900) in the workspace status
 * word, writes 1 to workspace word 2, and the kernel returns normally: a
 * following moe_get_device_status returns MOE_ERR_DEVICE_TIMEOUT and the CUDA
 * context stays usable.  The workspace is any zeroed buffer of >= 256 bytes
 * (256-byte aligned); clear it with moe_clear_device_status afterwards.
 */
MOE_API moe_status moe_selftest_wait_timeout(void *workspace, size_t workspace_bytes,
                                             int64_t limit_ns, void *stream);

/*
 * Number of kernels one moe_forward call launches for this configuration:
 * router 1 (bf16 with E <= 128 and T >= 2048: the tensor-core router, which
 * also routes and finishes the statistics; 2 when router_terms_given is 0,
 * the first splitting w_router into the workspace) or 2 (the SIMT logits GEMM
 * and the top-k kernel, plus a split-sum when that GEMM is split over d_model
 * in more than 4 parts), dispatch 1 (3 when the chunks of 2048 assignments
 * outnumber the resident blocks), gather 1, expert GEMMs 2, shared expert 3
 * (when F_shared > 0: its row offsets and two GEMMs), combine 1.  0 for an
 * invalid configuration.
 */
MOE_API int32_t moe_forward_kernel_count(const moe_config *cfg, int32_t router_terms_given);

/*
 * Kernel-boundary tracing for timing.  After moe_trace_attach(events, n),
 * moe_forward records events[i] (cudaEvent_t values passed as void*) on its
 * stream at each of the first n stage boundaries: 0 before the first kernel,
 * then after the router, the dispatch index pass, the gather, the gate/up
 * GEMM, the down GEMM, the shared expert (an empty stage without one) and the
 * combine (8 boundaries; moe_trace_stage_name names the stage that ends at
 * boundary i).  moe_trace_attach(NULL, 0)
 * detaches.  The table is process-wide and not thread-safe.
 */
MOE_API moe_status moe_trace_attach(void *const *events, int32_t n_events);
MOE_API int32_t moe_trace_boundary_count(void);
MOE_API const char *moe_trace_stage_name(int32_t boundary);

/*
 * The same for moe_backward (10 boundaries): start, rows (dYp and the
 * gate-weight gradients), router_bwd, dgrad_h, dgrad_x, wgrad_down,
 * wgrad_gate_up, shared_expert, router_wgrad, dx.  Separate from the
 * forward's events.
 */
MOE_API moe_status moe_trace_attach_backward(void *const *events, int32_t n_events);
MOE_API int32_t moe_trace_backward_boundary_count(void);
MOE_API const char *moe_trace_backward_stage_name(int32_t boundary);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
