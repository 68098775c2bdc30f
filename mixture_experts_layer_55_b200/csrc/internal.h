// internal.h -- host-side plan and launch declarations shared by the C ABI
// (api.cu) and the kernel files.  Not part of the public interface.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "moe.h"

namespace moe {

constexpr size_t kAlign = 256;

inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// A kernel attribute is per device: remember, per device, that a kernel's
// dynamic shared memory has been opted in (one bit per device for ordinals
// below 64; above that the attribute is set on every call).  Safe to use from
// several host threads: setting the attribute twice is harmless.
struct PerDeviceFlag {
    std::atomic<uint64_t> mask{0};
};
inline cudaError_t opt_in_smem(PerDeviceFlag& flag, const void* kernel, size_t smem)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t{1} << dev) : 0;
    if (bit && (flag.mask.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && bit) flag.mask.fetch_or(bit, std::memory_order_release);
    return e;
}

// ------------------------------------------------------------ router plan --
struct RouterPlan {
    int be;          // experts per logits block (8, 16, 32 or 64)
    int grid_t;      // token blocks of the logits GEMM (64 tokens each)
    int grid_e;      // expert blocks
    int splits;      // d_model splits of the logits GEMM
    int d_per_split; // multiple of 32
    int tpb_topk;    // tokens per block of the softmax/top-k kernel (8 or 16)
    int nb_topk;     // its blocks
};
RouterPlan router_plan(const moe_config& c);
// up to this many d_model splits the top-k kernel adds the partial logits itself
constexpr int kTopkMaxSplits = 4;

// Router options beyond the plain softmax / renormalised top-k.
struct RouteOpts {
    const float* sel_bias;  // E or null: added to the logits for selection only
    int score_func;         // 0 softmax, 1 sigmoid
    int renorm;             // 1: weights renormalised over the selected experts
    int n_groups;           // <= 1: no group limit
    int topk_groups;
    float route_scale;
};
inline RouteOpts route_opts(const moe_config& c, const float* sel_bias)
{
    RouteOpts o;
    o.sel_bias = sel_bias;
    o.score_func = c.score_func;
    o.renorm = c.renormalize;
    o.n_groups = c.n_groups > 1 ? c.n_groups : 1;
    o.topk_groups = c.n_groups > 1 ? c.topk_groups : 1;
    o.route_scale = c.route_scale;
    return o;
}

// ---------------------------------------------------------- dispatch plan --
constexpr int kDispatchChunk = 2048;  // assignments per dispatch block
inline int64_t dispatch_chunks(const moe_config& c)
{
    return (c.T * c.K + kDispatchChunk - 1) / kDispatchChunk;
}
// The index pass runs as one cooperative kernel (a block per chunk, all
// resident) up to one chunk per SM of a B200 (T*K <= 303104); beyond, or on a
// GPU where that many blocks cannot be resident, as three kernels.
inline bool dispatch_index_fused(const moe_config& c) { return dispatch_chunks(c) <= 148; }

// ------------------------------------------------------ workspace layout --
struct WsLayout {
    size_t status;      // int32[64]
    size_t r_part;      // splits * T * E fp32 partial logits of the SIMT router
    size_t r_terms;     // the tensor-core router's weight terms when the caller has none
    size_t r_mp;        // nb_topk * E fp32
    size_t r_z;         // nb_topk fp32
    size_t r_ent;       // nb_topk fp32 (entropy partials)
    size_t r_cnt;       // nb_topk * E int32
    size_t d_cnt;       // chunks * E int32
    size_t d_base;      // chunks * E int32
    size_t f_amaps;     // bf16 layers: the expert GEMMs' per-expert A maps (2 E tensor maps)
    size_t total;
};
WsLayout ws_layout(const moe_config& c);
constexpr size_t kTensorMapBytes = 128;  // one CUtensorMap

struct FwdLayout {
    WsLayout ws;        // scratch at offset 0
    size_t ids, w, counts, kept, offsets, perm, row_of, mean_prob, losses;
    size_t x_perm, h, y_perm;
    size_t sh_offsets, sh_h, sh_y;  // shared expert (when F_shared > 0)
    size_t total;
};
FwdLayout fwd_layout(const moe_config& c, int64_t max_rows);

// The training forward's state: the forward layout (its y_perm holds the
// unweighted expert outputs) plus what only the backward reads.
struct TrainLayout {
    FwdLayout f;
    size_t logits;      // (T, E) fp32: the logits the layer was routed on
    size_t gu;          // (max_rows, 2F) dtype: [g | u] pre-activations
    size_t sh_gu;       // (T, 2 F_shared) dtype
    size_t total;
};
TrainLayout train_layout(const moe_config& c, int64_t max_rows);

// The backward's scratch.
struct BwdLayout {
    size_t status;      // int32[64]
    size_t dyp;         // (max_rows, D): w_r * dY[t_r]
    size_t dw_row;      // (max_rows) fp32: gate-weight gradient of each row
    size_t dlogits;     // (T, E) fp32
    size_t dgu;         // (max_rows, 2F): [dg | du]
    size_t dxp;         // (max_rows, D)
    size_t rw_part;     // router weight-gradient partials
    size_t db_scratch;  // (E) fp32: the bias gradient when the caller wants none
    size_t sh_dgu;      // (T, 2 F_shared)
    size_t sh_dx;       // (T, D)
    size_t tmaps;       // the weight-gradient GEMMs' per-expert tensor maps (bf16 layers)
    size_t dmaps;       // the dgrad GEMMs' per-expert A maps (bf16 layers)
    size_t tmaps_sh;    // and the shared expert's
    int rw_splits;
    size_t total;
};
BwdLayout bwd_layout(const moe_config& c, int64_t max_rows);

int64_t capacity_of(const moe_config& c);
int64_t max_rows_of(const moe_config& c);

// Tensor-core router (router_tc.cu): bf16 layers with E <= 128 and T >= 2048.
// One kernel: logits, routing, and (when mean_prob or losses is given) the
// statistics, finished by the CTA that completes last.  It reads the router
// weight as its three exact bf16 terms (router_prepare_kernel).
bool router_tc_eligible(const moe_config& c);
int router_tc_blocks(const moe_config& c);
// CTAs per token tile (a cluster splitting d_model; 1: no split)
int router_tc_splits(const moe_config& c);
// Bytes of the weight terms, 3 x E16 x D bf16 (0: no tensor-core router for c).
size_t router_terms_bytes(const moe_config& c);
cudaError_t launch_router_prepare(const moe_config& c, const float* w_router, void* terms,
                                  cudaStream_t s);
cudaError_t launch_router_tc(const moe_config& c, const RouteOpts& o, const void* x,
                             const void* terms, const float* bias, const float* noise,
                             float* logits_out, float* probs_out, int32_t* ids, float* w,
                             float* blk_mp, float* blk_z, float* blk_ent, int32_t* blk_cnt,
                             float* mean_prob, float* losses, int* status, cudaStream_t s);

// ---------------------------------------------------------------- launches --
// Each returns cudaSuccess or the launch error.
// terms: the prepared router weight or null (the tensor-core router then
// prepares it in the workspace first).
cudaError_t launch_router(const moe_config& c, const RouterPlan& rp, const void* x,
                          const float* w_router, const void* terms, const float* bias,
                          const float* sel_bias,
                          const float* noise,
                          const float* logits_in, float* logits_out, float* probs_out,
                          int32_t* ids, float* w, float* mean_prob, float* losses, char* ws,
                          const WsLayout& L, cudaStream_t s);

cudaError_t launch_update_bias(int E, const int32_t* counts, float gamma, float* bias,
                               cudaStream_t s);

cudaError_t launch_dispatch_index(const moe_config& c, int64_t C, const int32_t* ids,
                                  int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* perm,
                                  int32_t* row_of, char* ws, const WsLayout& L, cudaStream_t s);

cudaError_t launch_gather(const moe_config& c, const void* x, const int32_t* row_of, void* x_perm,
                          int64_t max_rows, int* status, cudaStream_t s);

// slot_w (T, K) or null: when given, each slot's row is multiplied by its weight.
cudaError_t launch_combine(const moe_config& c, const void* y_perm, const int32_t* row_of,
                           const float* slot_w, const void* y_add, void* y, int64_t max_rows,
                           cudaStream_t s);

// Expert FFN: gate/up (+SwiGLU) into h, then down (+routing weight) into y_perm.
// The stage boundary between the two GEMMs is reported through `mid` (may be
// null): it is called after the gate/up launch.
typedef void (*StageHook)(void* ctx, cudaStream_t s);
// gu_keep (max_rows, 2F) or null: where the gate/up GEMM keeps [g | u] (bf16 only).
// amaps: null, or 2 E * kTensorMapBytes of device scratch, 128-byte aligned, where
// the bf16 GEMMs write each expert's A maps (rows past the expert's end then read
// as zeros instead of being fetched).
cudaError_t launch_expert_ffn(const moe_config& c, int64_t max_rows, const void* x_perm,
                              const int32_t* offsets, const int32_t* perm, const float* topk_w,
                              const void* w_gate, const void* w_up, const void* w_down, void* h,
                              void* y_perm, void* gu_keep, void* amaps, int* status, cudaStream_t s,
                              StageHook mid, void* mid_ctx);

// ---------------------------------------------------------------- backward --
// dH = dYp . Wd^T through SwiGLU into dgu = [dg | du], then dXp = dgu . [Wg | Wu]^T.
// amaps: null, or 2 E * kTensorMapBytes of device scratch (128-byte aligned) for
// each expert's A maps, as for the forward's expert GEMMs.
cudaError_t launch_dgrad_tc_bf16(const moe_config& c, int64_t max_rows, const void* dyp,
                                 const int32_t* offsets, const void* gu, const void* w_gate,
                                 const void* w_up, const void* w_down, void* dgu, void* dxp,
                                 void* amaps, int* status, cudaStream_t s, StageHook mid, void* mid_ctx);
// out0 / out1 (E, M, Nh) fp32 = A[block]^T . B[block] per expert block.
// `maps`: device scratch of wgrad_maps_bytes(E) bytes, 128-byte aligned,
// rewritten by the launch (each expert's operand tensor maps).
size_t wgrad_maps_bytes(int E);
cudaError_t launch_wgrad_tc_bf16(int E, int64_t max_rows, const int32_t* offsets, const void* A,
                                 int M, const void* B, int Nh, int halves, float* out0, float* out1,
                                 void* maps, int* status, cudaStream_t s);
cudaError_t launch_bwd_rows(const moe_config& c, const void* dy, const void* o, const int32_t* offsets,
                            const int32_t* perm, const float* topk_w, void* dyp, float* dw_row,
                            int64_t max_rows, int* status, cudaStream_t s);
cudaError_t launch_router_bwd(const moe_config& c, const float* logits, const int32_t* ids,
                              const int32_t* row_of, const float* dw_row, const int32_t* counts,
                              float c_bal, float c_z, float* dlogits, int64_t max_rows, int* status,
                              cudaStream_t s);
int router_wgrad_splits(const moe_config& c);
size_t router_wgrad_part_bytes(const moe_config& c, int splits);
cudaError_t launch_router_wgrad(const moe_config& c, const void* x, const float* dL, float* part,
                                int splits, float* dw, float* db, cudaStream_t s);
cudaError_t launch_ep_layout(const int32_t* recv, int W, int EL, int64_t max_rows, int32_t* offsets,
                             int32_t* seg_src, int32_t* seg_dst, int32_t* dst_of, int32_t* src_of,
                             int* status, cudaStream_t s);
cudaError_t launch_dgrad_simt_f32(const moe_config& c, int64_t max_rows, const void* dyp, const int32_t* offsets,
                                  const void* gu, const void* w_gate, const void* w_up, const void* w_down,
                                  void* dgu, void* dxp, int* status, cudaStream_t s, StageHook mid, void* mid_ctx);
cudaError_t launch_wgrad_simt_f32(int E, int64_t max_rows, const int32_t* offsets, const void* a, int M,
                                  const void* b, int N, int halves, float* out0, float* out1, int* status,
                                  cudaStream_t s);
cudaError_t launch_peer_dispatch(const moe_config& c, int rank, int W, const int32_t* kept_all, const void* x,
                                 const int32_t* ids, const int32_t* row_of, const int32_t* offsets,
                                 void* const* recv_bufs, int64_t recv_rows, int64_t max_rows,
                                 int32_t* local_offsets, int32_t* remote_row, int* status, cudaStream_t s);
cudaError_t launch_peer_combine(const moe_config& c, int W, const void* const* y_bufs, const int32_t* ids,
                                const int32_t* remote_row, const float* topk_w, int64_t recv_rows,
                                const void* y_add, void* y, int* status, cudaStream_t s);
cudaError_t launch_permute_rows(const void* in, const int32_t* idx, void* out, int64_t n, int64_t row_bytes,
                                int64_t in_rows, int* status, cudaStream_t s);
cudaError_t launch_dx_assemble(const moe_config& c, const float* dL, const float* w_r, const void* dxp,
                               const int32_t* row_of, const void* dx_shared, void* dx,
                               int64_t max_rows, cudaStream_t s);

}  // namespace moe
