// api.cu -- the extern "C" boundary of libmoe_b200.so (declared in moe.h):
// argument validation, workspace layout, and the launch sequence of each
// entry point.  No allocation, no host synchronisation (except the device
// status query).
#include <math.h>
#include <string.h>

#include "internal.h"

namespace moe {

cudaError_t launch_ffn_simt_f32(const moe_config& c, int64_t max_rows, const void* x_perm,
                                const int32_t* offsets, const int32_t* perm, const float* topk_w,
                                const void* w_gate, const void* w_up, const void* w_down, void* h,
                                void* y_perm, void* gu_keep, int* status, cudaStream_t s, StageHook mid,
                                void* mid_ctx);
cudaError_t launch_ffn_tc_bf16(const moe_config& c, int64_t max_rows, const void* x_perm,
                               const int32_t* offsets, const int32_t* perm, const float* topk_w,
                               const void* w_gate, const void* w_up, const void* w_down, void* h,
                               void* y_perm, void* gu_keep, void* amaps, int* status, cudaStream_t s,
                               StageHook mid, void* mid_ctx);

int64_t capacity_of(const moe_config& c)
{
    const int64_t tk = c.T * (int64_t)c.K;
    if (!(c.capacity_factor > 0.0f)) return tk;
    double v = ceil((double)c.capacity_factor * (double)c.T * (double)c.K / (double)c.E);
    if (v < 1.0) v = 1.0;
    if (v > (double)tk) v = (double)tk;  // no expert can receive more than T*K
    return (int64_t)v;
}

int64_t max_rows_of(const moe_config& c)
{
    const int64_t tk = c.T * (int64_t)c.K;
    const int64_t cap = capacity_of(c) * (int64_t)c.E;
    return cap < tk ? cap : tk;
}

WsLayout ws_layout(const moe_config& c)
{
    const RouterPlan rp = router_plan(c);
    const int64_t nch = dispatch_chunks(c);
    WsLayout L;
    size_t o = 0;
    L.status = o;
    o += align_up(64 * sizeof(int));
    L.r_part = o;
    // the SIMT router's (partial) logits per d_model split
    const size_t part_bytes = (size_t)rp.splits * (size_t)c.T * c.E * sizeof(float);
    o += align_up(part_bytes);
    L.r_terms = o;
    o += align_up(router_tc_eligible(c) ? router_terms_bytes(c) : 0);
    L.r_mp = o;
    o += align_up((size_t)rp.nb_topk * c.E * sizeof(float));
    L.r_z = o;
    o += align_up((size_t)rp.nb_topk * sizeof(float));
    L.r_ent = o;
    o += align_up((size_t)rp.nb_topk * sizeof(float));
    L.r_cnt = o;
    o += align_up((size_t)rp.nb_topk * c.E * sizeof(int32_t));
    L.d_cnt = o;
    o += align_up((size_t)nch * c.E * sizeof(int32_t));
    L.d_base = o;
    o += align_up((size_t)nch * c.E * sizeof(int32_t));
    L.f_amaps = o;
    o += c.dtype == MOE_BF16 ? align_up(2 * (size_t)c.E * kTensorMapBytes) : 0;
    L.total = o;
    return L;
}

FwdLayout fwd_layout(const moe_config& c, int64_t max_rows)
{
    FwdLayout F;
    F.ws = ws_layout(c);
    const size_t es = c.dtype == MOE_BF16 ? 2 : 4;
    const size_t tk = (size_t)c.T * c.K;
    size_t o = F.ws.total;
    F.ids = o;       o += align_up(tk * sizeof(int32_t));
    F.w = o;         o += align_up(tk * sizeof(float));
    F.counts = o;    o += align_up((size_t)c.E * sizeof(int32_t));
    F.kept = o;      o += align_up((size_t)c.E * sizeof(int32_t));
    F.offsets = o;   o += align_up((size_t)(c.E + 1) * sizeof(int32_t));
    F.perm = o;      o += align_up((size_t)max_rows * sizeof(int32_t));
    F.row_of = o;    o += align_up(tk * sizeof(int32_t));
    F.mean_prob = o; o += align_up((size_t)c.E * sizeof(float));
    F.losses = o;    o += align_up(3 * sizeof(float));
    F.x_perm = o;    o += align_up((size_t)max_rows * c.D * es);
    F.h = o;         o += align_up((size_t)max_rows * c.F * es);
    F.y_perm = o;    o += align_up((size_t)max_rows * c.D * es);
    F.sh_offsets = o; F.sh_h = o; F.sh_y = o;
    if (c.F_shared > 0) {
        F.sh_offsets = o; o += align_up(2 * sizeof(int32_t));
        F.sh_h = o;       o += align_up((size_t)c.T * c.F_shared * es);
        F.sh_y = o;       o += align_up((size_t)c.T * c.D * es);
    }
    F.total = o;
    return F;
}

TrainLayout train_layout(const moe_config& c, int64_t max_rows)
{
    TrainLayout L;
    L.f = fwd_layout(c, max_rows);
    const size_t es = c.dtype == MOE_BF16 ? 2 : 4;
    size_t o = L.f.total;
    L.logits = o; o += align_up((size_t)c.T * c.E * sizeof(float));
    L.gu = o;     o += align_up((size_t)max_rows * 2 * c.F * es);
    L.sh_gu = o;
    if (c.F_shared > 0) o += align_up((size_t)c.T * 2 * c.F_shared * es);
    L.total = o;
    return L;
}

BwdLayout bwd_layout(const moe_config& c, int64_t max_rows)
{
    BwdLayout B;
    const size_t es = c.dtype == MOE_BF16 ? 2 : 4;
    size_t o = 0;
    B.status = o;  o += align_up(64 * sizeof(int));
    B.dyp = o;     o += align_up((size_t)max_rows * c.D * es);
    B.dw_row = o;  o += align_up((size_t)max_rows * sizeof(float));
    B.dlogits = o; o += align_up((size_t)c.T * c.E * sizeof(float));
    B.dgu = o;     o += align_up((size_t)max_rows * 2 * c.F * es);
    B.dxp = o;     o += align_up((size_t)max_rows * c.D * es);
    B.rw_splits = router_wgrad_splits(c);
    B.rw_part = o; o += align_up(router_wgrad_part_bytes(c, B.rw_splits));
    B.db_scratch = o; o += align_up((size_t)c.E * sizeof(float));
    B.sh_dgu = o;  B.sh_dx = o;
    if (c.F_shared > 0) {
        B.sh_dgu = o; o += align_up((size_t)c.T * 2 * c.F_shared * es);
        B.sh_dx = o;  o += align_up((size_t)c.T * c.D * es);
    }
    // two launches (dWd, then [dWg | dWu]) of E experts each, one slot apiece
    B.tmaps = o;    o += c.dtype == MOE_BF16 ? 2 * align_up(wgrad_maps_bytes(c.E)) : 0;
    B.tmaps_sh = o; o += c.dtype == MOE_BF16 && c.F_shared > 0 ? 2 * align_up(wgrad_maps_bytes(1)) : 0;
    B.dmaps = o;    o += c.dtype == MOE_BF16 ? align_up(2 * (size_t)c.E * kTensorMapBytes) : 0;
    B.total = o;
    return B;
}

static moe_status check_config(const moe_config* c)
{
    if (c == nullptr) return MOE_ERR_ARG;
    if (c->T < 1 || c->D < 1 || c->F < 1 || c->E < 1) return MOE_ERR_SHAPE;
    if (c->E > 256) return MOE_ERR_ARG;
    if (c->K < 1 || c->K > c->E || c->K > 8) return MOE_ERR_ARG;
    if (c->T * (int64_t)c->K > (int64_t)INT32_MAX) return MOE_ERR_SHAPE;
    if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_ARG;
    if (c->score_func != MOE_SCORE_SOFTMAX && c->score_func != MOE_SCORE_SIGMOID)
        return MOE_ERR_UNSUPPORTED;
    if (c->renormalize != 0 && c->renormalize != 1) return MOE_ERR_ARG;
    if (c->n_groups < 0 || c->n_groups > 32) return MOE_ERR_ARG;
    if (c->n_groups > 1) {
        if (c->E % c->n_groups != 0) return MOE_ERR_ARG;
        if (c->topk_groups < 1 || c->topk_groups > c->n_groups) return MOE_ERR_ARG;
        if ((int64_t)c->topk_groups * (c->E / c->n_groups) < c->K) return MOE_ERR_ARG;
    }
    if (!(c->route_scale > 0.0f) || !isfinite(c->route_scale)) return MOE_ERR_ARG;
    if (c->F_shared < 0) return MOE_ERR_SHAPE;
    if (c->F_shared % 8 != 0) return MOE_ERR_ALIGN;
    if (c->D % 8 != 0 || c->F % 8 != 0) return MOE_ERR_ALIGN;
    if (!isfinite(c->capacity_factor)) return MOE_ERR_ARG;
    return MOE_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


// ------------------------------------------------------------- tracing --
static void* g_trace[16];
static int g_trace_n = 0;
static const char* kStageNames[8] = {"start",          "route",       "dispatch_index",
                                     "gather",         "expert_gate_up", "expert_down",
                                     "shared_expert",  "combine"};

static void trace(int boundary, cudaStream_t s)
{
    if (boundary < g_trace_n && g_trace[boundary] != nullptr)
        cudaEventRecord(static_cast<cudaEvent_t>(g_trace[boundary]), s);
}

static void trace_mid_ffn(void*, cudaStream_t s) { trace(4, s); }

static void* g_btrace[16];
static int g_btrace_n = 0;
static const char* kBwdStageNames[10] = {"start",      "rows",          "router_bwd",
                                         "dgrad_h",    "dgrad_x",       "wgrad_down",
                                         "wgrad_gate_up", "shared_expert", "router_wgrad", "dx"};

static void btrace(int boundary, cudaStream_t s)
{
    if (boundary < g_btrace_n && g_btrace[boundary] != nullptr)
        cudaEventRecord(static_cast<cudaEvent_t>(g_btrace[boundary]), s);
}

static void btrace_mid_dgrad(void*, cudaStream_t s) { btrace(3, s); }

// offsets {0, n} of a single expert block covering n rows
__global__ void set_row_range_kernel(int32_t* off, int32_t n)
{
    if (threadIdx.x == 0) {
        off[0] = 0;
        off[1] = n;
    }
}

cudaError_t launch_expert_ffn(const moe_config& c, int64_t max_rows, const void* x_perm,
                              const int32_t* offsets, const int32_t* perm, const float* topk_w,
                              const void* w_gate, const void* w_up, const void* w_down, void* h,
                              void* y_perm, void* gu_keep, void* amaps, int* status, cudaStream_t s,
                              StageHook mid, void* mid_ctx)
{
    if (c.dtype == MOE_F32)
        return launch_ffn_simt_f32(c, max_rows, x_perm, offsets, perm, topk_w, w_gate, w_up,
                                   w_down, h, y_perm, gu_keep, status, s, mid, mid_ctx);
    return launch_ffn_tc_bf16(c, max_rows, x_perm, offsets, perm, topk_w, w_gate, w_up, w_down, h,
                              y_perm, gu_keep, amaps, status, s, mid, mid_ctx);
}

// the backward's GEMMs in the layer's dtype: tensor cores for bf16, fp32 SIMT for fp32
static cudaError_t launch_dgrad(const moe_config& c, int64_t max_rows, const void* dyp, const int32_t* offsets,
                                const void* gu, const void* w_gate, const void* w_up, const void* w_down,
                                void* dgu, void* dxp, void* amaps, int* status, cudaStream_t s, StageHook mid,
                                void* mid_ctx)
{
    if (c.dtype == MOE_F32)
        return launch_dgrad_simt_f32(c, max_rows, dyp, offsets, gu, w_gate, w_up, w_down, dgu, dxp, status, s,
                                     mid, mid_ctx);
    return launch_dgrad_tc_bf16(c, max_rows, dyp, offsets, gu, w_gate, w_up, w_down, dgu, dxp, amaps, status, s,
                                mid, mid_ctx);
}

static cudaError_t launch_wgrad(int32_t dt, int E, int64_t max_rows, const int32_t* offsets, const void* a,
                                int M, const void* b, int N, int halves, float* out0, float* out1, void* maps,
                                int* status, cudaStream_t s)
{
    if (dt == MOE_F32)
        return launch_wgrad_simt_f32(E, max_rows, offsets, a, M, b, N, halves, out0, out1, status, s);
    return launch_wgrad_tc_bf16(E, max_rows, offsets, a, M, b, N, halves, out0, out1, maps, status, s);
}

// the shared expert as a layer of one expert over every token
static moe_config shared_config(const moe_config& c)
{
    moe_config cs = c;
    cs.E = 1;
    cs.K = 1;
    cs.F = c.F_shared;
    cs.capacity_factor = 0.f;
    cs.n_groups = 1;
    return cs;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int32_t st)
{
    switch (st) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_SHAPE: return "invalid shape";
        case MOE_ERR_UNSUPPORTED: return "unsupported option";
        case MOE_ERR_ALIGN: return "misaligned size or buffer";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case MOE_ERR_DEVICE_BOUNDS: return "device index out of range";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int32_t moe_version(void) { return 100; }

moe_status moe_check_config(const moe_config* cfg) { return check_config(cfg); }

moe_status moe_capacity(const moe_config* cfg, int64_t* capacity)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (capacity == nullptr) return MOE_ERR_ARG;
    *capacity = capacity_of(*cfg);
    return MOE_OK;
}

moe_status moe_max_rows(const moe_config* cfg, int64_t* rows)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (rows == nullptr) return MOE_ERR_ARG;
    *rows = max_rows_of(*cfg);
    return MOE_OK;
}

moe_status moe_workspace_size(const moe_config* cfg, size_t* bytes)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_ARG;
    *bytes = ws_layout(*cfg).total;
    return MOE_OK;
}

moe_status moe_forward_workspace_size(const moe_config* cfg, size_t* bytes)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_ARG;
    *bytes = fwd_layout(*cfg, max_rows_of(*cfg)).total;
    return MOE_OK;
}

static moe_status check_ws(const moe_config* cfg, const void* ws, size_t bytes, size_t need)
{
    (void)cfg;
    if (ws == nullptr || bytes < need) return MOE_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_ALIGN;
    return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const void* x, const float* w_router,
                     const void* w_router_terms, const float* router_bias,
                     const float* selection_bias, const float* logit_noise, const float* logits_in,
                     float* logits_out, float* probs_out, int32_t* topk_ids, float* topk_w,
                     float* mean_prob, float* losses, void* workspace, size_t workspace_bytes,
                     void* stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (topk_ids == nullptr || topk_w == nullptr) return MOE_ERR_ARG;
    if (logits_in == nullptr && (x == nullptr || w_router == nullptr)) return MOE_ERR_ARG;
    if (logits_in == nullptr && !aligned16(x)) return MOE_ERR_ALIGN;
    if (w_router_terms != nullptr && !aligned16(w_router_terms)) return MOE_ERR_ALIGN;
    const WsLayout L = ws_layout(*cfg);
    st = check_ws(cfg, workspace, workspace_bytes, L.total);
    if (st != MOE_OK) return st;
    const RouterPlan rp = router_plan(*cfg);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_router(*cfg, rp, x, w_router, w_router_terms, router_bias,
                                     selection_bias, logit_noise, logits_in,
                                     logits_out, probs_out, topk_ids, topk_w, mean_prob, losses,
                                     static_cast<char*>(workspace), L, s));
}

moe_status moe_router_terms_size(const moe_config* cfg, size_t* bytes)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_ARG;
    *bytes = router_terms_bytes(*cfg);
    return MOE_OK;
}

moe_status moe_router_prepare(const moe_config* cfg, const float* w_router, void* w_router_terms,
                              void* stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (router_terms_bytes(*cfg) == 0) return MOE_ERR_UNSUPPORTED;
    if (w_router == nullptr || w_router_terms == nullptr) return MOE_ERR_ARG;
    if (!aligned16(w_router_terms)) return MOE_ERR_ALIGN;
    return cuda_status(
        launch_router_prepare(*cfg, w_router, w_router_terms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch(const moe_config* cfg, const void* x, const int32_t* topk_ids,
                        int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* perm,
                        int32_t* row_of, void* x_perm, void* workspace, size_t workspace_bytes,
                        void* stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!topk_ids || !counts || !kept || !offsets || !perm || !row_of) return MOE_ERR_ARG;
    if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_ARG;
    if (x && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_ALIGN;
    const WsLayout L = ws_layout(*cfg);
    st = check_ws(cfg, workspace, workspace_bytes, L.total);
    if (st != MOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    cudaError_t e = launch_dispatch_index(*cfg, capacity_of(*cfg), topk_ids, counts, kept, offsets,
                                          perm, row_of, ws, L, s);
    if (e == cudaSuccess && x)
        e = launch_gather(*cfg, x, row_of, x_perm, max_rows_of(*cfg),
                          reinterpret_cast<int*>(ws + L.status), s);
    return cuda_status(e);
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                          const int32_t* perm, const float* topk_w, const void* w_gate,
                          const void* w_up, const void* w_down, void* h, void* y_perm,
                          void* workspace, size_t workspace_bytes, void* stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!x_perm || !offsets || !w_gate || !w_up || !w_down || !h || !y_perm) return MOE_ERR_ARG;
    if ((perm == nullptr) != (topk_w == nullptr)) return MOE_ERR_ARG;
    if (!aligned16(x_perm) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
        !aligned16(h) || !aligned16(y_perm))
        return MOE_ERR_ALIGN;
    const WsLayout L = ws_layout(*cfg);
    st = check_ws(cfg, workspace, workspace_bytes, L.total);
    if (st != MOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = reinterpret_cast<int*>(static_cast<char*>(workspace) + L.status);
    return cuda_status(launch_expert_ffn(*cfg, max_rows_of(*cfg), x_perm, offsets, perm, topk_w,
                                         w_gate, w_up, w_down, h, y_perm, nullptr,
                                         static_cast<char*>(workspace) + L.f_amaps, status, s,
                                         nullptr, nullptr));
}

moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* row_of,
                       const void* y_add, void* y, void* stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!y_perm || !row_of || !y) return MOE_ERR_ARG;
    if (!aligned16(y_perm) || !aligned16(y) || (y_add && !aligned16(y_add))) return MOE_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_combine(*cfg, y_perm, row_of, nullptr, y_add, y, max_rows_of(*cfg), s));
}

// The forward's launch sequence; with TL (training) the routed logits and
// [g | u] are kept, the down projection stores unweighted rows and the combine
// applies the weights, and the routing results stay in the state (copied to
// the caller's buffers when asked for).
static cudaError_t run_forward(const moe_config& c, const void* x, const float* w_router,
                               const void* w_terms, const float* router_bias,
                               const float* selection_bias, const float* logit_noise,
                               const void* w_gate, const void* w_up,
                               const void* w_down, const void* w_gate_shared,
                               const void* w_up_shared, const void* w_down_shared, void* y,
                               float* losses, float* mean_prob, int32_t* counts, int32_t* topk_ids,
                               float* topk_w, char* ws, const FwdLayout& F, const TrainLayout* TL,
                               cudaStream_t s)
{
    const int64_t max_rows = max_rows_of(c);
    const bool train = TL != nullptr;
    int* status = reinterpret_cast<int*>(ws + F.ws.status);
    int32_t* ids = (topk_ids && !train) ? topk_ids : reinterpret_cast<int32_t*>(ws + F.ids);
    float* w = (topk_w && !train) ? topk_w : reinterpret_cast<float*>(ws + F.w);
    int32_t* cnt = (counts && !train) ? counts : reinterpret_cast<int32_t*>(ws + F.counts);
    int32_t* kept = reinterpret_cast<int32_t*>(ws + F.kept);
    int32_t* offsets = reinterpret_cast<int32_t*>(ws + F.offsets);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + F.perm);
    int32_t* row_of = reinterpret_cast<int32_t*>(ws + F.row_of);
    void* x_perm = ws + F.x_perm;
    void* h = ws + F.h;
    void* y_perm = ws + F.y_perm;
    float* logits_keep = train ? reinterpret_cast<float*>(ws + TL->logits) : nullptr;

    trace(0, s);
    const RouterPlan rp = router_plan(c);
    cudaError_t e = launch_router(c, rp, x, w_router, w_terms, router_bias, selection_bias,
                                  logit_noise, nullptr, logits_keep, nullptr, ids, w, mean_prob, losses, ws,
                                  F.ws, s);
    trace(1, s);
    if (e == cudaSuccess)
        e = launch_dispatch_index(c, capacity_of(c), ids, cnt, kept, offsets, perm, row_of, ws,
                                  F.ws, s);
    trace(2, s);
    if (e == cudaSuccess) e = launch_gather(c, x, row_of, x_perm, max_rows, status, s);
    trace(3, s);
    if (e == cudaSuccess)
        e = launch_expert_ffn(c, max_rows, x_perm, offsets, train ? nullptr : perm,
                              train ? nullptr : w, w_gate, w_up, w_down, h, y_perm,
                              train ? ws + TL->gu : nullptr, ws + F.ws.f_amaps, status, s, trace_mid_ffn,
                              nullptr);
    trace(5, s);
    const void* y_add = nullptr;
    if (e == cudaSuccess && c.F_shared > 0) {
        // the shared expert: one expert over every token, rows = x, weight 1
        const moe_config cs = shared_config(c);
        int32_t* sh_off = reinterpret_cast<int32_t*>(ws + F.sh_offsets);
        set_row_range_kernel<<<1, 32, 0, s>>>(sh_off, (int32_t)c.T);
        e = cudaGetLastError();
        if (e == cudaSuccess)
            e = launch_expert_ffn(cs, c.T, x, sh_off, nullptr, nullptr, w_gate_shared, w_up_shared,
                                  w_down_shared, ws + F.sh_h, ws + F.sh_y,
                                  train ? ws + TL->sh_gu : nullptr, nullptr, status, s, nullptr, nullptr);
        y_add = ws + F.sh_y;
    }
    trace(6, s);
    if (e == cudaSuccess) e = launch_combine(c, y_perm, row_of, train ? w : nullptr, y_add, y, max_rows, s);
    trace(7, s);
    if (train && e == cudaSuccess) {  // the caller's copies of the routing results
        const size_t tk = (size_t)c.T * c.K;
        if (topk_ids) e = cudaMemcpyAsync(topk_ids, ids, tk * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess && topk_w)
            e = cudaMemcpyAsync(topk_w, w, tk * sizeof(float), cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess && counts)
            e = cudaMemcpyAsync(counts, cnt, (size_t)c.E * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    }
    return e;
}

static moe_status check_forward_args(const moe_config* cfg, const void* x, const float* w_router,
                                     const void* w_gate, const void* w_up, const void* w_down,
                                     const void* w_gate_shared, const void* w_up_shared,
                                     const void* w_down_shared, const void* y)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!x || !w_router || !w_gate || !w_up || !w_down || !y) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(w_gate) || !aligned16(w_up) ||
        !aligned16(w_down))
        return MOE_ERR_ALIGN;
    if (cfg->F_shared > 0) {
        if (!w_gate_shared || !w_up_shared || !w_down_shared) return MOE_ERR_ARG;
        if (!aligned16(w_gate_shared) || !aligned16(w_up_shared) || !aligned16(w_down_shared))
            return MOE_ERR_ALIGN;
    }
    return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const void* x, const float* w_router,
                       const void* w_router_terms, const float* router_bias,
                       const float* selection_bias, const float* logit_noise, const void* w_gate,
                       const void* w_up, const void* w_down, const void* w_gate_shared,
                       const void* w_up_shared, const void* w_down_shared, void* y, float* losses,
                       float* mean_prob, int32_t* counts, int32_t* topk_ids, float* topk_w,
                       void* workspace, size_t workspace_bytes, void* stream)
{
    moe_status st = check_forward_args(cfg, x, w_router, w_gate, w_up, w_down, w_gate_shared,
                                       w_up_shared, w_down_shared, y);
    if (st != MOE_OK) return st;
    if (w_router_terms != nullptr && !aligned16(w_router_terms)) return MOE_ERR_ALIGN;
    const FwdLayout F = fwd_layout(*cfg, max_rows_of(*cfg));
    st = check_ws(cfg, workspace, workspace_bytes, F.total);
    if (st != MOE_OK) return st;
    return cuda_status(run_forward(*cfg, x, w_router, w_router_terms, router_bias, selection_bias,
                                   logit_noise, w_gate, w_up, w_down, w_gate_shared, w_up_shared,
                                   w_down_shared, y, losses, mean_prob, counts, topk_ids, topk_w,
                                   static_cast<char*>(workspace), F, nullptr,
                                   static_cast<cudaStream_t>(stream)));
}

moe_status moe_train_state_size(const moe_config* cfg, size_t* bytes)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_ARG;
    *bytes = train_layout(*cfg, max_rows_of(*cfg)).total;
    return MOE_OK;
}

moe_status moe_forward_train(const moe_config* cfg, const void* x, const float* w_router,
                             const float* router_bias, const float* selection_bias,
                             const float* logit_noise, const void* w_gate, const void* w_up,
                             const void* w_down, const void* w_gate_shared, const void* w_up_shared,
                             const void* w_down_shared, void* y, float* losses, float* mean_prob,
                             int32_t* counts, int32_t* topk_ids, float* topk_w, void* state,
                             size_t state_bytes, void* stream)
{
    moe_status st = check_forward_args(cfg, x, w_router, w_gate, w_up, w_down, w_gate_shared,
                                       w_up_shared, w_down_shared, y);
    if (st != MOE_OK) return st;
    const TrainLayout TL = train_layout(*cfg, max_rows_of(*cfg));
    st = check_ws(cfg, state, state_bytes, TL.total);
    if (st != MOE_OK) return st;
    // the training forward splits the router weight itself (it changes every step)
    return cuda_status(run_forward(*cfg, x, w_router, nullptr, router_bias, selection_bias,
                                   logit_noise, w_gate, w_up, w_down, w_gate_shared, w_up_shared,
                                   w_down_shared, y, losses, mean_prob, counts, topk_ids, topk_w,
                                   static_cast<char*>(state), TL.f, &TL,
                                   static_cast<cudaStream_t>(stream)));
}

moe_status moe_backward_workspace_size(const moe_config* cfg, size_t* bytes)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_ARG;
    *bytes = bwd_layout(*cfg, max_rows_of(*cfg)).total;
    return MOE_OK;
}

moe_status moe_backward(const moe_config* cfg, const void* x, const float* w_router,
                        const void* w_gate, const void* w_up, const void* w_down,
                        const void* w_gate_shared, const void* w_up_shared,
                        const void* w_down_shared, const void* state, size_t state_bytes,
                        const void* dy, float c_balance, float c_z, void* dx, float* dw_router,
                        float* db_router, float* dw_gate, float* dw_up, float* dw_down,
                        float* dw_gate_shared, float* dw_up_shared, float* dw_down_shared,
                        void* workspace, size_t workspace_bytes, void* stream)
{
    moe_status st = check_forward_args(cfg, x, w_router, w_gate, w_up, w_down, w_gate_shared,
                                       w_up_shared, w_down_shared, dx);
    if (st != MOE_OK) return st;
    if (!dy || !dw_router || !dw_gate || !dw_up || !dw_down) return MOE_ERR_ARG;
    if (!aligned16(dy) || !aligned16(dw_gate) || !aligned16(dw_up) || !aligned16(dw_down))
        return MOE_ERR_ALIGN;
    if (cfg->F_shared > 0) {
        if (!dw_gate_shared || !dw_up_shared || !dw_down_shared) return MOE_ERR_ARG;
        if (!aligned16(dw_gate_shared) || !aligned16(dw_up_shared) || !aligned16(dw_down_shared))
            return MOE_ERR_ALIGN;
    }
    if (!isfinite(c_balance) || !isfinite(c_z)) return MOE_ERR_ARG;
    const moe_config& c = *cfg;
    const int64_t max_rows = max_rows_of(c);
    const TrainLayout TL = train_layout(c, max_rows);
    st = check_ws(cfg, state, state_bytes, TL.total);
    if (st != MOE_OK) return st;
    const BwdLayout B = bwd_layout(c, max_rows);
    st = check_ws(cfg, workspace, workspace_bytes, B.total);
    if (st != MOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const char* sv = static_cast<const char*>(state);
    char* ws = static_cast<char*>(workspace);
    const FwdLayout& F = TL.f;
    int* status = reinterpret_cast<int*>(ws + B.status);
    const int32_t* ids = reinterpret_cast<const int32_t*>(sv + F.ids);
    const float* w = reinterpret_cast<const float*>(sv + F.w);
    const int32_t* cnt = reinterpret_cast<const int32_t*>(sv + F.counts);
    const int32_t* offsets = reinterpret_cast<const int32_t*>(sv + F.offsets);
    const int32_t* perm = reinterpret_cast<const int32_t*>(sv + F.perm);
    const int32_t* row_of = reinterpret_cast<const int32_t*>(sv + F.row_of);
    const float* logits = reinterpret_cast<const float*>(sv + TL.logits);
    float* dw_row = reinterpret_cast<float*>(ws + B.dw_row);
    float* dlogits = reinterpret_cast<float*>(ws + B.dlogits);

    btrace(0, s);
    cudaError_t e = launch_bwd_rows(c, dy, sv + F.y_perm, offsets, perm, w, ws + B.dyp, dw_row,
                                    max_rows, status, s);
    btrace(1, s);
    if (e == cudaSuccess)
        e = launch_router_bwd(c, logits, ids, row_of, dw_row, cnt, c_balance, c_z, dlogits,
                              max_rows, status, s);
    btrace(2, s);
    if (e == cudaSuccess)  // dH -> [dg | du], then dXp (boundary 3 between the two)
        e = launch_dgrad(c, max_rows, ws + B.dyp, offsets, sv + TL.gu, w_gate, w_up, w_down,
                         ws + B.dgu, ws + B.dxp, ws + B.dmaps, status, s, btrace_mid_dgrad, nullptr);
    btrace(4, s);
    if (e == cudaSuccess)  // dWd = h^T dYp
        e = launch_wgrad(c.dtype, c.E, max_rows, offsets, sv + F.h, c.F, ws + B.dyp, c.D, 1, dw_down,
                         nullptr, ws + B.tmaps, status, s);
    btrace(5, s);
    if (e == cudaSuccess)  // [dWg | dWu] = x_perm^T [dg | du]
        e = launch_wgrad(c.dtype, c.E, max_rows, offsets, sv + F.x_perm, c.D, ws + B.dgu, c.F, 2,
                         dw_gate, dw_up, ws + B.tmaps + align_up(wgrad_maps_bytes(c.E)), status, s);
    btrace(6, s);
    const void* dx_shared = nullptr;
    if (e == cudaSuccess && c.F_shared > 0) {
        const moe_config cs = shared_config(c);
        const int32_t* sh_off = reinterpret_cast<const int32_t*>(sv + F.sh_offsets);
        e = launch_dgrad(cs, c.T, dy, sh_off, sv + TL.sh_gu, w_gate_shared, w_up_shared,
                         w_down_shared, ws + B.sh_dgu, ws + B.sh_dx, nullptr, status, s, nullptr,
                         nullptr);
        if (e == cudaSuccess)
            e = launch_wgrad(c.dtype, 1, c.T, sh_off, sv + F.sh_h, c.F_shared, dy, c.D, 1,
                             dw_down_shared, nullptr, ws + B.tmaps_sh, status, s);
        if (e == cudaSuccess)
            e = launch_wgrad(c.dtype, 1, c.T, sh_off, x, c.D, ws + B.sh_dgu, c.F_shared, 2,
                             dw_gate_shared, dw_up_shared, ws + B.tmaps_sh + align_up(wgrad_maps_bytes(1)),
                             status, s);
        dx_shared = ws + B.sh_dx;
    }
    btrace(7, s);
    if (e == cudaSuccess)
        e = launch_router_wgrad(c, x, dlogits, reinterpret_cast<float*>(ws + B.rw_part), B.rw_splits,
                                dw_router,
                                db_router ? db_router : reinterpret_cast<float*>(ws + B.db_scratch), s);
    btrace(8, s);
    if (e == cudaSuccess)
        e = launch_dx_assemble(c, dlogits, w_router, ws + B.dxp, row_of, dx_shared, dx, max_rows, s);
    btrace(9, s);
    return cuda_status(e);
}

moe_status moe_update_selection_bias(const moe_config* cfg, const int32_t* counts, float gamma,
                                     float* selection_bias, void* stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!counts || !selection_bias) return MOE_ERR_ARG;
    if (!isfinite(gamma)) return MOE_ERR_ARG;
    return cuda_status(launch_update_bias(cfg->E, counts, gamma, selection_bias,
                                          static_cast<cudaStream_t>(stream)));
}

moe_status moe_get_device_status(const void* workspace, void* stream, int32_t* flags)
{
    if (workspace == nullptr || flags == nullptr) return MOE_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t word[2] = {0, 0};
    cudaError_t e = cudaMemcpyAsync(word, workspace, sizeof word, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    *flags = word[0];
    if (word[0] & MOE_DEVFLAG_TIMEOUT) return MOE_ERR_DEVICE_TIMEOUT;
    if (word[0] & MOE_DEVFLAG_BOUNDS) return MOE_ERR_DEVICE_BOUNDS;
    return MOE_OK;
}

moe_status moe_clear_device_status(void* workspace, void* stream)
{
    if (workspace == nullptr) return MOE_ERR_ARG;
    return cuda_status(
        cudaMemsetAsync(workspace, 0, 64 * sizeof(int), static_cast<cudaStream_t>(stream)));
}

int32_t moe_forward_kernel_count(const moe_config* cfg, int32_t router_terms_given)
{
    if (check_config(cfg) != MOE_OK) return 0;
    const int shared = cfg->F_shared > 0 ? 3 : 0;  // row offsets + two GEMMs
    // dispatch 1 (one cooperative kernel; 3 for more chunks than resident blocks),
    // gather 1, expert GEMMs 2, combine 1; router: the tensor-core kernel (after
    // the weight split when the caller passes no prepared terms), or the SIMT
    // logits (+ their split sum) and the top-k kernel
    // (bf16: and the kernel that writes the experts' A maps before the GEMMs)
    const int rest = 5 + (cfg->dtype == MOE_BF16 ? 1 : 0) + (dispatch_index_fused(*cfg) ? 0 : 2) + shared;
    if (router_tc_eligible(*cfg)) return (router_terms_given ? 1 : 2) + rest;
    return 2 + (router_plan(*cfg).splits > kTopkMaxSplits ? 1 : 0) + rest;
}

moe_status moe_ep_workspace_size(int32_t world, int32_t experts_per_rank, size_t* bytes)
{
    if (bytes == nullptr || world < 1 || experts_per_rank < 1 || world * experts_per_rank > 256)
        return MOE_ERR_ARG;
    *bytes = align_up(64 * sizeof(int)) + align_up((size_t)(2 * world * experts_per_rank + 1) * sizeof(int32_t));
    return MOE_OK;
}

moe_status moe_ep_layout(int32_t world, int32_t experts_per_rank, const int32_t* recv_counts,
                         int64_t max_rows, int32_t* offsets, int32_t* dst_of, int32_t* src_of,
                         void* workspace, size_t workspace_bytes, void* stream)
{
    size_t need = 0;
    moe_status st = moe_ep_workspace_size(world, experts_per_rank, &need);
    if (st != MOE_OK) return st;
    if (!recv_counts || !offsets || !dst_of || !src_of) return MOE_ERR_ARG;
    if (max_rows < 1 || max_rows > (int64_t)INT32_MAX) return MOE_ERR_SHAPE;
    st = check_ws(nullptr, workspace, workspace_bytes, need);
    if (st != MOE_OK) return st;
    char* ws = static_cast<char*>(workspace);
    int32_t* seg = reinterpret_cast<int32_t*>(ws + align_up(64 * sizeof(int)));
    const int n = world * experts_per_rank;
    return cuda_status(launch_ep_layout(recv_counts, world, experts_per_rank, max_rows, offsets, seg + n,
                                        seg, dst_of, src_of, reinterpret_cast<int*>(ws),
                                        static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_rows(const void* in, int64_t in_rows, const int32_t* idx, int64_t n,
                            int64_t row_bytes, void* out, void* workspace, void* stream)
{
    if (n < 0 || in_rows < 0 || row_bytes < 16) return MOE_ERR_SHAPE;
    if (row_bytes % 16 != 0) return MOE_ERR_ALIGN;
    if (n > 0 && (!in || !idx || !out)) return MOE_ERR_ARG;
    if (n > 0 && (!aligned16(in) || !aligned16(out))) return MOE_ERR_ALIGN;
    if (workspace == nullptr) return MOE_ERR_WORKSPACE;
    return cuda_status(launch_permute_rows(in, idx, out, n, row_bytes, in_rows,
                                           static_cast<int*>(workspace), static_cast<cudaStream_t>(stream)));
}

moe_status moe_combine_weighted(const moe_config* cfg, const void* y_perm, const int32_t* row_of,
                                const float* topk_w, const void* y_add, void* y, void* stream)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!y_perm || !row_of || !topk_w || !y) return MOE_ERR_ARG;
    if (!aligned16(y_perm) || !aligned16(y) || (y_add && !aligned16(y_add))) return MOE_ERR_ALIGN;
    return cuda_status(launch_combine(*cfg, y_perm, row_of, topk_w, y_add, y, max_rows_of(*cfg),
                                      static_cast<cudaStream_t>(stream)));
}

moe_status moe_ipc_alloc(size_t bytes, void** ptr, void* handle)
{
    static_assert(sizeof(cudaIpcMemHandle_t) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
    if (ptr == nullptr || handle == nullptr || bytes == 0) return MOE_ERR_ARG;
    *ptr = nullptr;
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    e = cudaIpcGetMemHandle(&h, p);
    if (e != cudaSuccess) {
        cudaFree(p);
        return MOE_ERR_CUDA;
    }
    memcpy(handle, &h, sizeof h);
    *ptr = p;
    return MOE_OK;
}

moe_status moe_ipc_free(void* ptr)
{
    if (ptr == nullptr) return MOE_OK;
    return cuda_status(cudaFree(ptr));
}

moe_status moe_ipc_open(const void* handle, void** ptr)
{
    if (ptr == nullptr || handle == nullptr) return MOE_ERR_ARG;
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof h);
    void* p = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    *ptr = p;
    return MOE_OK;
}

moe_status moe_ipc_close(void* ptr)
{
    if (ptr == nullptr) return MOE_OK;
    return cuda_status(cudaIpcCloseMemHandle(ptr));
}

static moe_status check_peer_args(const moe_config* cfg, int32_t world, int64_t recv_rows, const void* ws,
                                  size_t ws_bytes)
{
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (world < 1 || world > 64 || cfg->E % world != 0) return MOE_ERR_ARG;
    if (recv_rows < 1 || recv_rows > (int64_t)INT32_MAX) return MOE_ERR_SHAPE;
    size_t need = 0;
    st = moe_ep_workspace_size(world, cfg->E / world, &need);
    if (st != MOE_OK) return st;
    return check_ws(nullptr, ws, ws_bytes, need);
}

moe_status moe_ep_peer_dispatch(const moe_config* cfg, int32_t rank, int32_t world, const int32_t* kept_all,
                                const void* x, const int32_t* topk_ids, const int32_t* row_of,
                                const int32_t* offsets, void* const* recv_bufs, int64_t recv_rows,
                                int32_t* local_offsets, int32_t* remote_row, void* workspace,
                                size_t workspace_bytes, void* stream)
{
    moe_status st = check_peer_args(cfg, world, recv_rows, workspace, workspace_bytes);
    if (st != MOE_OK) return st;
    if (rank < 0 || rank >= world) return MOE_ERR_ARG;
    if (!kept_all || !x || !topk_ids || !row_of || !offsets || !recv_bufs || !local_offsets || !remote_row)
        return MOE_ERR_ARG;
    if (!aligned16(x)) return MOE_ERR_ALIGN;
    return cuda_status(launch_peer_dispatch(*cfg, rank, world, kept_all, x, topk_ids, row_of, offsets,
                                            recv_bufs, recv_rows, max_rows_of(*cfg), local_offsets,
                                            remote_row, static_cast<int*>(workspace),
                                            static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_peer_combine(const moe_config* cfg, int32_t world, const int32_t* topk_ids,
                               const int32_t* remote_row, const float* topk_w, const void* const* y_bufs,
                               int64_t recv_rows, const void* y_add, void* y, void* workspace,
                               size_t workspace_bytes, void* stream)
{
    moe_status st = check_peer_args(cfg, world, recv_rows, workspace, workspace_bytes);
    if (st != MOE_OK) return st;
    if (!topk_ids || !remote_row || !topk_w || !y_bufs || !y) return MOE_ERR_ARG;
    if (!aligned16(y) || (y_add && !aligned16(y_add))) return MOE_ERR_ALIGN;
    return cuda_status(launch_peer_combine(*cfg, world, y_bufs, topk_ids, remote_row, topk_w, recv_rows, y_add,
                                           y, static_cast<int*>(workspace), static_cast<cudaStream_t>(stream)));
}

int32_t moe_backward_kernel_count(const moe_config* cfg)
{
    if (check_config(cfg) != MOE_OK) return 0;
    // rows, router, two dgrad GEMMs, two wgrad GEMMs, router weight partials,
    // their sum, the bias gradient, dx; the shared expert adds its two dgrad
    // and two wgrad GEMMs.  In bf16 layers each wgrad GEMM is preceded by the
    // kernel that writes its experts' operand maps, and the dgrad GEMMs by one
    // that writes their experts' A maps.
    const int maps = cfg->dtype == MOE_BF16 ? 1 : 0;
    return 10 + 3 * maps + (cfg->F_shared > 0 ? 4 + 2 * maps : 0);
}

moe_status moe_trace_attach_backward(void* const* events, int32_t n_events)
{
    if (n_events < 0 || n_events > 16 || (n_events > 0 && events == nullptr)) return MOE_ERR_ARG;
    for (int i = 0; i < 16; ++i) g_btrace[i] = i < n_events ? events[i] : nullptr;
    g_btrace_n = n_events;
    return MOE_OK;
}

int32_t moe_trace_backward_boundary_count(void) { return 10; }

const char* moe_trace_backward_stage_name(int32_t boundary)
{
    if (boundary < 0 || boundary >= 10) return "";
    return kBwdStageNames[boundary];
}

moe_status moe_trace_attach(void* const* events, int32_t n_events)
{
    if (n_events < 0 || n_events > 16 || (n_events > 0 && events == nullptr)) return MOE_ERR_ARG;
    for (int i = 0; i < 16; ++i) g_trace[i] = i < n_events ? events[i] : nullptr;
    g_trace_n = n_events;
    return MOE_OK;
}

int32_t moe_trace_boundary_count(void) { return 8; }

const char* moe_trace_stage_name(int32_t boundary)
{
    if (boundary < 0 || boundary >= 8) return "";
    return kStageNames[boundary];
}

}  // extern "C"
