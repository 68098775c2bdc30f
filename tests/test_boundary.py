"""The C ABI library loads, exports every symbol include/moe.h declares, and
rejects bad arguments on the host before any device work (no GPU needed)."""
import ctypes

import pytest

from mixture_experts_layer_55_b200 import build as build_mod
from mixture_experts_layer_55_b200 import _binding as B


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def test_exports_every_declared_symbol(lib):
    names = B.header_symbols()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moe.h but not exported"
    assert set(B._SIG) == set(names), "binding signatures out of sync with moe.h"
    assert lib.moe_version() == 100


def _cfg(**kw):
    base = dict(T=64, D=128, F=256, E=8, K=2, dtype="bf16", capacity_factor=0.0)
    base.update(kw)
    return B.MoeConfig.make(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(), B.MOE_OK),
    (dict(K=0), B.MOE_ERR_ARG),
    (dict(K=9, E=16), B.MOE_ERR_ARG),       # register top-k bound
    (dict(K=5, E=4), B.MOE_ERR_ARG),        # K > E
    (dict(E=257, K=2), B.MOE_ERR_ARG),
    (dict(T=0), B.MOE_ERR_SHAPE),
    (dict(D=0), B.MOE_ERR_SHAPE),
    (dict(F=-8), B.MOE_ERR_SHAPE),
    (dict(D=100), B.MOE_ERR_ALIGN),         # 16-byte rows
    (dict(F=12), B.MOE_ERR_ALIGN),
    (dict(T=2**31, K=2), B.MOE_ERR_SHAPE),  # T*K beyond int32
    (dict(score_func="sigmoid"), B.MOE_OK),
    (dict(renormalize=False), B.MOE_OK),
    (dict(score_func=2), B.MOE_ERR_UNSUPPORTED),
    (dict(renormalize=2), B.MOE_OK),            # make() maps any truthy value to 1
    (dict(capacity_factor=float("nan")), B.MOE_ERR_ARG),
    (dict(n_groups=4, topk_groups=2), B.MOE_OK),  # E = 8: groups of 2, 4 eligible >= K
    (dict(n_groups=3, topk_groups=1), B.MOE_ERR_ARG),   # E not divisible
    (dict(n_groups=4, topk_groups=0), B.MOE_ERR_ARG),
    (dict(n_groups=4, topk_groups=5), B.MOE_ERR_ARG),
    (dict(n_groups=8, topk_groups=1), B.MOE_ERR_ARG),   # 1 eligible expert < K = 2
    (dict(n_groups=33, topk_groups=1, E=66), B.MOE_ERR_ARG),
    (dict(route_scale=0.0), B.MOE_ERR_ARG),
    (dict(route_scale=float("inf")), B.MOE_ERR_ARG),
    (dict(F_shared=64), B.MOE_OK),
    (dict(F_shared=60), B.MOE_ERR_ALIGN),
    (dict(F_shared=-8), B.MOE_ERR_SHAPE),
])
def test_check_config(lib, kw, code):
    assert B.check_config(_cfg(**kw)) == code


def test_capacity_and_rows(lib):
    c = _cfg(T=32768, D=1024, F=4096, E=32, K=2, capacity_factor=1.25)
    assert B.capacity(c) == 2560
    assert B.max_rows(c) == min(32768 * 2, 2560 * 32)
    c = _cfg(T=4096, E=16, K=2, capacity_factor=1.5)
    assert B.capacity(c) == 768
    c = _cfg(T=100, E=8, K=2)  # dropless
    assert B.capacity(c) == 200 and B.max_rows(c) == 200
    c = _cfg(T=3, E=8, K=1, capacity_factor=0.5)
    assert B.capacity(c) == 1 and B.max_rows(c) == 3
    c = _cfg(T=10, E=2, K=1, capacity_factor=100.0)  # never above T*K
    assert B.capacity(c) == 10


def test_workspace_sizes_grow_with_problem(lib):
    small = B.workspace_size(_cfg(T=64))
    big = B.workspace_size(_cfg(T=65536))
    assert 0 < small < big
    fwd = B.forward_workspace_size(_cfg(T=64))
    assert fwd > small


FAKE = 0x10000  # an aligned address the library never dereferences here


def _call_route(lib, cfg, x=FAKE, w=FAKE, ids=FAKE, tw=FAKE, ws=FAKE, nbytes=None, terms=None):
    nb = B.workspace_size(cfg) if nbytes is None else nbytes
    return lib.moe_route(ctypes.byref(cfg), x, w, terms, None, None, None, None, None, None, ids,
                         tw, None, None, ws, nb, None)


def test_route_argument_errors(lib):
    c = _cfg()
    assert _call_route(lib, c, ids=None) == B.MOE_ERR_ARG
    assert _call_route(lib, c, tw=None) == B.MOE_ERR_ARG
    assert _call_route(lib, c, x=None) == B.MOE_ERR_ARG
    assert _call_route(lib, c, x=FAKE + 8) == B.MOE_ERR_ALIGN
    assert _call_route(lib, c, terms=FAKE + 8) == B.MOE_ERR_ALIGN
    assert _call_route(lib, c, ws=None) == B.MOE_ERR_WORKSPACE
    assert _call_route(lib, c, nbytes=16) == B.MOE_ERR_WORKSPACE
    assert _call_route(lib, c, ws=FAKE + 16) == B.MOE_ERR_ALIGN  # workspace wants 256 B
    bad = _cfg(K=9, E=8)
    assert _call_route(lib, bad, nbytes=1 << 20) == B.MOE_ERR_ARG


def test_dispatch_ffn_combine_forward_argument_errors(lib):
    c = _cfg()
    nb = B.workspace_size(c)
    cr = ctypes.byref(c)
    # x and x_perm must be both given or both NULL
    assert lib.moe_dispatch(cr, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, nb,
                            None) == B.MOE_ERR_ARG
    assert lib.moe_dispatch(cr, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, nb,
                            None) == B.MOE_ERR_ARG
    assert lib.moe_dispatch(cr, FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, nb,
                            None) == B.MOE_ERR_ALIGN
    assert lib.moe_expert_ffn(cr, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, nb,
                              None) == B.MOE_ERR_ARG
    assert lib.moe_expert_ffn(cr, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, FAKE, FAKE,
                              nb, None) == B.MOE_ERR_ALIGN
    assert lib.moe_combine(cr, FAKE, None, None, FAKE, None) == B.MOE_ERR_ARG
    assert lib.moe_combine(cr, FAKE, FAKE, None, FAKE + 8, None) == B.MOE_ERR_ALIGN
    assert lib.moe_combine(cr, FAKE, FAKE, FAKE + 4, FAKE, None) == B.MOE_ERR_ALIGN
    # perm and topk_w: both given, or both NULL (unit weights)
    assert lib.moe_expert_ffn(cr, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, nb,
                              None) == B.MOE_ERR_ARG
    fb = B.forward_workspace_size(c)
    assert lib.moe_forward(cr, FAKE, FAKE, None, None, None, None, FAKE, FAKE, FAKE, None, None,
                           None, FAKE, None, None, None, None, None, FAKE, fb - 1,
                           None) == B.MOE_ERR_WORKSPACE
    assert lib.moe_forward(cr, FAKE, None, None, None, None, None, FAKE, FAKE, FAKE, None, None,
                           None, FAKE, None, None, None, None, None, FAKE, fb, None) == B.MOE_ERR_ARG
    assert lib.moe_forward(cr, FAKE, FAKE, FAKE + 8, None, None, None, FAKE, FAKE, FAKE, None,
                           None, None, FAKE, None, None, None, None, None, FAKE, fb,
                           None) == B.MOE_ERR_ALIGN
    # a shared expert needs its three weights
    cs = _cfg(F_shared=64)
    fbs = B.forward_workspace_size(cs)
    assert fbs > fb
    assert lib.moe_forward(ctypes.byref(cs), FAKE, FAKE, None, None, None, None, FAKE, FAKE, FAKE,
                           FAKE, None, FAKE, FAKE, None, None, None, None, None, FAKE, fbs,
                           None) == B.MOE_ERR_ARG
    assert lib.moe_update_selection_bias(cr, None, ctypes.c_float(0.01), FAKE, None) == B.MOE_ERR_ARG
    assert lib.moe_update_selection_bias(cr, FAKE, ctypes.c_float(float("nan")), FAKE,
                                         None) == B.MOE_ERR_ARG


def test_selftest_argument_errors(lib):
    assert lib.moe_selftest_wait_timeout(None, 256, 10_000, None) == B.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_wait_timeout(FAKE, 16, 10_000, None) == B.MOE_ERR_WORKSPACE
    assert lib.moe_selftest_wait_timeout(FAKE + 16, 256, 10_000, None) == B.MOE_ERR_ALIGN
    assert lib.moe_selftest_wait_timeout(FAKE, 256, 10, None) == B.MOE_ERR_ARG
    assert lib.moe_selftest_wait_timeout(FAKE, 256, 5_000_000_000, None) == B.MOE_ERR_ARG


def test_forward_kernel_count(lib):
    # dispatch 1 (one cooperative kernel), gather 1, expert GEMMs 2, combine 1, and the
    # router: SIMT logits GEMM + top-k (the top-k kernel finishes the statistics)
    assert B.forward_kernel_count(_cfg(T=512, D=256, F=512, E=8, K=2, dtype="f32")) == 7
    # tensor-core router: one kernel for routing and statistics, with or without the
    # d_model split (64 tiles of 128 tokens: a cluster of 2 CTAs per tile), after the
    # weight split unless the caller passes prepared terms; bf16 layers also write the
    # experts' A maps before the GEMMs (one kernel)
    assert B.forward_kernel_count(_cfg(T=16384, D=2048, F=1408, E=16, K=2), True) == 7
    assert B.forward_kernel_count(_cfg(T=16384, D=2048, F=1408, E=64, K=6), True) == 7
    assert B.forward_kernel_count(_cfg(T=8192, D=4096, F=14336, E=8, K=2), True) == 7
    assert B.forward_kernel_count(_cfg(T=8192, D=4096, F=14336, E=8, K=2)) == 8
    assert B.forward_kernel_count(_cfg(T=128, D=7168, F=2048, E=256, K=8)) == 9  # split SIMT router
    assert B.forward_kernel_count(_cfg(T=128, D=7168, F=2048, E=256, K=8), True) == 9
    assert B.forward_kernel_count(_cfg(K=0)) == 0
    assert B.forward_kernel_count(_cfg(T=8192, D=4096, F=14336, E=8, K=2, F_shared=256), True) == 10
    # more chunks of 2048 assignments than SMs: the three-kernel index pass
    assert B.forward_kernel_count(_cfg(T=160000, D=256, F=256, E=8, K=2), True) == 9


def test_router_terms_size_and_prepare_checks(lib):
    # 3 terms x E rounded up to 16/32/64/128 x D bf16 for bf16 layers with E <= 128
    assert B.router_terms_size(_cfg(T=8192, D=4096, F=14336, E=8, K=2)) == 3 * 16 * 4096 * 2
    assert B.router_terms_size(_cfg(T=16384, D=2048, F=1408, E=64, K=6)) == 3 * 64 * 2048 * 2
    assert B.router_terms_size(_cfg(T=64, D=256, F=256, E=100, K=2)) == 3 * 128 * 256 * 2
    assert B.router_terms_size(_cfg(T=128, D=7168, F=2048, E=256, K=8)) == 0
    assert B.router_terms_size(_cfg(T=512, D=256, F=512, E=8, K=2, dtype="f32")) == 0
    c = ctypes.byref(_cfg(T=8192, D=4096, F=14336, E=8, K=2))
    assert lib.moe_router_prepare(c, FAKE, None, None) == B.MOE_ERR_ARG
    assert lib.moe_router_prepare(c, None, FAKE, None) == B.MOE_ERR_ARG
    assert lib.moe_router_prepare(c, FAKE, FAKE + 8, None) == B.MOE_ERR_ALIGN
    c32 = ctypes.byref(_cfg(T=512, D=256, F=512, E=8, K=2, dtype="f32"))
    assert lib.moe_router_prepare(c32, FAKE, FAKE, None) == B.MOE_ERR_UNSUPPORTED
    bad = ctypes.byref(_cfg(K=0))
    assert lib.moe_router_prepare(bad, FAKE, FAKE, None) != B.MOE_OK


def test_status_strings_and_trace_table(lib):
    assert B.status_string(0) == "ok"
    assert "workspace" in B.status_string(B.MOE_ERR_WORKSPACE)
    names = B.trace_stage_names()
    assert names[0] == "start" and names[-1] == "combine" and len(names) == 8
    assert "shared_expert" in names
    assert lib.moe_trace_attach(None, 0) == B.MOE_OK
    assert lib.moe_trace_attach(None, 3) == B.MOE_ERR_ARG
    assert lib.moe_trace_attach(None, 17) == B.MOE_ERR_ARG


def test_backward_sizes_counts_and_trace(lib):
    c = _cfg(T=1200, D=256, F=384, E=4, K=2)
    assert B.train_state_size(c) > B.forward_workspace_size(c)
    assert B.backward_workspace_size(c) > 0
    # bf16: each weight-gradient GEMM is preceded by its operand-map kernel, and the
    # dgrad GEMMs by one that writes their experts' A maps
    assert B.backward_kernel_count(c) == 13
    assert B.backward_kernel_count(_cfg(T=600, F=320, F_shared=192, capacity_factor=1.0)) == 19
    cf = _cfg(dtype="f32")  # fp32 layers: SIMT GEMMs, no tensor maps
    assert B.backward_kernel_count(cf) == 10
    assert B.train_state_size(cf) > B.train_state_size(_cfg())  # 4-byte activations
    assert B.backward_workspace_size(cf) > B.backward_workspace_size(_cfg())
    names = B.trace_backward_stage_names()
    assert names[0] == "start" and names[-1] == "dx" and len(names) == 10
    assert lib.moe_trace_attach_backward(None, 0) == B.MOE_OK
    assert lib.moe_trace_attach_backward(None, 2) == B.MOE_ERR_ARG


def test_training_argument_errors(lib):
    c = _cfg()
    cr = ctypes.byref(c)
    sb = B.train_state_size(c)
    bb = B.backward_workspace_size(c)
    fwd = lambda state, nbytes, x=FAKE: lib.moe_forward_train(  # noqa: E731
        cr, x, FAKE, None, None, None, FAKE, FAKE, FAKE, None, None, None, FAKE, None, None, None,
        None, None, state, nbytes, None)
    assert fwd(FAKE, sb - 1) == B.MOE_ERR_WORKSPACE
    assert fwd(None, sb) == B.MOE_ERR_WORKSPACE
    assert fwd(FAKE + 16, sb) == B.MOE_ERR_ALIGN
    assert fwd(FAKE, sb, x=None) == B.MOE_ERR_ARG
    cf = _cfg(dtype="f32")  # fp32 layers are checked the same way (the state is larger)
    assert lib.moe_forward_train(ctypes.byref(cf), FAKE, FAKE, None, None, None, FAKE, FAKE, FAKE,
                                 None, None, None, FAKE, None, None, None, None, None, FAKE,
                                 B.train_state_size(cf) - 1, None) == B.MOE_ERR_WORKSPACE

    def bwd(dy=FAKE, state_bytes=sb, ws_bytes=bb, c_bal=0.0, dw_gate=FAKE, shared=None, cfg=c):
        return lib.moe_backward(ctypes.byref(cfg), FAKE, FAKE, FAKE, FAKE, FAKE, shared, shared,
                                shared, FAKE, state_bytes, dy, ctypes.c_float(c_bal),
                                ctypes.c_float(0.0), FAKE, FAKE, None, dw_gate, FAKE, FAKE, shared,
                                shared, shared, FAKE, ws_bytes, None)
    assert bwd(dy=None) == B.MOE_ERR_ARG
    assert bwd(dw_gate=None) == B.MOE_ERR_ARG
    assert bwd(dy=FAKE + 2) == B.MOE_ERR_ALIGN
    assert bwd(state_bytes=sb - 1) == B.MOE_ERR_WORKSPACE
    assert bwd(ws_bytes=bb - 1) == B.MOE_ERR_WORKSPACE
    assert bwd(c_bal=float("inf")) == B.MOE_ERR_ARG
    cs = _cfg(F_shared=64)
    assert bwd(cfg=cs, state_bytes=B.train_state_size(cs),
               ws_bytes=B.backward_workspace_size(cs)) == B.MOE_ERR_ARG  # shared grads missing


def test_expert_parallel_argument_errors(lib):
    v = ctypes.c_size_t()
    assert lib.moe_ep_workspace_size(2, 4, ctypes.byref(v)) == B.MOE_OK and v.value > 0
    assert lib.moe_ep_workspace_size(0, 4, ctypes.byref(v)) == B.MOE_ERR_ARG
    assert lib.moe_ep_workspace_size(16, 32, ctypes.byref(v)) == B.MOE_ERR_ARG  # 512 segments > 256
    need = B.ep_workspace_size(2, 4)
    ok = lambda **kw: lib.moe_ep_layout(  # noqa: E731
        kw.get("W", 2), kw.get("EL", 4), kw.get("recv", FAKE), kw.get("max_rows", 100), FAKE, FAKE,
        kw.get("src_of", FAKE), kw.get("ws", FAKE), kw.get("nb", need), None)
    assert ok(recv=None) == B.MOE_ERR_ARG
    assert ok(src_of=None) == B.MOE_ERR_ARG
    assert ok(max_rows=0) == B.MOE_ERR_SHAPE
    assert ok(nb=need - 1) == B.MOE_ERR_WORKSPACE
    assert ok(ws=FAKE + 16) == B.MOE_ERR_ALIGN
    assert lib.moe_permute_rows(FAKE, 10, FAKE, 5, 24, FAKE, FAKE, None) == B.MOE_ERR_ALIGN
    assert lib.moe_permute_rows(FAKE, 10, FAKE, -1, 32, FAKE, FAKE, None) == B.MOE_ERR_SHAPE
    assert lib.moe_permute_rows(FAKE, 10, None, 5, 32, FAKE, FAKE, None) == B.MOE_ERR_ARG
    assert lib.moe_permute_rows(FAKE, 10, FAKE, 5, 32, FAKE, None, None) == B.MOE_ERR_WORKSPACE
    c = _cfg()
    assert lib.moe_combine_weighted(ctypes.byref(c), FAKE, FAKE, None, None, FAKE, None) == B.MOE_ERR_ARG
    assert lib.moe_combine_weighted(ctypes.byref(c), FAKE, FAKE, FAKE, None, FAKE + 8, None) == B.MOE_ERR_ALIGN


def test_peer_exchange_argument_errors(lib):
    """Host-side checks of the peer-memory exchange, all before any launch."""
    c = _cfg()  # E = 8
    need = B.ep_workspace_size(2, c.E // 2)
    disp = lambda **kw: lib.moe_ep_peer_dispatch(  # noqa: E731
        ctypes.byref(kw.get("cfg", c)), kw.get("rank", 0), kw.get("W", 2), kw.get("kept_all", FAKE),
        kw.get("x", FAKE), FAKE, FAKE, FAKE, kw.get("bufs", FAKE), kw.get("rows", 64), FAKE,
        kw.get("remote", FAKE), kw.get("ws", FAKE), kw.get("nb", need), None)
    assert disp(W=3) == B.MOE_ERR_ARG            # 8 experts do not divide among 3 ranks
    assert disp(W=0) == B.MOE_ERR_ARG
    assert disp(W=128) == B.MOE_ERR_ARG          # more ranks than the kernels' table
    assert disp(rank=2) == B.MOE_ERR_ARG
    assert disp(rank=-1) == B.MOE_ERR_ARG
    assert disp(kept_all=None) == B.MOE_ERR_ARG
    assert disp(bufs=None) == B.MOE_ERR_ARG
    assert disp(remote=None) == B.MOE_ERR_ARG
    assert disp(rows=0) == B.MOE_ERR_SHAPE
    assert disp(nb=need - 1) == B.MOE_ERR_WORKSPACE
    assert disp(x=FAKE + 8) == B.MOE_ERR_ALIGN
    comb = lambda **kw: lib.moe_ep_peer_combine(  # noqa: E731
        ctypes.byref(c), kw.get("W", 2), FAKE, FAKE, kw.get("w", FAKE), kw.get("bufs", FAKE),
        kw.get("rows", 64), kw.get("add", None), kw.get("y", FAKE), FAKE, need, None)
    assert comb(W=3) == B.MOE_ERR_ARG
    assert comb(w=None) == B.MOE_ERR_ARG
    assert comb(bufs=None) == B.MOE_ERR_ARG
    assert comb(y=FAKE + 8) == B.MOE_ERR_ALIGN
    assert comb(add=FAKE + 4) == B.MOE_ERR_ALIGN
    assert comb(rows=-5) == B.MOE_ERR_SHAPE
    # the IPC entry points refuse null arguments without touching CUDA
    p = ctypes.c_void_p()
    h = ctypes.create_string_buffer(B.IPC_HANDLE_BYTES)
    assert lib.moe_ipc_alloc(0, ctypes.byref(p), h) == B.MOE_ERR_ARG
    assert lib.moe_ipc_alloc(64, None, h) == B.MOE_ERR_ARG
    assert lib.moe_ipc_open(None, ctypes.byref(p)) == B.MOE_ERR_ARG
    assert lib.moe_ipc_open(h, None) == B.MOE_ERR_ARG
    assert lib.moe_ipc_close(None) == B.MOE_OK
    assert lib.moe_ipc_free(None) == B.MOE_OK
