"""Parity of the layer's backward (moe_forward_train + moe_backward through the
C ABI) with the CPU oracle's backward.

Loss: sum <dY, y> + c_bal * balance + c_z * z ("Lab: build a tiny MoE in
PyTorch", "Smoke test and backward pass"); top-k is a stop-gradient ("2.9
Mixture-of-Experts (MoE) Architectures", "The Router").  The oracle routes on
the CUDA path's own fp32 logits (as the forward's parity tests do), so the
discrete decisions agree and every gradient is compared element by element.

Tolerance, per gradient tensor G (bf16 path): |gpu - oracle| <= 2e-2 * max|oracle|
per element and ||gpu - oracle|| <= 1e-2 * ||oracle|| as a whole; fp32 layers:
1e-4 * max|oracle| per element and 1e-5 normwise.  The CUDA path
rounds five intermediates to bf16 on the way to dx (the expert output o for
dw, w * dY, the saved [g | u], [dg | du], each expert's dx row), each within
2^-9 relative; every sum is fp32.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_55_b200 import _binding as B
from workloads import WORKLOADS, Workload, make_inputs, make_output_grad

from tests.gpu_common import to_np

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("cuda_ok")]

C_BAL, C_Z = 0.3, 0.2  # large enough for the auxiliary terms to be visible


def _dev(inp):
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif isinstance(v, tuple):
            out[k] = tuple(t.cuda() for t in v)
        else:
            out[k] = v.cuda()
    return out


def run_train(wl: Workload, inp, dy, c_bal=C_BAL, c_z=C_Z):
    """forward_train + backward on the GPU; returns host arrays, the fp32
    logits the layer was routed on, and the kernel-reported status."""
    g = _dev(inp)
    dyd = dy.cuda()
    cfg = B.MoeConfig.make(wl.T, wl.D, wl.F, wl.E, wl.K, wl.dtype, wl.capacity_factor,
                           F_shared=wl.F_shared, **wl.routing())
    T, D, F, E, K = wl.T, wl.D, wl.F, wl.E, wl.K
    dev = "cuda"
    f32 = dict(dtype=torch.float32, device=dev)
    # the routed logits, from the same router kernels
    ws = torch.zeros(B.workspace_size(cfg), dtype=torch.uint8, device=dev)
    L = torch.empty((T, E), **f32)
    ids = torch.empty((T, K), dtype=torch.int32, device=dev)
    w = torch.empty((T, K), **f32)
    B.moe_route(cfg, g["x"], g["w_router"], ids, w, ws, router_bias=g["bias"],
                logit_noise=g["noise"], selection_bias=g["sel_bias"], logits_out=L)
    state = torch.zeros(B.train_state_size(cfg), dtype=torch.uint8, device=dev)
    y = torch.empty_like(g["x"])
    B.moe_forward_train(cfg, g["x"], g["w_router"], g["w_gate"], g["w_up"], g["w_down"], y, state,
                        router_bias=g["bias"], logit_noise=g["noise"],
                        selection_bias=g["sel_bias"], shared=g["shared"])
    bws = torch.zeros(B.backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    dx = torch.empty_like(g["x"])
    dwr = torch.empty((D, E), **f32)
    db = torch.empty((E,), **f32) if g["bias"] is not None else None
    dwg = torch.empty((E, D, F), **f32)
    dwu = torch.empty((E, D, F), **f32)
    dwd = torch.empty((E, F, D), **f32)
    dsh = None
    if g["shared"] is not None:
        dsh = tuple(torch.empty(t.shape, **f32) for t in g["shared"])
    B.moe_backward(cfg, g["x"], g["w_router"], g["w_gate"], g["w_up"], g["w_down"], state, dyd, dx,
                   dwr, dwg, dwu, dwd, bws, c_balance=c_bal, c_z=c_z, db_router=db,
                   shared=g["shared"], dshared=dsh)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(state) == 0
    assert B.moe_get_device_status(bws) == 0
    return dict(cfg=cfg, L=L.cpu().numpy(), y=y, dx=dx, dw_router=dwr, db_router=db, dw_gate=dwg,
                dw_up=dwu, dw_down=dwd, dshared=dsh)


def assert_grad(got, ref, what, elem=2e-2, norm=1e-2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    m = float(np.abs(ref).max()) if ref.size else 0.0
    err = np.abs(got - ref)
    bad = err > elem * m
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {ref.size} beyond {elem:g}*max|ref| "
                           f"(max err {err.max():.3e}, max|ref| {m:.3e})")
    nr = float(np.linalg.norm(ref))
    if nr > 0:
        rel = float(np.linalg.norm(got - ref)) / nr
        assert rel <= norm, f"{what}: normwise error {rel:.3e}"


def grad_tolerances(wl):
    """(per element of max|ref|, normwise): the bf16 bar above; for fp32 layers
    every value stays fp32, so only fp32 sums of at most a few thousand terms
    separate the path from the fp64 oracle (relative error a few 1e-6)."""
    return (1e-4, 1e-5) if wl.dtype == "f32" else (2e-2, 1e-2)


def compare_all(wl, inp, dy, got, c_bal=C_BAL, c_z=C_Z):
    sb = None if inp["sel_bias"] is None else inp["sel_bias"].numpy()
    ref = oracle.backward(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], dy,
                          wl.K, wl.capacity_factor, bias=inp["bias"], noise=inp["noise"],
                          logits=got["L"], shared=inp["shared"], c_bal=c_bal, c_z=c_z,
                          sel_bias=sb, **wl.routing())
    fwd_y = ref["fwd"]["y"]
    m = float(np.abs(fwd_y).max())
    ytol = 1e-4 * m if wl.dtype == "f32" else 1e-2 * m + 1e-3
    assert np.abs(to_np(got["y"]) - fwd_y).max() <= ytol, "training forward y"
    el, nm = grad_tolerances(wl)
    assert_grad(to_np(got["dx"]), ref["dx"], "dx", el, nm)
    assert_grad(to_np(got["dw_router"]), ref["dw_router"], "dw_router", el, nm)
    if got["db_router"] is not None:
        assert_grad(to_np(got["db_router"]), ref["db_router"], "db_router", el, nm)
    for k in ("dw_gate", "dw_up", "dw_down"):
        assert_grad(to_np(got[k]), ref[k], k, el, nm)
    if got["dshared"] is not None:
        for name, a, b in zip(("dw_gate_s", "dw_up_s", "dw_down_s"), got["dshared"],
                              ref["dshared"]):
            assert_grad(to_np(a), b, name, el, nm)
    return ref


SMALL = {
    # single CTAs (experts under 128 rows on average); ragged N and K tiles
    "single_ragged": Workload("single_ragged", T=300, D=320, F=448, E=8, K=2),
    # CTA pairs (256-row tiles)
    "pair": Workload("pair", T=1200, D=256, F=384, E=4, K=2),
    "drops": Workload("drops", T=512, D=256, F=256, E=8, K=2, capacity_factor=0.5),
    "sigmoid_scaled": Workload("sigmoid_scaled", T=400, D=192, F=320, E=16, K=3,
                               score_func="sigmoid", renormalize=False, route_scale=2.0),
    "groups_selbias": Workload("groups_selbias", T=320, D=256, F=256, E=16, K=4, n_groups=4,
                               topk_groups=2, sel_bias=True),
    "shared_bias_noise": Workload("shared_bias_noise", T=600, D=256, F=320, E=8, K=2,
                                  bias="zipf", noise=True, F_shared=192, capacity_factor=1.0),
    "many_experts_top1": Workload("many_experts_top1", T=256, D=128, F=128, E=64, K=1),
    # more than 128 experts: the operand tensor maps of the weight-gradient GEMMs are written
    # by two blocks; a few rows per expert (single CTAs, and CTA pairs for M >= 256)
    "e256_single": Workload("e256_single", T=512, D=128, F=128, E=256, K=4),
    "e200_pair": Workload("e200_pair", T=600, D=256, F=320, E=200, K=3, bias="zipf"),
    "single_expert": Workload("single_expert", T=100, D=128, F=192, E=1, K=1),
    "one_token": Workload("one_token", T=1, D=128, F=128, E=8, K=2),
    # few tokens and a long d_model: the combine splits each row over several warps
    # (weighted slots here, the training forward's combine), with a shared expert
    "split_combine_shared": Workload("split_combine_shared", T=64, D=2048, F=64, E=8, K=3,
                                     F_shared=64),
    # fp32 layers (SIMT GEMMs): the fp32 reference layer's shape, and drops with a shared expert
    "f32_layer": Workload("f32_layer", T=512, D=256, F=512, E=8, K=2, dtype="f32"),
    "f32_drops_shared": Workload("f32_drops_shared", T=300, D=128, F=192, E=8, K=2, dtype="f32",
                                 capacity_factor=0.5, F_shared=64, bias="zipf"),
    "f32_sigmoid": Workload("f32_sigmoid", T=200, D=96, F=160, E=16, K=3, dtype="f32",
                            score_func="sigmoid", renormalize=False),
}


def _random_backward_cases(n=24, seed=91):
    """Seeded random layers for the backward: bf16 and fp32, a few to a thousand tokens,
    d_model and d_hidden any multiple of 8 (ragged K tails in the weight-gradient GEMMs,
    ragged N tiles in dH and dX), 1 to 256 experts, drops, every routing option, some
    with a shared expert."""
    import random
    rng = random.Random(seed)
    cases = {}
    while len(cases) < n:
        dtype = "f32" if rng.random() < 0.3 else "bf16"
        E = rng.choice([1, 2, 3, 5, 8, 16, 32, 64, 200, 256])
        K = rng.randint(1, min(E, 8))
        T = rng.choice([3, 50, 257, 600, 1000])
        D = 8 * rng.randint(1, 40)
        F = 8 * rng.randint(1, 40)
        kw = dict(T=T, D=D, F=F, E=E, K=K, dtype=dtype, seed=900 + len(cases))
        if rng.random() < 0.35:
            kw["capacity_factor"] = rng.choice([0.5, 1.0, 1.25])
        if rng.random() < 0.3:
            kw["bias"] = "zipf"
        if rng.random() < 0.3:
            kw["noise"] = True
        if rng.random() < 0.25:
            kw["score_func"] = "sigmoid"
        if rng.random() < 0.25:
            kw["renormalize"] = False
        if rng.random() < 0.2:
            kw["route_scale"] = 1.5
        if rng.random() < 0.25:
            kw["sel_bias"] = True
        groups = [g for g in (2, 4, 8) if E % g == 0]
        if groups and rng.random() < 0.25:
            g = rng.choice(groups)
            tg = rng.randint(1, g)
            if tg * (E // g) >= K:
                kw["n_groups"], kw["topk_groups"] = g, tg
        if rng.random() < 0.2:
            kw["F_shared"] = 8 * rng.randint(1, 24)
        name = "rand_" + "_".join(f"{k}{v}" for k, v in kw.items() if k != "seed")
        cases[name] = Workload(name, **kw)
    return cases


RANDOM = _random_backward_cases()


@pytest.mark.parametrize("name", sorted(RANDOM))
def test_backward_random(name):
    wl = RANDOM[name]
    inp = make_inputs(wl)
    dy = make_output_grad(wl)
    got = run_train(wl, inp, dy)
    compare_all(wl, inp, dy, got)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_backward_small(name):
    wl = SMALL[name]
    inp = make_inputs(wl)
    dy = make_output_grad(wl)
    got = run_train(wl, inp, dy)
    ref = compare_all(wl, inp, dy, got)
    if name == "drops":
        assert (ref["fwd"]["row_of"] < 0).any()


def test_backward_empty_expert():
    """An expert nobody chose gets exactly zero weight gradients."""
    wl = Workload("empty", T=256, D=128, F=192, E=8, K=2, sel_bias=True)
    inp = make_inputs(wl)
    inp["sel_bias"] = inp["sel_bias"].clone()
    inp["sel_bias"][3] = -100.0
    dy = make_output_grad(wl)
    got = run_train(wl, inp, dy)
    ref = compare_all(wl, inp, dy, got)
    assert ref["fwd"]["counts"][3] == 0
    for k in ("dw_gate", "dw_up", "dw_down"):
        assert not got[k][3].any()


def test_backward_deterministic():
    wl = SMALL["drops"]
    inp = make_inputs(wl)
    dy = make_output_grad(wl)
    a = run_train(wl, inp, dy)
    b = run_train(wl, inp, dy)
    for k in ("dx", "dw_router", "dw_gate", "dw_up", "dw_down"):
        assert torch.equal(a[k], b[k]), k


def test_training_forward_matches_inference_forward():
    """moe_forward_train's y equals moe_forward's up to the weight's rounding
    position (the combine instead of the down epilogue)."""
    wl = SMALL["pair"]
    inp = make_inputs(wl)
    got = run_train(wl, inp, make_output_grad(wl))
    g = _dev(inp)
    cfg = got["cfg"]
    ws = torch.zeros(B.forward_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(g["x"])
    B.moe_forward(cfg, g["x"], g["w_router"], g["w_gate"], g["w_up"], g["w_down"], y, ws)
    torch.cuda.synchronize()
    a, b = to_np(got["y"]), to_np(y)
    assert np.abs(a - b).max() <= 1e-2 * np.abs(b).max()


# ----------------------------------------------------------------- full size
def _full_setup(wl):
    inp = make_inputs(wl)
    dy = make_output_grad(wl)
    return inp, dy


def _route_oracle(wl, L, inp):
    sb = None if inp["sel_bias"] is None else inp["sel_bias"].numpy()
    ids, w, probs, lse = oracle.route(L, wl.K, sel_bias=sb, **wl.routing())
    C = oracle.capacity(wl.T, wl.K, wl.E, wl.capacity_factor)
    d = oracle.dispatch(ids, wl.E, C)
    return ids, w, d


@pytest.mark.parametrize("name", ["mixtral_8x", "stmoe_capacity"])
def test_backward_full_size_sampled(name):
    """Full-size layer: dx of sampled tokens, and sampled hidden columns of every
    expert's weight gradients (all rows of the expert), against the oracle."""
    wl = WORKLOADS[name]
    inp, dy = _full_setup(wl)
    got = run_train(wl, inp, dy)
    ids, w, d = _route_oracle(wl, got["L"], inp)
    T, K, E = wl.T, wl.K, wl.E
    row_of = d["row_of"].reshape(T, K)
    perm, offsets = d["perm"], d["offsets"]
    rng = np.random.default_rng(0)
    toks = sorted(set([0, T - 1] + [int(t) for t in rng.choice(T, 6, replace=False)]
                      + [int(t) for t in np.nonzero((row_of < 0).any(1))[0][:2]]))
    # dx of the sampled tokens: their kept rows' backward + the router term
    sel = [(t, k) for t in toks for k in range(K) if row_of[t, k] >= 0]
    tok = np.array([t for t, _ in sel], np.int32)
    ex = np.array([ids[t, k] for t, k in sel], np.int32)
    wt = np.array([w[t, k] for t, k in sel])
    dw_rows, dx_rows = oracle.expert_backward_rows(tok, ex, wt, inp["x"], dy, inp["w_gate"],
                                                   inp["w_up"], inp["w_down"])
    dw_slot = np.zeros((T, K))
    for j, (t, k) in enumerate(sel):
        dw_slot[t, k] = dw_rows[j]
    dL = oracle.router_backward(got["L"], ids, dw_slot, d["counts"], C_BAL, C_Z,
                                score_func=wl.score_func, renormalize=wl.renormalize,
                                route_scale=wl.route_scale)
    _, _, dx_r = oracle.router_linear_backward(inp["x"], inp["w_router"], dL)
    ref_dx = np.stack([dx_r[t] + sum(dx_rows[j] for j, (tt, _) in enumerate(sel) if tt == t)
                       for t in toks])
    assert_grad(to_np(got["dx"][toks]), ref_dx, "dx (sampled tokens)")
    # weight gradients: two experts, four hidden columns each, over all their rows
    fcols = np.array([0, 1, wl.F // 2 + 3, wl.F - 1], np.int32)
    for e in sorted({0, int(np.argmax(d["kept"])), E - 1}):
        a, b = int(offsets[e]), int(offsets[e + 1])
        tk = (perm[a:b] // K).astype(np.int32)
        wte = w.reshape(-1)[perm[a:b]]
        h, dg, du = oracle.expert_backward_cols(tk, np.full(b - a, e, np.int32), wte, fcols,
                                                inp["x"], dy, inp["w_gate"], inp["w_up"],
                                                inp["w_down"])
        dWg, dWu, dWd = oracle.expert_wgrad(tk, wte, inp["x"], dy, h, dg, du)
        fc = torch.from_numpy(fcols).long().cuda()
        assert_grad(to_np(got["dw_gate"][e][:, fc]), dWg, f"dw_gate[{e}] (sampled columns)")
        assert_grad(to_np(got["dw_up"][e][:, fc]), dWu, f"dw_up[{e}] (sampled columns)")
        assert_grad(to_np(got["dw_down"][e][fc, :]), dWd, f"dw_down[{e}] (sampled rows)")


def test_backward_full_size_auxiliary_only():
    """Full-size Mixtral layer with dY = 0: only the auxiliary losses drive the
    router, which the oracle computes for every token: dx, dW_r and db compared
    in full; every expert-weight gradient must be exactly zero."""
    wl = WORKLOADS["mixtral_8x"].with_(bias="zipf")
    inp, dy = _full_setup(wl)
    dy = torch.zeros_like(dy)
    got = run_train(wl, inp, dy, c_bal=1.0, c_z=0.5)
    ids, w, d = _route_oracle(wl, got["L"], inp)
    dL = oracle.router_backward(got["L"], ids, np.zeros((wl.T, wl.K)), d["counts"], 1.0, 0.5)
    dWr, db, dx_r = oracle.router_linear_backward(inp["x"], inp["w_router"], dL)
    assert_grad(to_np(got["dx"]), dx_r, "dx")
    assert_grad(to_np(got["dw_router"]), dWr, "dw_router")
    assert_grad(to_np(got["db_router"]), db, "db_router")
    for k in ("dw_gate", "dw_up", "dw_down"):
        assert not bool(got[k].any()), f"{k} must be zero when dY = 0"
