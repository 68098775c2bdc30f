"""Pins of the oracle's backward to things other than itself.

The loss is  sum <dY, y> + c_bal * balance + c_z * z  ("Lab: build a tiny MoE in
PyTorch", "Smoke test and backward pass": main + 0.01 * balance + 0.001 * z,
differentiated by autograd), with the top-k decision a stop-gradient ("2.9
Mixture-of-Experts (MoE) Architectures", "The Router").

1. torch fp64 autograd of a dense statement of the forward (a loop over tokens
   and slots, every variant: renormalised / plain softmax, sigmoid, route scale,
   capacity drops, group limit and selection bias, shared expert, router bias
   and noise).  Autograd differentiates independently of the oracle's chain
   rule, so a dropped term, a wrong sign or a transposed weight fails here.
2. central finite differences of the oracle's own forward (not its backward).
3. closed forms and invariants: a one-expert layer, the softmax Jacobian's
   zero row sums, linearity in (dY, c_bal, c_z), an unused expert, an
   all-dropped token.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

import oracle


def _inputs(seed, T, D, F, E, Fs=0, quant=None, scale=0.4):
    rng = np.random.default_rng(seed)

    def r(*shape, s=1.0):
        a = rng.standard_normal(shape) * s
        if quant is not None:
            a = np.round(a / quant) * quant
        return a.astype(np.float32)

    d = dict(x=r(T, D), wr=r(D, E, s=0.6), bias=r(E, s=0.3), noise=r(T, E, s=0.2),
             wg=r(E, D, F, s=scale), wu=r(E, D, F, s=scale), wd=r(E, F, D, s=scale),
             dy=rng.standard_normal((T, D)))
    if Fs:
        d["shared"] = (r(D, Fs, s=scale), r(D, Fs, s=scale), r(Fs, D, s=scale))
    return d


def _t(a, grad=True):
    return torch.tensor(np.asarray(a, dtype=np.float64), dtype=torch.float64, requires_grad=grad)


def _autograd(inp, K, cf, c_bal, c_z, use_bias, use_noise, shared, routing):
    """Dense fp64 statement of the layer's loss; ids and the keep mask come from
    the oracle forward (the stop-gradient decision), everything else is
    differentiated by autograd."""
    fwd = oracle.forward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], K, cf,
                         bias=inp["bias"] if use_bias else None,
                         noise=inp["noise"] if use_noise else None,
                         shared=inp.get("shared") if shared else None, **routing)
    ids = torch.tensor(fwd["ids"], dtype=torch.long)
    keep = torch.tensor(fwd["row_of"].reshape(ids.shape) >= 0)
    T, D = inp["x"].shape
    E = inp["wr"].shape[1]
    x, wr, b = _t(inp["x"]), _t(inp["wr"]), _t(inp["bias"])
    wg, wu, wd = _t(inp["wg"]), _t(inp["wu"]), _t(inp["wd"])
    L = x @ wr
    if use_bias:
        L = L + b
    if use_noise:
        L = L + torch.tensor(inp["noise"], dtype=torch.float64)
    sf = routing.get("score_func", "softmax")
    score = torch.softmax(L, -1) if sf == "softmax" else torch.sigmoid(L)
    sel = score.gather(1, ids)
    w = sel / sel.sum(-1, keepdim=True) if routing.get("renormalize", True) else sel
    w = w * routing.get("route_scale", 1.0)
    rows = []
    for t in range(T):
        acc = torch.zeros(D, dtype=torch.float64)
        for k in range(K):
            if keep[t, k]:
                e = int(ids[t, k])
                xe = x[t]
                acc = acc + w[t, k] * ((Fn.silu(xe @ wg[e]) * (xe @ wu[e])) @ wd[e])
        rows.append(acc)
    y = torch.stack(rows)
    sh = None
    if shared:
        sh = [_t(a) for a in inp["shared"]]
        y = y + (Fn.silu(x @ sh[0]) * (x @ sh[1])) @ sh[2]
    counts = torch.bincount(ids.reshape(-1), minlength=E).to(torch.float64)
    f = counts / (T * K)
    norm = score / score.sum(-1, keepdim=True)
    bal = E * (f * norm.mean(0)).sum()
    z = (torch.logsumexp(L, -1) ** 2).mean()
    loss = (torch.tensor(inp["dy"]) * y).sum() + c_bal * bal + c_z * z
    loss.backward()
    out = dict(dx=x.grad, dw_router=wr.grad, dw_gate=wg.grad, dw_up=wu.grad, dw_down=wd.grad)
    if use_bias:
        out["db_router"] = b.grad
    if shared:
        out["dshared"] = tuple(a.grad for a in sh)
    return {k: (tuple(t.numpy() for t in v) if isinstance(v, tuple) else v.numpy())
            for k, v in out.items()}


CASES = {
    "softmax_renorm": dict(K=2, cf=0.0, routing={}),
    "softmax_plain_scaled": dict(K=2, cf=0.0, routing=dict(renormalize=False, route_scale=2.5)),
    "sigmoid_renorm": dict(K=2, cf=0.0, routing=dict(score_func="sigmoid")),
    "sigmoid_plain": dict(K=3, cf=0.0, routing=dict(score_func="sigmoid", renormalize=False)),
    "capacity_drops": dict(K=2, cf=0.5, routing={}),
    "groups_selbias": dict(K=2, cf=0.0, routing=dict(n_groups=2, topk_groups=1,
                                                    sel_bias=np.array([0.5, -0.3, 0.1, 0.9]))),
    "top1": dict(K=1, cf=0.0, routing={}),
    "bias_noise_shared": dict(K=2, cf=1.0, routing={}, bias=True, noise=True, shared=True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_autograd(name):
    c = CASES[name]
    T, D, F, E = 11, 12, 10, 4
    inp = _inputs(7 + len(name), T, D, F, E, Fs=6 if c.get("shared") else 0)
    c_bal, c_z = 0.37, 0.21  # large, so the auxiliary terms are visible
    ref = _autograd(inp, c["K"], c["cf"], c_bal, c_z, c.get("bias", False), c.get("noise", False),
                    c.get("shared", False), c["routing"])
    got = oracle.backward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], inp["dy"], c["K"],
                          c["cf"], bias=inp["bias"] if c.get("bias") else None,
                          noise=inp["noise"] if c.get("noise") else None,
                          shared=inp.get("shared") if c.get("shared") else None,
                          c_bal=c_bal, c_z=c_z, **c["routing"])
    if name == "capacity_drops":
        assert (got["fwd"]["row_of"] < 0).sum() > 0, "case must drop assignments"
    for k in ("dx", "dw_router", "dw_gate", "dw_up", "dw_down", "db_router"):
        if k in ref:
            np.testing.assert_allclose(got[k], ref[k], rtol=1e-10, atol=1e-13, err_msg=k)
    if "dshared" in ref:
        for a, b in zip(got["dshared"], ref["dshared"]):
            np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-13)


def _loss(inp, K, cf, c_bal, c_z, routing, shared):
    fwd = oracle.forward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], K, cf,
                         bias=inp["bias"], shared=inp.get("shared") if shared else None, **routing)
    return (float((inp["dy"] * fwd["y"]).sum()) + c_bal * fwd["balance_loss"]
            + c_z * fwd["z_loss"]), fwd["ids"]


@pytest.mark.parametrize("routing,shared", [({}, True), (dict(score_func="sigmoid"), False),
                                            (dict(renormalize=False, route_scale=1.5), False)])
def test_backward_matches_finite_differences(routing, shared):
    T, D, F, E, K, cf = 9, 8, 6, 4, 2, 1.0
    q = 2.0 ** -16  # inputs on a 2^-16 grid, so x +- 2^-14 is exact in fp32
    inp = _inputs(3, T, D, F, E, Fs=4 if shared else 0, quant=q)
    c_bal, c_z = 0.3, 0.2
    g = oracle.backward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], inp["dy"], K, cf,
                        bias=inp["bias"], shared=inp.get("shared") if shared else None,
                        c_bal=c_bal, c_z=c_z, **routing)
    h = 2.0 ** -14
    rng = np.random.default_rng(11)
    targets = [("x", "dx"), ("wr", "dw_router"), ("bias", "db_router"), ("wg", "dw_gate"),
               ("wu", "dw_up"), ("wd", "dw_down")]
    if shared:
        targets += [("shared0", 0), ("shared1", 1), ("shared2", 2)]
    for key, gkey in targets:
        for _ in range(4):
            if key.startswith("shared"):
                arr = inp["shared"][int(key[-1])]
                grad = g["dshared"][gkey]
            else:
                arr = inp[key]
                grad = g[gkey]
            idx = tuple(rng.integers(0, n) for n in arr.shape)
            old = arr[idx]
            arr[idx] = np.float32(old + h)
            lp, ids_p = _loss(inp, K, cf, c_bal, c_z, routing, shared)
            arr[idx] = np.float32(old - h)
            lm, ids_m = _loss(inp, K, cf, c_bal, c_z, routing, shared)
            arr[idx] = old
            assert (ids_p == ids_m).all(), "perturbation crossed a routing decision"
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * (1 + abs(grad[idx])), (key, idx, fd, grad[idx])


def test_one_expert_layer_closed_form():
    """E = K = 1: the gate weight is identically 1 (softmax of one logit,
    renormalised), so the router sees only the z-loss: dL[t] = c_z * 2 L[t] / T
    (lse of one logit is the logit), and dW_r = x^T dL, db = sum dL."""
    T, D, F = 7, 5, 6
    inp = _inputs(5, T, D, F, 1)
    c_z = 0.3
    g = oracle.backward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], inp["dy"], 1,
                        bias=inp["bias"], c_bal=0.5, c_z=c_z)
    L = inp["x"].astype(np.float64) @ inp["wr"].astype(np.float64) + inp["bias"]
    dl = c_z * 2.0 * L / T
    np.testing.assert_allclose(g["dlogits"], dl, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(g["dw_router"], inp["x"].astype(np.float64).T @ dl, rtol=1e-12,
                               atol=1e-15)
    np.testing.assert_allclose(g["db_router"], dl.sum(0), rtol=1e-12, atol=1e-15)
    assert np.all(g["dw_slot"] != 0)  # the slot's weight gradient exists but has no effect


def test_softmax_logit_gradient_rows_sum_to_zero():
    """Without the z-loss every softmax-routed token's logit gradient lies in
    the softmax Jacobian's range, whose rows sum to zero."""
    inp = _inputs(9, 13, 8, 6, 5)
    g = oracle.backward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], inp["dy"], 2,
                        c_bal=0.4, c_z=0.0)
    assert np.abs(g["dlogits"].sum(1)).max() < 1e-15 * 100
    assert np.abs(g["dlogits"]).max() > 1e-3


def test_gradient_is_linear_in_dy_and_coefficients():
    inp = _inputs(13, 10, 8, 6, 4)
    args = (inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"])
    full = oracle.backward(*args, inp["dy"], 2, c_bal=0.3, c_z=0.2)
    zero = np.zeros_like(inp["dy"])
    parts = [oracle.backward(*args, inp["dy"], 2),
             oracle.backward(*args, zero, 2, c_bal=0.3),
             oracle.backward(*args, zero, 2, c_z=0.2)]
    for k in ("dx", "dw_router", "dw_gate", "dw_up", "dw_down"):
        np.testing.assert_allclose(full[k], sum(p[k] for p in parts), rtol=1e-12, atol=1e-14)
    # with dY = 0 the experts' weights get nothing
    assert not parts[1]["dw_gate"].any() and not parts[2]["dw_down"].any()


def test_unused_expert_and_dropped_token():
    """An expert no token chose has zero weight gradients; a token whose every
    slot was dropped receives input gradient from the router only."""
    T, D, F, E, K = 12, 8, 6, 4, 2
    inp = _inputs(17, T, D, F, E)
    sel = np.array([0.0, 0.0, -50.0, 0.0])  # expert 2 is never selected
    g = oracle.backward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], inp["dy"], K, 0.25,
                        c_bal=0.1, c_z=0.1, sel_bias=sel)
    f = g["fwd"]
    assert f["counts"][2] == 0
    assert not g["dw_gate"][2].any() and not g["dw_up"][2].any() and not g["dw_down"][2].any()
    dropped = np.where((f["row_of"].reshape(T, K) < 0).all(1))[0]
    assert dropped.size > 0, "case must drop a whole token"
    _, _, dx_r = oracle.router_linear_backward(inp["x"], inp["wr"], g["dlogits"])
    np.testing.assert_allclose(g["dx"][dropped], dx_r[dropped], rtol=0, atol=0)
    assert np.all(g["dw_slot"].reshape(-1)[f["row_of"] < 0] == 0)


def test_column_restricted_backward_matches_full():
    """expert_backward_cols + expert_wgrad on a column subset equal the
    corresponding columns of the full per-row computation."""
    T, D, F, E, K = 10, 8, 12, 3, 2
    inp = _inputs(21, T, D, F, E)
    g = oracle.backward(inp["x"], inp["wr"], inp["wg"], inp["wu"], inp["wd"], inp["dy"], K)
    f = g["fwd"]
    e = int(np.argmax(np.diff(f["offsets"])))
    a, b = int(f["offsets"][e]), int(f["offsets"][e + 1])
    tok = f["perm"][a:b] // K
    wt = f["row_weight"][a:b]
    cols = np.array([0, 5, 11], np.int32)
    h, dg, du = oracle.expert_backward_cols(tok, np.full(b - a, e), wt, cols, inp["x"], inp["dy"],
                                            inp["wg"], inp["wu"], inp["wd"])
    dWg, dWu, dWd = oracle.expert_wgrad(tok, wt, inp["x"], inp["dy"], h, dg, du)
    np.testing.assert_allclose(dWg, g["dw_gate"][e][:, cols], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dWu, g["dw_up"][e][:, cols], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dWd, g["dw_down"][e][cols, :], rtol=1e-12, atol=1e-15)
