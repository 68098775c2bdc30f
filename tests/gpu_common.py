"""Helpers of the GPU parity tests: run the library through its C ABI on
seeded inputs and compare with the CPU oracle.

Tolerances (from the acceptance bar of the layer):
  * routing ids, counts, kept, offsets, perm, row_of: bit-exact, the oracle
    routed on the CUDA path's own fp32 logits;
  * probabilities and combine weights: 1e-5 absolute;
  * losses and mean probabilities: 1e-5 relative / absolute;
  * bf16 outputs: |gpu - oracle| <= 1e-2 * max|oracle| + 1e-3 per element;
  * fp32 outputs: |gpu - oracle| <= 1e-4 * max|oracle| per element.
The fp32 logits themselves are checked against the fp64 logits with the
classical bound for a length-n floating-point sum, gamma_n * sum|terms|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_layer_55_b200 import _binding as B
from workloads import Workload

U32 = 2.0 ** -24


def out_tol(wl: Workload, ref: np.ndarray) -> np.ndarray:
    m = float(np.abs(ref).max()) if ref.size else 0.0
    return 1e-4 * m if wl.dtype == "f32" else 1e-2 * m + 1e-3


def assert_close_out(wl, got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    tol = out_tol(wl, ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements out of tolerance; "
                           f"max err {err.max():.3e} > tol {tol:.3e}")
    return float(err.max()), tol


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.double()
    return t.numpy()


class Bufs:
    """Every buffer of the op-by-op path, allocated through torch."""

    def __init__(self, wl: Workload, device="cuda"):
        self.wl = wl
        self.cfg = B.MoeConfig.make(wl.T, wl.D, wl.F, wl.E, wl.K, wl.dtype, wl.capacity_factor,
                                    F_shared=wl.F_shared, **wl.routing())
        T, D, F, E, K = wl.T, wl.D, wl.F, wl.E, wl.K
        dt = wl.torch_dtype
        self.max_rows = B.max_rows(self.cfg)
        R = self.max_rows
        i32, f32 = torch.int32, torch.float32
        self.ws = torch.zeros(B.workspace_size(self.cfg), dtype=torch.uint8, device=device)
        self.logits = torch.empty(T, E, dtype=f32, device=device)
        self.probs = torch.empty(T, E, dtype=f32, device=device)
        self.ids = torch.empty(T, K, dtype=i32, device=device)
        self.w = torch.empty(T, K, dtype=f32, device=device)
        self.mean_prob = torch.empty(E, dtype=f32, device=device)
        self.losses = torch.empty(3, dtype=f32, device=device)
        self.counts = torch.empty(E, dtype=i32, device=device)
        self.kept = torch.empty(E, dtype=i32, device=device)
        self.offsets = torch.empty(E + 1, dtype=i32, device=device)
        self.perm = torch.full((R,), -7, dtype=i32, device=device)
        self.row_of = torch.empty(T * K, dtype=i32, device=device)
        self.x_perm = torch.empty(R, D, dtype=dt, device=device)
        self.h = torch.empty(R, F, dtype=dt, device=device)
        self.y_perm = torch.empty(R, D, dtype=dt, device=device)
        self.y = torch.empty(T, D, dtype=dt, device=device)
        self.y_shared = None
        if wl.F_shared:
            # the shared expert, run op by op as a one-expert problem over x
            self.cfg_s = B.MoeConfig.make(T, D, wl.F_shared, 1, 1, wl.dtype)
            self.ws_s = torch.zeros(B.workspace_size(self.cfg_s), dtype=torch.uint8, device=device)
            self.offs_s = torch.tensor([0, T], dtype=i32, device=device)
            self.h_s = torch.empty(T, wl.F_shared, dtype=dt, device=device)
            self.y_shared = torch.empty(T, D, dtype=dt, device=device)

    def run_ops(self, inp, logits_in=None):
        c = self.cfg
        B.moe_route(c, inp["x"], inp["w_router"], self.ids, self.w, self.ws,
                    router_bias=inp["bias"], logit_noise=inp["noise"], logits_in=logits_in,
                    logits_out=self.logits if logits_in is None else None, probs_out=self.probs,
                    mean_prob=self.mean_prob, losses=self.losses,
                    selection_bias=inp.get("sel_bias"))
        if logits_in is not None:
            self.logits.copy_(logits_in)
        B.moe_dispatch(c, inp["x"], self.ids, self.counts, self.kept, self.offsets, self.perm,
                       self.row_of, self.x_perm, self.ws)
        B.moe_expert_ffn(c, self.x_perm, self.offsets, self.perm, self.w, inp["w_gate"],
                         inp["w_up"], inp["w_down"], self.h, self.y_perm, self.ws)
        if self.y_shared is not None:
            sg, su, sd = inp["shared"]
            B.moe_expert_ffn(self.cfg_s, inp["x"], self.offs_s, None, None, sg, su, sd, self.h_s,
                             self.y_shared, self.ws_s)
        B.moe_combine(c, self.y_perm, self.row_of, self.y, y_add=self.y_shared)
        torch.cuda.synchronize()
        flags = B.moe_get_device_status(self.ws)
        assert flags == 0, f"device status flags {flags:#x}"


def prepared_terms(cfg, w_router):
    """The router weight split by moe_router_prepare (None where the layer's
    router takes no prepared weight)."""
    nb = B.router_terms_size(cfg)
    if nb == 0:
        return None
    terms = torch.empty(nb, dtype=torch.uint8, device="cuda")
    B.moe_router_prepare(cfg, w_router, terms)
    return terms


def check_logits(wl, inp_cpu, logits_gpu):
    """fp32 logits against the fp64 ones, within gamma_n * sum|terms|."""
    L64 = oracle.router_logits(inp_cpu["x"], inp_cpu["w_router"], inp_cpu["bias"],
                               inp_cpu["noise"])
    ax = inp_cpu["x"].double().abs()
    aw = inp_cpu["w_router"].double().abs()
    mag = (ax @ aw).numpy()
    if inp_cpu["bias"] is not None:
        mag = mag + inp_cpu["bias"].double().abs().numpy()[None, :]
    if inp_cpu["noise"] is not None:
        mag = mag + inp_cpu["noise"].double().abs().numpy()
    n = wl.D + 4
    gamma = n * U32 / (1 - n * U32)
    err = np.abs(logits_gpu.astype(np.float64) - L64)
    assert (err <= gamma * mag + 1e-30).all(), f"logit error {err.max():.3e} beyond the fp32 bound"
    return float((err / np.maximum(mag, 1e-30)).max())


def check_routing(wl, b: Bufs, sel_bias=None):
    """Everything the router and the dispatch index pass produce."""
    L = b.logits.cpu().numpy()
    sb = None if sel_bias is None else sel_bias.detach().cpu().numpy()
    ids, w, probs, lse, ent = oracle.route(L, wl.K, sel_bias=sb, with_entropy=True,
                                           **wl.routing())
    counts64, mp, z, bal = oracle.router_stats(ids, probs, lse, wl.E)
    np.testing.assert_array_equal(b.ids.cpu().numpy(), ids)
    np.testing.assert_allclose(b.w.cpu().numpy(), w, rtol=0, atol=1e-5)
    np.testing.assert_allclose(b.probs.cpu().numpy(), probs, rtol=0, atol=1e-5)
    np.testing.assert_allclose(b.mean_prob.cpu().numpy(), mp, rtol=0, atol=1e-5)
    lg = b.losses.cpu().numpy().astype(np.float64)
    assert abs(lg[0] - z) <= 1e-5 * abs(z) + 1e-7, (lg[0], z)
    assert abs(lg[1] - bal) <= 1e-5 * abs(bal) + 1e-7, (lg[1], bal)
    h = float(ent.mean())
    assert abs(lg[2] - h) <= 1e-5 * abs(h) + 1e-6, (lg[2], h)
    C = oracle.capacity(wl.T, wl.K, wl.E, wl.capacity_factor)
    assert C == B.capacity(b.cfg)
    d = oracle.dispatch(ids, wl.E, C)
    np.testing.assert_array_equal(b.counts.cpu().numpy(), d["counts"])
    assert int(counts64.sum()) == wl.T * wl.K
    np.testing.assert_array_equal(b.kept.cpu().numpy(), d["kept"])
    np.testing.assert_array_equal(b.offsets.cpu().numpy(), d["offsets"])
    R = int(d["offsets"][-1])
    np.testing.assert_array_equal(b.perm[:R].cpu().numpy(), d["perm"])
    np.testing.assert_array_equal(b.row_of.cpu().numpy(), d["row_of"])
    return dict(ids=ids, w=w, probs=probs, lse=lse, z=z, bal=bal, C=C, **d)


def expert_getter(inp):
    """Host copies of one expert's weights (fetched one expert at a time)."""
    def get(e):
        return (inp["w_gate"][e].cpu(), inp["w_up"][e].cpu(), inp["w_down"][e].cpu())
    return get


def sample_tokens(wl, rt, n_random=16, seed=0):
    """Token sample: first, last, random, hottest/coldest experts' tokens, and
    any token with a dropped slot."""
    rng = np.random.default_rng(seed)
    T, K = wl.T, wl.K
    toks = {0, T - 1}
    toks.update(int(t) for t in rng.choice(T, size=min(n_random, T), replace=False))
    ids = rt["ids"]
    counts = rt["counts"]
    nz = np.nonzero(counts)[0]
    for e in (int(np.argmax(counts)), int(nz[np.argmin(counts[nz])])):
        tt = np.nonzero((ids == e).any(1))[0]
        toks.update(int(t) for t in tt[:2])
        toks.update(int(t) for t in tt[-1:])
    dropped = np.nonzero((rt["row_of"].reshape(T, K) < 0).any(1))[0]
    toks.update(int(t) for t in dropped[:3])
    toks.update(int(t) for t in dropped[-2:])
    return sorted(toks)


def stratified_rows(rt, block=128, seed=0):
    """Expert-major rows that reach every tile of the grouped GEMMs.

    For each expert with kept rows [a, b): its first and last row, and one row
    at a seeded random position inside every `block`-row block of [a, b).  A
    128-row block is one single-CTA tile, or one CTA's half of a 256-row
    CTA-pair tile, so every m-tile (and both CTAs of a pair) is compared; the
    random position varies the tensor-memory lane and epilogue warp.  Each
    compared row spans all output columns, so every n-tile of the down GEMM
    is reached through it.  Returns (rows, number of blocks, number of
    (expert, 256-row tile) pairs).
    """
    rng = np.random.default_rng(seed)
    offs = np.asarray(rt["offsets"])
    rows, blocks, tiles256 = set(), 0, 0
    for e in range(len(offs) - 1):
        a, b = int(offs[e]), int(offs[e + 1])
        if b <= a:
            continue
        rows.update((a, b - 1))
        for s in range(a, b, block):
            rows.add(int(rng.integers(s, min(s + block, b))))
            blocks += 1
        tiles256 += (b - a + 255) // 256
    return sorted(rows), blocks, tiles256


def full_size_tokens(wl, rt, seed=0, drop_cap=256):
    """Tokens whose outputs a full-size test compares: the owners of the
    stratified rows, the first/last/random/hottest/coldest-expert sample, and
    the tokens with a dropped slot (up to drop_cap, spread over the batch).
    Returns (tokens, stratified rows, blocks, (expert, 256-row tile) pairs)."""
    rows, blocks, tiles = stratified_rows(rt, seed=seed)
    perm = np.asarray(rt["perm"])
    toks = {int(perm[r]) // wl.K for r in rows}
    toks.update(sample_tokens(wl, rt, 12, seed))
    dropped = np.nonzero((np.asarray(rt["row_of"]).reshape(wl.T, wl.K) < 0).any(1))[0]
    if dropped.size > drop_cap:
        dropped = dropped[np.linspace(0, dropped.size - 1, drop_cap).round().astype(np.int64)]
    toks.update(int(t) for t in dropped)
    return sorted(toks), rows, blocks, tiles


def check_tokens(wl, inp, rt, tokens, y_gpu, y_perm=None, x_perm=None):
    """Sampled tokens: the direct per-token computation against y, and (when
    given) each kept slot's y_perm row against w * expert(x) and its x_perm
    row against the token row (an exact copy).  The oracle evaluates each
    expert's sampled rows in one call.  Returns (max error, tolerance, the
    y_perm rows compared)."""
    T, K = wl.T, wl.K
    row_of = rt["row_of"].reshape(T, K)
    kept = row_of >= 0
    x_rows = inp["x"][tokens].cpu()
    outs = oracle.slot_outputs(x_rows, rt["ids"][tokens], kept[tokens], expert_getter(inp))
    ref = oracle.token_outputs(x_rows, rt["ids"][tokens], rt["w"][tokens], kept[tokens], None,
                               outs=outs)
    err, tol = assert_close_out(wl, to_np(y_gpu[tokens]), ref, "y (sampled tokens)")
    rows, refs, src = [], [], []
    for i, t in enumerate(tokens):
        for k in range(K):
            r = int(row_of[t, k])
            if r >= 0:
                rows.append(r)
                refs.append(rt["w"][t, k] * outs[i, k])
                src.append(t)
    if y_perm is not None and rows:
        assert_close_out(wl, to_np(y_perm[rows]), np.stack(refs), "y_perm (sampled rows)")
    if x_perm is not None and rows:
        ri = torch.tensor(rows, dtype=torch.int64, device=x_perm.device)
        ti = torch.tensor(src, dtype=torch.int64, device=inp["x"].device)
        same = (x_perm.index_select(0, ri) == inp["x"].index_select(0, ti)).all(1).cpu()
        bad = [rows[j] for j in np.nonzero(~same.numpy())[0][:5]]
        assert not bad, f"x_perm rows {bad} are not exact copies of their token rows"
    return err, tol, rows
