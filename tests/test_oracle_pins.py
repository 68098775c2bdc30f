"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with a retyped copy of its own formulas: the
checks are values the pages give (tests/golden/), closed forms, invariants,
special cases that reduce to a library routine (torch fp64 on the CPU), and
brute force on tiny inputs.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import golden
from workloads import Workload, make_inputs

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _wl(T=24, D=32, F=48, E=4, K=2, dtype="f32", cf=0.0, bias=None, noise=False, seed=3):
    return Workload("t", T=T, D=D, F=F, E=E, K=K, dtype=dtype, capacity_factor=cf, bias=bias,
                    noise=noise, seed=seed)


def _fwd(inp, wl, **kw):
    return oracle.forward(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"],
                          wl.K, wl.capacity_factor, inp["bias"], inp["noise"], **kw)


def _swiglu_torch(x64, wg, wu, wd):
    """Library form of one SwiGLU expert (torch fp64 matmuls)."""
    g = x64 @ wg.double()
    u = x64 @ wu.double()
    return (torch.nn.functional.silu(g) * u) @ wd.double()


# ---------------------------------------------------------------- routing ---

def test_worked_logit_vector():
    """Worked router example of the llm-stack-book chapter (golden fixture)."""
    g = golden("worked_router_logits.json")
    L = np.array([g["logits"]], dtype=np.float64)
    ids, w, probs, lse = oracle.route(L, g["k"])
    assert ids[0].tolist() == g["expected_ids"]
    e = math.e
    assert w[0, 0] == pytest.approx(e / (1 + e), abs=1e-15)
    assert w[0, 1] == pytest.approx(1 / (1 + e), abs=1e-15)
    # softmax is fixed by: positive, sums to one, log-ratios equal logit gaps
    p = probs[0]
    assert (p > 0).all() and p.sum() == pytest.approx(1.0, abs=1e-15)
    for a in range(8):
        for b in range(8):
            assert math.log(p[a] / p[b]) == pytest.approx(L[0, a] - L[0, b], abs=1e-12)
    # lse lies in [max, max + ln E] and shifts with the logits
    assert 3.0 < lse[0] < 3.0 + math.log(8)
    _, _, _, lse2 = oracle.route(L + 5.25, g["k"])
    assert lse2[0] - lse[0] == pytest.approx(5.25, abs=1e-12)


def test_uniform_logits_closed_forms_and_tie_rule():
    """Equal logits: ties go to the lower expert id; lse = c + ln E."""
    for E, K in [(8, 2), (8, 8), (5, 3), (64, 6)]:
        L = np.full((3, E), 0.75)
        ids, w, probs, lse = oracle.route(L, K)
        assert (ids == np.arange(K)[None, :]).all()
        np.testing.assert_allclose(w, 1.0 / K, atol=1e-15)
        np.testing.assert_allclose(probs, 1.0 / E, atol=1e-15)
        np.testing.assert_allclose(lse, 0.75 + math.log(E), atol=1e-14)


def test_top1_weight_is_exactly_one():
    """top_k = 1 with renormalisation gives a combine weight of exactly 1."""
    rng = np.random.default_rng(0)
    L = rng.normal(size=(50, 16))
    _, w, _, _ = oracle.route(L, 1)
    assert (w == 1.0).all()


def _brute_force_topk(Lrow, K):
    """Enumerate all K-subsets; keep the unique one whose every member ranks
    before every non-member under (logit desc, id asc)."""
    E = len(Lrow)

    def before(a, b):
        return Lrow[a] > Lrow[b] or (Lrow[a] == Lrow[b] and a < b)

    found = []
    for S in itertools.combinations(range(E), K):
        rest = [e for e in range(E) if e not in S]
        if all(before(a, b) for a in S for b in rest):
            found.append(S)
    assert len(found) == 1
    S = list(found[0])
    # slot order: repeatedly the member that ranks before all remaining members
    order = []
    while S:
        top = [a for a in S if all(a == b or before(a, b) for b in S)][0]
        order.append(top)
        S.remove(top)
    return order


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    T, E = 16, 7
    L = np.round(rng.normal(size=(T, E)), 0)  # coarse values: many exact ties
    for K in (1, 2, 3, 7):
        ids, w, _, _ = oracle.route(L, K)
        for t in range(T):
            assert ids[t].tolist() == _brute_force_topk(L[t].tolist(), K)
        np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-14)


def test_route_matches_torch_library_on_tie_free_inputs():
    """torch fp64 softmax / topk / logsumexp on inputs without ties."""
    g = torch.Generator().manual_seed(11)
    L = torch.randn(200, 32, generator=g, dtype=torch.float64)
    ids, w, probs, lse = oracle.route(L.numpy(), 4)
    p_ref = torch.softmax(L, dim=-1)
    top_w, top_i = p_ref.topk(4, dim=-1)
    assert (torch.from_numpy(ids).long() == top_i).all()
    np.testing.assert_allclose(w, (top_w / top_w.sum(-1, keepdim=True)).numpy(), atol=1e-14)
    np.testing.assert_allclose(probs, p_ref.numpy(), atol=1e-15)
    np.testing.assert_allclose(lse, torch.logsumexp(L, -1).numpy(), atol=1e-13)


def test_router_logits_match_library_matmul():
    """x W_r + b + noise against a torch fp64 matmul, bf16 and fp32 inputs."""
    for dtype in ("f32", "bf16"):
        wl = _wl(T=37, D=40, E=12, dtype=dtype, bias="zipf", noise=True)
        inp = make_inputs(wl)
        L = oracle.router_logits(inp["x"], inp["w_router"], inp["bias"], inp["noise"])
        ref = (inp["x"].double() @ inp["w_router"].double() + inp["bias"].double()
               + inp["noise"].double())
        np.testing.assert_allclose(L, ref.numpy(), rtol=0, atol=1e-12)
        L0 = oracle.router_logits(inp["x"], inp["w_router"])
        np.testing.assert_allclose(L0, (inp["x"].double() @ inp["w_router"].double()).numpy(),
                                   atol=1e-12)


# ------------------------------------------------------------------ stats ---

def test_balance_and_z_loss_closed_forms():
    g = golden("balance_loss_closed_forms.json")["hand_example"]
    L = np.array([[0.0, math.log(3.0)], [0.0, math.log(3.0)]])
    ids, w, probs, lse = oracle.route(L, 1)
    counts, mp, z, bal = oracle.router_stats(ids, probs, lse, 2)
    assert counts.tolist() == [0, 2]
    np.testing.assert_allclose(mp, [0.25, 0.75], atol=1e-15)
    assert bal == pytest.approx(g["expected_balance"], abs=1e-14)
    assert z == pytest.approx(math.log(4.0) ** 2, abs=1e-14)


def test_balance_is_one_when_uniform_and_E_when_collapsed():
    """Uniform routing gives 1; a collapsed router gives E."""
    T, E = 40, 8
    L = np.zeros((T, E))
    ids, w, probs, lse = oracle.route(L, E)  # every token takes every expert
    _, _, z, bal = oracle.router_stats(ids, probs, lse, E)
    assert bal == pytest.approx(1.0, abs=1e-14)
    assert z == pytest.approx(math.log(E) ** 2, abs=1e-13)
    L = np.zeros((T, E))
    L[:, 3] = 800.0  # all mass on expert 3
    ids, w, probs, lse = oracle.route(L, 1)
    counts, _, _, bal = oracle.router_stats(ids, probs, lse, E)
    assert counts[3] == T and counts.sum() == T
    assert bal == pytest.approx(float(E), abs=1e-12)


def test_tinymoe_smoke_shapes():
    """The lab's smoke test: (3, 7, 32), 4 experts, top-2 -> 42 assignments."""
    g = golden("tinymoe_smoke.json")
    T = g["batch"] * g["sequence"]
    wl = _wl(T=T, D=g["d_model"], F=g["d_hidden"], E=g["n_experts"], K=g["top_k"], seed=23)
    out = _fwd(make_inputs(wl), wl)
    assert out["y"].shape == (T, g["d_model"])
    assert np.isfinite(out["y"]).all()
    assert int(out["counts"].sum()) == g["expected_assignment_count"]
    np.testing.assert_allclose(out["weights"].sum(1), 1.0, atol=1e-14)
    assert np.isfinite(out["z_loss"]) and np.isfinite(out["balance_loss"])


# --------------------------------------------------------------- capacity ---

def test_capacity_exercise_closed_form():
    g = golden("capacity_exercise.json")
    N, E, k, cf = g["N"], g["E"], g["k"], g["capacity_factor"]
    assert N * k // E == g["expected_mean_per_expert"]
    C = oracle.capacity(N, k, E, cf)
    assert C == g["expected_capacity"]
    # hand-built routing: tokens 0..899 put expert 0 in slot 0; every other
    # slot goes round-robin over experts 1..15, so no other expert overflows
    ids = np.zeros((N, k), np.int32)
    nxt = 0
    for t in range(N):
        for s in range(k):
            if s == 0 and t < g["hot_expert_tokens"]:
                ids[t, s] = 0
            else:
                ids[t, s] = 1 + nxt % (E - 1)
                nxt += 1
    d = oracle.dispatch(ids, E, C)
    assert d["counts"][0] == g["hot_expert_tokens"]
    assert d["counts"][0] - d["kept"][0] == g["expected_dropped_at_hot_expert"]
    assert (d["counts"][1:] <= C).all() and (d["kept"][1:] == d["counts"][1:]).all()
    # the dropped ones are the last 132 hot-expert tokens in token order
    dropped = np.nonzero(d["row_of"].reshape(N, k)[:, 0] < 0)[0]
    assert dropped.tolist() == list(range(768, 900))


def test_stmoe_capacity_value():
    g = golden("stmoe_capacity.json")
    assert oracle.capacity(g["T"], g["k"], g["E"], g["capacity_factor"]) == g["expected_capacity"]


def test_capacity_rounding_and_floor():
    assert oracle.capacity(3, 1, 8, 0.5) == 1          # ceil(0.1875) = 1
    assert oracle.capacity(1, 1, 64, 0.01) == 1        # max(1, ...)
    assert oracle.capacity(10, 2, 4, 1.0) == 5         # exact
    assert oracle.capacity(10, 2, 3, 1.0) == 7         # ceil(6.67)
    assert oracle.capacity(10, 2, 4, 0.0) == 20        # dropless: T*K


def _brute_force_keep(ids, C):
    """(t,k) is kept iff fewer than C earlier assignments chose the same expert
    (earlier = smaller token index; a token picks an expert at most once)."""
    T, K = ids.shape
    keep = np.zeros((T, K), bool)
    for t in range(T):
        for k in range(K):
            e = ids[t, k]
            earlier = int((ids[:t] == e).sum())
            keep[t, k] = earlier < C
    return keep


@pytest.mark.parametrize("seed", range(5))
def test_dispatch_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    T, E, K = 16, 5, 2
    L = rng.normal(size=(T, E))
    L[:, 1] += 1.5  # a hot expert, so that some capacity overflows
    ids, _, _, _ = oracle.route(L, K)
    for C in (1, 2, 3, 5, T * K):
        d = oracle.dispatch(ids, E, C)
        keep = _brute_force_keep(ids, C)
        assert ((d["row_of"].reshape(T, K) >= 0) == keep).all()
        counts = np.bincount(ids.reshape(-1), minlength=E)
        assert (d["counts"] == counts).all() and counts.sum() == T * K
        assert (d["kept"] == np.minimum(counts, C)).all()
        assert (d["offsets"] == np.concatenate([[0], np.cumsum(d["kept"])])).all()
        # perm and row_of are inverse on the kept assignments
        R = int(d["offsets"][-1])
        assert R <= min(T * K, E * C)
        for row in range(R):
            assert d["row_of"][d["perm"][row]] == row
        # each expert's rows are its kept assignments in increasing token order
        for e in range(E):
            seg = d["perm"][d["offsets"][e]:d["offsets"][e + 1]]
            assert (ids.reshape(-1)[seg] == e).all()
            assert (np.diff(seg // K) > 0).all()


# ----------------------------------------------------------- expert + combine

def test_identity_experts_return_x():
    """Identity experts with a dropless combine give back x (weights sum to 1)."""
    wl = _wl(T=30, D=16, E=6, K=3, dtype="bf16")
    inp = make_inputs(wl)
    L = oracle.router_logits(inp["x"], inp["w_router"])
    ids, w, _, _ = oracle.route(L, wl.K)
    d = oracle.dispatch(ids, wl.E, oracle.capacity(wl.T, wl.K, wl.E, 0.0))
    x_perm = oracle.gather(inp["x"], d["perm"], wl.K)
    y = oracle.combine(x_perm, d["row_of"], w, wl.T, wl.K)
    np.testing.assert_allclose(y, inp["x"].double().numpy(), rtol=0, atol=1e-14)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_identical_experts_reduce_to_dense_ffn(dtype):
    """Identical experts, dropless, any router: the layer is one dense SwiGLU
    FFN (upcycling invariant), computed here with torch fp64 matmuls."""
    wl = _wl(T=40, D=24, F=40, E=5, K=2, dtype=dtype, bias="zipf", noise=True, seed=7)
    inp = make_inputs(wl)
    for key in ("w_gate", "w_up", "w_down"):
        inp[key] = inp[key][:1].expand_as(inp[key]).contiguous()
    out = _fwd(inp, wl)
    ref = _swiglu_torch(inp["x"].double(), inp["w_gate"][0], inp["w_up"][0], inp["w_down"][0])
    np.testing.assert_allclose(out["y"], ref.numpy(), rtol=0, atol=1e-12)


def test_K_equals_E_uniform_router_is_mean_of_experts():
    """K = E with a zero router: every expert, weight 1/E each, ids 0..E-1."""
    wl = _wl(T=20, D=16, F=24, E=4, K=4)
    inp = make_inputs(wl)
    inp["w_router"] = torch.zeros_like(inp["w_router"])
    out = _fwd(inp, wl)
    assert (out["ids"] == np.arange(4)[None, :]).all()
    x64 = inp["x"].double()
    ref = sum(_swiglu_torch(x64, inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e])
              for e in range(4)) / 4.0
    np.testing.assert_allclose(out["y"], ref.numpy(), rtol=0, atol=1e-12)


def test_direct_token_computation_matches_layer():
    """'Trace one token by hand': per-token sums equal the dispatch/combine
    output; checked against torch fp64 expert matmuls too."""
    wl = _wl(T=33, D=16, F=32, E=6, K=2, dtype="bf16", seed=5)
    inp = make_inputs(wl)
    out = _fwd(inp, wl)
    kept = out["row_of"].reshape(wl.T, wl.K) >= 0
    tokens = [0, 7, 32]
    direct = oracle.token_outputs(
        inp["x"][tokens], out["ids"][tokens], out["weights"][tokens], kept[tokens],
        lambda e: (inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e]))
    np.testing.assert_allclose(out["y"][tokens], direct, rtol=0, atol=1e-13)
    x64 = inp["x"].double()
    for t in tokens:
        ref = sum(float(out["weights"][t, k]) * _swiglu_torch(
            x64[t:t + 1], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e])[0]
            for k, e in enumerate(out["ids"][t].tolist()))
        np.testing.assert_allclose(out["y"][t], ref.numpy(), rtol=0, atol=1e-12)


def test_dropped_assignments_contribute_zero():
    """With a tight capacity, dropped slots add nothing and a token whose every
    slot is dropped gets an all-zero output."""
    wl = _wl(T=48, D=16, F=24, E=4, K=2, cf=0.25, seed=9)
    inp = make_inputs(wl)
    out = _fwd(inp, wl)
    C = out["capacity"]
    assert C == 6
    kept = out["row_of"].reshape(wl.T, wl.K) >= 0
    assert (~kept).any()
    all_dropped = np.nonzero(~kept.any(1))[0]
    assert all_dropped.size > 0
    assert (out["y"][all_dropped] == 0.0).all()
    x64 = inp["x"].double()
    for t in range(wl.T):
        ref = torch.zeros(wl.D, dtype=torch.float64)
        for k in range(wl.K):
            if kept[t, k]:
                e = int(out["ids"][t, k])
                ref += float(out["weights"][t, k]) * _swiglu_torch(
                    x64[t:t + 1], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e])[0]
        np.testing.assert_allclose(out["y"][t], ref.numpy(), rtol=0, atol=1e-12)
    assert (out["kept"] <= C).all()


def test_empty_experts_are_fine():
    """An expert that no token chooses is skipped without error."""
    wl = _wl(T=12, D=8, F=16, E=6, K=1)
    inp = make_inputs(wl)
    inp["w_router"] = torch.zeros_like(inp["w_router"])
    inp["bias"] = torch.tensor([0, 0, 5.0, 0, 0, 0])
    out = _fwd(inp, wl)
    assert out["counts"].tolist() == [0, 0, 12, 0, 0, 0]
    assert (out["offsets"] == [0, 0, 0, 12, 12, 12, 12]).all()
    ref = _swiglu_torch(inp["x"].double(), inp["w_gate"][2], inp["w_up"][2], inp["w_down"][2])
    np.testing.assert_allclose(out["y"], ref.numpy(), atol=1e-12)


def test_parity_mode_uses_given_logits():
    """Routing from given fp32 logits equals routing from those logits' fp64
    copy (the conversion is exact) and differs from the internal logits only
    through the logits themselves."""
    wl = _wl(T=20, D=16, E=8, K=2)
    inp = make_inputs(wl)
    L32 = oracle.router_logits(inp["x"], inp["w_router"]).astype(np.float32)
    a = _fwd(inp, wl, logits=L32)
    ids, w, _, _ = oracle.route(L32.astype(np.float64), wl.K)
    assert (a["ids"] == ids).all()
    np.testing.assert_array_equal(a["weights"], w)


def test_shared_expert_adds_a_dense_swiglu():
    """"Add a shared expert": the layer with a shared expert equals the routed
    layer plus one dense SwiGLU FFN over every token (torch fp64 matmuls)."""
    wl = _wl(T=30, D=16, F=24, E=4, K=2, dtype="bf16", seed=31)
    inp = make_inputs(wl)
    g = torch.Generator().manual_seed(4)
    Fs = 40
    sh = tuple((torch.randn(*s, generator=g) * 0.05).to(torch.bfloat16)
               for s in ((16, Fs), (16, Fs), (Fs, 16)))
    a = _fwd(inp, wl)
    b = _fwd(inp, wl, shared=sh)
    dense = _swiglu_torch(inp["x"].double(), *sh)
    np.testing.assert_allclose(b["y"] - a["y"], dense.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(b["y_shared"], dense.numpy(), rtol=0, atol=1e-12)


def test_results_do_not_depend_on_thread_count():
    """Every parallel loop of the oracle owns disjoint outputs: one thread and
    several give the same bits."""
    from workloads import Workload, make_inputs
    wl = Workload("threads", T=96, D=64, F=48, E=8, K=2, capacity_factor=0.75, bias="zipf", seed=3)
    inp = make_inputs(wl)
    n = oracle.num_threads()
    try:
        oracle.set_num_threads(1)
        a = oracle.forward(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], wl.K,
                           wl.capacity_factor, bias=inp["bias"])
        oracle.set_num_threads(4)
        b = oracle.forward(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], wl.K,
                           wl.capacity_factor, bias=inp["bias"])
    finally:
        oracle.set_num_threads(n)
    for k in ("logits", "ids", "weights", "row_of", "o", "y", "z_loss", "balance_loss"):
        assert np.array_equal(a[k], b[k]), k
