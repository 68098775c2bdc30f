"""Pins of the oracle's router variants: softmax-then-top-k without
renormalisation, sigmoid scores, the DeepSeek-V3 selection-only bias and its
update step, group-limited routing, route scaling and the router entropy.

Each is checked against a closed form, a library routine (torch fp64) or an
independent formulation, never against a retyped copy of the oracle's code.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import golden


def test_softmax_then_topk_keeps_the_probability_slice():
    """GShard/Switch convention of the llm-stack-book chapter: the selected
    weights are the full softmax's probabilities, not renormalised."""
    g = golden("worked_router_logits.json")
    L = np.array([g["logits"]])
    ids, w, probs, _ = oracle.route(L, 2, renormalize=False)
    assert ids[0].tolist() == g["expected_ids"]
    np.testing.assert_allclose(w[0], probs[0, ids[0]], rtol=0, atol=1e-15)
    assert w[0].sum() < 1.0
    assert w[0, 0] / w[0, 1] == pytest.approx(math.e, rel=1e-14)  # exp(3 - 2)
    # Switch top-1 keeps the selected probability (lab, ablation 2)
    ids1, w1, probs1, _ = oracle.route(L, 1, renormalize=False)
    assert w1[0, 0] == pytest.approx(probs1[0].max(), abs=1e-15) and ids1[0, 0] == 5


def test_sigmoid_scores_closed_forms_and_library():
    L = np.zeros((3, 6))
    _, w, probs, _ = oracle.route(L, 4, score_func="sigmoid")
    np.testing.assert_allclose(w, 0.25, atol=1e-15)           # 0.5 / (4 * 0.5)
    _, w, _, _ = oracle.route(L, 4, score_func="sigmoid", renormalize=False)
    np.testing.assert_allclose(w, 0.5, atol=1e-15)            # sigmoid(0)
    np.testing.assert_allclose(probs.sum(1), 1.0, atol=1e-15)
    g = torch.Generator().manual_seed(5)
    Lt = torch.randn(100, 16, generator=g, dtype=torch.float64) * 3
    ids, w, probs, _ = oracle.route(Lt.numpy(), 3, score_func="sigmoid")
    s = torch.sigmoid(Lt)
    top = Lt.topk(3, dim=-1).indices
    assert (torch.from_numpy(ids).long() == top).all()
    sel = torch.gather(s, 1, top)
    np.testing.assert_allclose(w, (sel / sel.sum(1, keepdim=True)).numpy(), atol=1e-14)
    np.testing.assert_allclose(probs, (s / s.sum(1, keepdim=True)).numpy(), atol=1e-15)


def test_selection_only_bias_against_library():
    """llm-stack-book Exercise 6: top-k on h + b, gate weights = softmax of the
    unbiased logits over the chosen experts."""
    g = torch.Generator().manual_seed(7)
    L = torch.randn(200, 8, generator=g, dtype=torch.float64)
    b = torch.tensor([-5.0, 0.3, 0.0, 1.0, -0.2, 0.0, 0.5, -1.0], dtype=torch.float64)
    ids, w, _, _ = oracle.route(L.numpy(), 2, sel_bias=b.numpy())
    idx = (L + b).topk(2, dim=-1).indices
    assert (torch.from_numpy(ids).long() == idx).all()
    gate = torch.softmax(torch.gather(L, 1, idx), dim=-1)
    np.testing.assert_allclose(w, gate.numpy(), atol=1e-14)
    assert (ids != 0).all()  # the -5 bias keeps expert 0 out here
    # a constant bias selects exactly like no bias
    ids0, w0, _, _ = oracle.route(L.numpy(), 2)
    idsc, wc, _, _ = oracle.route(L.numpy(), 2, sel_bias=np.full(8, 2.5))
    assert (ids0 == idsc).all() and np.array_equal(w0, wc)


def test_update_bias_sign_rule_closed_form():
    b = oracle.update_bias(np.zeros(4), [10, 2, 0, 4], 0.01)  # mean 4
    np.testing.assert_array_equal(b, [-0.01, 0.01, 0.01, 0.0])


def test_bias_balancer_makes_load_more_uniform():
    """The chapter's demo: a hot expert, 200 steps of select + update; the
    final counts are far more uniform than at step 0 and the hot expert's
    bias ends negative."""
    rng = np.random.default_rng(0)
    N, E, k = 4096, 8, 2
    L = rng.normal(size=(N, E))
    L[:, 0] += 3.0
    bias = np.zeros(E)
    ids, _, _, _ = oracle.route(L, k, sel_bias=bias)
    c0 = np.bincount(ids.reshape(-1), minlength=E)
    for _ in range(200):
        ids, _, _, _ = oracle.route(L, k, sel_bias=bias)
        counts = np.bincount(ids.reshape(-1), minlength=E)
        bias = oracle.update_bias(bias, counts, 1e-2)
    assert counts.max() / counts.mean() < 0.5 * (c0.max() / c0.mean())
    assert bias[0] < 0


def _groups_reference(u, K, G, TG):
    """Independent formulation: rank groups by their best score with a stable
    sort, keep the first TG, then a stable descending sort of the eligible."""
    E = u.shape[0]
    gs = E // G
    gmax = np.array([u[g * gs:(g + 1) * gs].max() for g in range(G)])
    order = sorted(range(G), key=lambda g: (-gmax[g], g))
    keep = set(order[:TG])
    elig = [e for e in range(E) if e // gs in keep]
    return sorted(elig, key=lambda e: (-u[e], e))[:K]


@pytest.mark.parametrize("seed", range(4))
def test_group_limited_routing(seed):
    rng = np.random.default_rng(seed)
    T, E, K, G, TG = 40, 16, 4, 4, 2
    L = np.round(rng.normal(size=(T, E)) * 2, 1)  # some exact ties
    ids, w, _, _ = oracle.route(L, K, n_groups=G, topk_groups=TG)
    for t in range(T):
        assert ids[t].tolist() == _groups_reference(L[t], K, G, TG)
        assert len({e // (E // G) for e in ids[t]}) <= TG  # lab extension invariant
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-14)
    # one group, or all groups kept, is plain top-k
    a = oracle.route(L, K)
    for G2, TG2 in ((1, 1), (4, 4)):
        b = oracle.route(L, K, n_groups=G2, topk_groups=TG2)
        assert (a[0] == b[0]).all() and np.array_equal(a[1], b[1])


def test_route_scale_and_entropy_closed_forms():
    L = np.zeros((2, 8))
    _, w, _, _, ent = oracle.route(L, 2, route_scale=2.5, with_entropy=True)
    np.testing.assert_allclose(w, 1.25, atol=1e-15)
    np.testing.assert_allclose(ent, math.log(8), atol=1e-14)  # uniform: ln E
    L = np.zeros((1, 8))
    L[0, 3] = 900.0
    _, _, _, _, ent = oracle.route(L, 1, with_entropy=True)
    assert abs(ent[0]) < 1e-6  # one-hot: zero (up to the 1e-9 clamp)
