"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small cases compare every output element by element; they span several
tiles and ragged tails, and two of them put three or more tiles through every
CTA pair.  The five full-size layer shapes (and the ST-MoE shape at capacity
factor 1.0, which drops) compare the routing and dispatch results in full,
and, through moe_forward, the call the benchmark times: every token of the
two small-T layers, and elsewhere a stratified sample that reaches every
(expert, 128-row block) of the grouped GEMMs plus the tokens with dropped
slots, compared on y, y_perm and x_perm.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_55_b200 import _binding as B
from tests.gpu_common import (Bufs, assert_close_out, check_logits, check_routing, check_tokens,
                              full_size_tokens, prepared_terms, to_np)
from workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def _wl(name, **kw):
    base = dict(T=300, D=136, F=200, E=8, K=2, dtype="bf16", seed=1)
    base.update(kw)
    return Workload(name, **base)


SMALL = [
    _wl("ragged_bf16"),
    _wl("ragged_f32", dtype="f32"),
    _wl("tiles_bf16", T=700, D=264, F=392, E=6, K=3, seed=2),  # several 128-row tiles, K/N tails
    _wl("fine_bias", T=512, D=128, F=72, E=64, K=6, bias="zipf", seed=3),
    _wl("capacity_drops", T=400, D=64, F=96, E=8, K=2, capacity_factor=0.5, noise=True, seed=4),
    _wl("capacity_f32", T=257, D=64, F=64, E=4, K=2, capacity_factor=0.3, dtype="f32", seed=5),
    _wl("k_equals_e", T=96, D=64, F=64, E=4, K=4, seed=6),
    _wl("e256_k8", T=40, D=256, F=128, E=256, K=8, seed=7),
    _wl("one_token", T=1, D=64, F=64, E=8, K=2, seed=8),
    _wl("top1", T=130, D=72, F=80, E=5, K=1, seed=9),
    _wl("one_expert", T=33, D=32, F=48, E=1, K=1, seed=10),
    # CTA-pair tiles (256 rows): chosen when experts average >= 128 rows
    _wl("pair_ragged", T=1200, D=200, F=392, E=4, K=2, seed=13),
    _wl("pair_skewed", T=1500, D=128, F=136, E=8, K=2, bias="zipf", seed=14),
    _wl("pair_drops", T=2000, D=64, F=256, E=8, K=2, capacity_factor=0.75, noise=True, seed=15),
    # three or more tiles through every CTA pair (74 pairs on 148 SMs), so each
    # tensor-memory accumulator buffer is reused and the operand ring wraps many
    # times: 256 gate/up tiles (4 m-tiles x 8 n-tiles x 8 experts), then 256
    # down tiles with the long d_model
    _wl("pair_reuse_gateup", T=4096, D=256, F=1024, E=8, K=2, seed=42),
    _wl("pair_reuse_down", T=4096, D=2048, F=256, E=8, K=2, seed=43),
    # tensor-core router (bf16, E <= 128, T >= 2048): ragged 128-token tail, E not
    # a multiple of 64, bias and noise, K = 8
    _wl("tcr_ragged", T=2500, D=136, F=64, E=8, K=2, seed=16),
    _wl("tcr_e100", T=2100, D=264, F=64, E=100, K=4, bias="zipf", noise=True, seed=17),
    _wl("tcr_e128_k8", T=2048, D=128, F=32, E=128, K=8, seed=18),
    # 16 token tiles would split d_model in two, but the leader's receive buffer for
    # 128 experts leaves the rings too small: the plan falls back to one split
    _wl("tcr_e128_split_fit", T=2048, D=1024, F=32, E=128, K=4, bias="zipf", seed=61),
    # more token tiles than SMs: two router CTAs per SM (shallower rings)
    _wl("tcr_two_per_sm", T=19200, D=136, F=32, E=24, K=3, noise=True, seed=44),
    _wl("tcr_two_per_sm_e64", T=19000, D=64, F=32, E=64, K=6, bias="zipf", seed=45),
    # tensor-core router split over d_model (few token tiles, long d_model): 2 splits with a
    # ragged last one, and 4 splits under the group limit, selection bias and sigmoid scores
    _wl("tcr_split2", T=2200, D=1088, F=64, E=8, K=2, bias="zipf", noise=True, seed=40),
    _wl("tcr_split4_groups", T=2048, D=2048, F=32, E=64, K=6, n_groups=8, topk_groups=3,
        sel_bias=True, score_func="sigmoid", seed=41),
    # router variants, SIMT router (T < 2048) and tensor-core router
    _wl("sigmoid_simt", T=300, E=16, K=3, score_func="sigmoid", seed=23),
    _wl("norenorm_scale_simt", T=300, E=8, K=2, renormalize=False, route_scale=2.5, seed=24),
    _wl("selbias_groups_simt", T=500, D=128, F=64, E=64, K=6, sel_bias=True, n_groups=8,
        topk_groups=3, seed=25),
    _wl("e256_groups_sigmoid_simt", T=64, D=256, F=64, E=256, K=8, n_groups=8, topk_groups=4,
        sel_bias=True, score_func="sigmoid", seed=26),
    _wl("sigmoid_selbias_tcr", T=2300, D=128, F=32, E=32, K=4, score_func="sigmoid",
        sel_bias=True, seed=27),
    _wl("groups_norenorm_tcr", T=2048, D=128, F=32, E=128, K=8, n_groups=8, topk_groups=4,
        renormalize=False, route_scale=1.5, bias="zipf", seed=28),
    # shared expert (one expert over every token, added in the combine)
    _wl("shared_bf16_pair", T=700, D=136, F=200, E=4, K=2, F_shared=264, seed=29),
    _wl("shared_f32", T=300, D=64, F=96, E=8, K=2, F_shared=72, dtype="f32", seed=30),
    _wl("shared_drops", T=400, D=64, F=96, E=8, K=2, capacity_factor=0.5, F_shared=128, seed=31),
    # few tokens, long d_model: the combine splits each row over several warps; a shared
    # expert's rows are added first and a capacity drop leaves a slot out
    _wl("split_combine", T=96, D=2048, F=64, E=8, K=3, F_shared=64, capacity_factor=0.6, seed=48),
    _wl("split_combine_f32", T=40, D=1024, F=32, E=4, K=2, dtype="f32", seed=49),
]


def _to_dev(inp):
    def dev(v):
        if v is None:
            return None
        if isinstance(v, tuple):
            return tuple(t.cuda() for t in v)
        return v.cuda()
    return {k: dev(v) for k, v in inp.items()}


def _random_layer_cases(n=32, seed=77):
    """Seeded random layers for the whole forward: bf16 and fp32, T from 1 token to
    past the tensor-core router's threshold, d_model and d_hidden any multiple of 8
    (ragged K and N tiles), 1 to 256 experts (single CTAs and CTA pairs), capacity
    drops, every routing option, sometimes a shared expert."""
    import random
    rng = random.Random(seed)
    cases = []
    while len(cases) < n:
        dtype = "f32" if rng.random() < 0.25 else "bf16"
        E = rng.choice([1, 2, 3, 5, 8, 13, 16, 32, 64, 100, 256])
        K = rng.randint(1, min(E, 8))
        T = rng.choice([1, 7, 100, 333, 1000, 2049, 3000])
        D = 8 * rng.randint(1, 66)
        F = 8 * rng.randint(1, 66)
        if T * K * D * F > 2_000_000_000:
            continue
        kw = dict(T=T, D=D, F=F, E=E, K=K, dtype=dtype, seed=500 + len(cases))
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
            kw["F_shared"] = 8 * rng.randint(1, 40)
        name = "rand_" + "_".join(f"{k}{v}" for k, v in kw.items() if k != "seed")
        cases.append(_wl(name, **kw))
    return cases


RANDOM_LAYERS = _random_layer_cases()


@pytest.mark.parametrize("wl", SMALL + RANDOM_LAYERS, ids=[w.name for w in SMALL + RANDOM_LAYERS])
def test_small_layers_elementwise(cuda_ok, wl):
    inp_cpu = make_inputs(wl, device="cpu")
    inp = _to_dev(inp_cpu)
    b = Bufs(wl)
    b.run_ops(inp)
    check_logits(wl, inp_cpu, b.logits.cpu().numpy())
    rt = check_routing(wl, b, inp_cpu["sel_bias"])
    sb = None if inp_cpu["sel_bias"] is None else inp_cpu["sel_bias"].double().numpy()
    ref = oracle.forward(inp_cpu["x"], inp_cpu["w_router"], inp_cpu["w_gate"], inp_cpu["w_up"],
                         inp_cpu["w_down"], wl.K, wl.capacity_factor, inp_cpu["bias"],
                         inp_cpu["noise"], logits=b.logits.cpu().numpy(), sel_bias=sb,
                         shared=inp_cpu["shared"], **wl.routing())
    R = int(ref["offsets"][-1])
    # dispatch gather: exact copies
    assert torch.equal(b.x_perm[:R].cpu().to(torch.float64),
                       torch.from_numpy(ref["x_perm"])), "x_perm differs"
    # expert outputs with the routing weight applied
    assert_close_out(wl, to_np(b.y_perm[:R]), ref["o"] * ref["row_weight"][:, None], "y_perm")
    assert_close_out(wl, to_np(b.y), ref["y"], "y")
    # dropped-everything tokens get exactly zero from the routed experts (so
    # exactly the shared expert's output when there is one)
    kept = ref["row_of"].reshape(wl.T, wl.K) >= 0
    none = np.nonzero(~kept.any(1))[0]
    if none.size:
        if b.y_shared is None:
            assert (to_np(b.y[none]) == 0).all()
        else:
            assert torch.equal(b.y[none], b.y_shared[none])
    # the whole layer in one call gives the same bits as the op-by-op path (the
    # latter splits the router weight inside moe_route; here it is prepared once)
    ws = torch.zeros(B.forward_workspace_size(b.cfg), dtype=torch.uint8, device="cuda")
    y2 = torch.empty_like(b.y)
    losses = torch.empty(3, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    terms = prepared_terms(b.cfg, inp["w_router"])
    B.moe_forward(b.cfg, inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], y2,
                  ws, router_bias=inp["bias"], logit_noise=inp["noise"], losses=losses,
                  counts=counts, selection_bias=inp["sel_bias"], shared=inp["shared"],
                  w_router_terms=terms)
    torch.cuda.synchronize()
    assert torch.equal(y2, b.y)
    assert torch.equal(losses, b.losses)
    assert torch.equal(counts, b.counts)
    assert B.moe_get_device_status(ws) == 0


def test_parity_mode_routes_given_logits(cuda_ok):
    """logits_in: the router kernel routes exactly the logits it is given,
    ties included (tie rule: lower expert id)."""
    wl = _wl("given_logits", T=200, E=16, K=4, seed=11)
    inp = _to_dev(make_inputs(wl, device="cpu"))
    g = torch.Generator().manual_seed(3)
    L = torch.round(torch.randn(wl.T, wl.E, generator=g) * 2) / 2  # many exact ties
    L[:5] = 0.0  # all-equal rows
    b = Bufs(wl)
    b.run_ops(inp, logits_in=L.cuda())
    rt = check_routing(wl, b)
    assert (rt["ids"][:5] == np.arange(4)[None, :]).all()


def test_tensor_core_router_ties(cuda_ok):
    """Exact ties through the fused tensor-core router: a zero router weight and
    a bias with repeated values; the lower expert id must win every tie."""
    wl = _wl("tcr_ties", T=2048, D=64, F=32, E=16, K=5, seed=19)
    inp_cpu = make_inputs(wl, device="cpu")
    inp_cpu["w_router"] = torch.zeros_like(inp_cpu["w_router"])
    inp_cpu["bias"] = torch.tensor([0., 1, 1, 0, 2, 1, 0, 2, 1, 0, 0, 2, 1, 1, 0, 2])
    inp = _to_dev(inp_cpu)
    b = Bufs(wl)
    b.run_ops(inp)
    rt = check_routing(wl, b)
    # bias 2 at experts 4, 7, 11, 15; then bias 1 at 1, 2, 5, ...
    assert (rt["ids"] == np.array([4, 7, 11, 15, 1])[None, :]).all()
    np.testing.assert_array_equal(b.logits.cpu().numpy(), np.broadcast_to(
        inp_cpu["bias"].numpy(), (wl.T, wl.E)))


def test_update_selection_bias_matches_oracle(cuda_ok):
    """DeepSeek-V3 balancing step on the device against the oracle's update,
    with one count exactly at the mean (its bias must not move)."""
    wl = _wl("upd", T=64, E=8, K=2)
    cfg = B.MoeConfig.make(wl.T, wl.D, wl.F, wl.E, wl.K)
    counts = torch.tensor([40, 3, 16, 0, 16, 25, 12, 16], dtype=torch.int32)  # mean 16
    bias0 = torch.linspace(-0.5, 0.5, 8, dtype=torch.float32)
    b = bias0.cuda()
    B.moe_update_selection_bias(cfg, counts.cuda(), 0.125, b)
    torch.cuda.synchronize()
    ref = oracle.update_bias(bias0.double().numpy(), counts.numpy(), 0.125)
    np.testing.assert_allclose(b.cpu().double().numpy(), ref, rtol=0, atol=1e-7)
    assert float(b[2]) == float(bias0[2])


def test_unaligned_router_weight(cuda_ok):
    """A router weight that is not 16-byte aligned: the weight split reads it
    with plain loads, so the tensor-core router still serves the layer, with
    the same results against the oracle."""
    wl = _wl("unaligned_wr", T=2304, D=128, F=32, E=12, K=3, bias="zipf", seed=47)
    inp_cpu = make_inputs(wl, device="cpu")
    inp = _to_dev(inp_cpu)
    buf = torch.empty(wl.D * wl.E + 1, device="cuda")
    w_un = buf[1:].view(wl.D, wl.E)
    w_un.copy_(inp["w_router"])
    assert w_un.data_ptr() % 16 != 0
    inp["w_router"] = w_un
    b = Bufs(wl)
    b.run_ops(inp)
    check_logits(wl, inp_cpu, b.logits.cpu().numpy())
    check_routing(wl, b)


def _split3_cpu(w):
    """The three bf16 terms of fp32 weights, as the pages' fp32 logits need them
    written exactly: hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid),
    each rounded to nearest even (torch's float -> bfloat16 conversion)."""
    hi = w.bfloat16()
    r = w - hi.float()
    mid = r.bfloat16()
    lo = (r - mid.float()).bfloat16()
    return hi, mid, lo


@pytest.mark.parametrize("E", [8, 24, 100])
def test_router_prepare_writes_the_exact_terms(cuda_ok, E):
    """moe_router_prepare: terms[p][e][d] (p = hi, mid, lo; e < E16, rows past E
    zero) equal the exact three-term split of W_r computed on the CPU, bit for bit."""
    D = 200
    cfg = B.MoeConfig.make(4096, D, 64, E, 2, "bf16")
    g = torch.Generator().manual_seed(E)
    w = torch.randn(D, E, generator=g) * 0.02
    w[0, 0] = 1.0 + 2.0 ** -9 + 2.0 ** -18  # a value whose split needs all three terms
    terms = torch.empty(B.router_terms_size(cfg), dtype=torch.uint8, device="cuda")
    B.moe_router_prepare(cfg, w.cuda(), terms)
    torch.cuda.synchronize()
    e16 = B.router_terms_size(cfg) // (3 * D * 2)
    assert e16 >= E and e16 in (16, 32, 64, 128)
    got = terms.view(torch.bfloat16).view(3, e16, D).cpu()
    for p, ref in enumerate(_split3_cpu(w)):
        assert torch.equal(got[p, :E].view(torch.int16), ref.t().contiguous().view(torch.int16)), p
        assert (got[p, E:].view(torch.int16) == 0).all()
    # the three terms add up to the weight exactly (24 significand bits in 3 x 8)
    s = got[0, :E].double() + got[1, :E].double() + got[2, :E].double()
    assert torch.equal(s, w.t().double())


def test_layer_prepares_the_router_terms_again_after_an_update(cuda_ok):
    """MoELayer splits w_router once; after the weight is changed in place (its
    version counter moves) or replaced, the next forward uses the new terms: the
    same bits as a layer built on the new weight."""
    from mixture_experts_layer_55_b200 import MoELayer
    wl = _wl("terms_refresh", T=2304, D=128, F=64, E=16, K=2, seed=62)
    inp = _to_dev(make_inputs(wl, device="cpu"))
    layer = MoELayer(wl.T, inp["w_router"].clone(), inp["w_gate"], inp["w_up"], inp["w_down"], wl.K)
    x = inp["x"]
    y0 = layer.forward(x).clone()
    layer.w_router.mul_(-1.5)  # in place: new routing
    y1 = layer.forward(x).clone()
    ref = MoELayer(wl.T, inp["w_router"] * -1.5, inp["w_gate"], inp["w_up"], inp["w_down"], wl.K)
    torch.cuda.synchronize()
    assert torch.equal(y1, ref.forward(x))
    assert not torch.equal(y0, y1)
    layer.w_router = inp["w_router"].clone()  # replaced: back to the first routing
    assert torch.equal(layer.forward(x), y0)
    assert B.moe_get_device_status(layer.workspace) == 0


def _random_router_cases(n=20, seed=2024):
    """Seeded random shapes for the tensor-core router (bf16, T >= 2048, E <= 128):
    any E (so E16 = 16, 32, 64 or 128 and ragged expert rows), d_model splits or
    none, one or two CTAs per SM, and the options (bias, noise, sigmoid scores,
    no renormalisation, selection bias, group limit)."""
    import random
    rng = random.Random(seed)
    cases = []
    while len(cases) < n:
        E = rng.choice([1, 3, 8, 13, 16, 24, 33, 50, 64, 77, 100, 128])
        K = rng.randint(1, min(E, 8))
        T = rng.choice([2048, 2049, 3000, 5000, 9000, 19000])
        D = rng.choice([64, 136, 264, 520, 1032, 2056])
        if T * D * E > 1_500_000_000:
            continue
        kw = dict(T=T, D=D, F=32, E=E, K=K, seed=300 + len(cases))
        if rng.random() < 0.4:
            kw["bias"] = "zipf"
        if rng.random() < 0.4:
            kw["noise"] = True
        if rng.random() < 0.3:
            kw["score_func"] = "sigmoid"
        if rng.random() < 0.3:
            kw["renormalize"] = False
        if rng.random() < 0.3:
            kw["sel_bias"] = True
        groups = [g for g in (2, 4, 8) if E % g == 0 and E // g >= 1]
        if groups and rng.random() < 0.3:
            g = rng.choice(groups)
            tg = rng.randint(1, g)
            if tg * (E // g) >= K:
                kw["n_groups"], kw["topk_groups"] = g, tg
        name = "rand_" + "_".join(f"{k}{v}" for k, v in kw.items() if k not in ("F", "seed"))
        cases.append(_wl(name, **kw))
    return cases


RANDOM_ROUTER = _random_router_cases() + [
    _wl("rand_T2048_D64_E1_K1", T=2048, D=64, F=32, E=1, K=1, seed=330),
    _wl("rand_T2100_D136_E3_K3_noise_sigmoid", T=2100, D=136, F=32, E=3, K=3, noise=True,
        score_func="sigmoid", seed=331),
]


@pytest.mark.parametrize("wl", RANDOM_ROUTER, ids=[w.name for w in RANDOM_ROUTER])
def test_tensor_core_router_random_shapes(cuda_ok, wl):
    """Logits within the fp32 bound and every routing output bit-exact (ids,
    weights and probabilities within 1e-5, statistics, counts) against the
    oracle, over seeded random shapes and options of the tensor-core router."""
    assert B.check_config(B.MoeConfig.make(wl.T, wl.D, wl.F, wl.E, wl.K, wl.dtype,
                                           wl.capacity_factor, **wl.routing())) == B.MOE_OK
    inp_cpu = make_inputs(wl, device="cpu")
    inp = _to_dev(inp_cpu)
    b = Bufs(wl)
    b.run_ops(inp)
    check_logits(wl, inp_cpu, b.logits.cpu().numpy())
    check_routing(wl, b, inp["sel_bias"])


def test_dispatch_index_three_kernel_path(cuda_ok):
    """More chunks of 2048 assignments than SMs (T*K = 320000): the index pass
    runs as three kernels instead of one cooperative launch; routing, counts,
    kept, offsets, perm and row_of are bit-exact against the oracle, with drops."""
    wl = _wl("many_chunks", T=160000, D=64, F=32, E=8, K=2, capacity_factor=1.0, noise=True,
             seed=46)
    inp = _to_dev(make_inputs(wl, device="cpu"))
    b = Bufs(wl)
    b.run_ops(inp)
    rt = check_routing(wl, b)
    assert int((rt["row_of"] < 0).sum()) > 0
    R = int(rt["offsets"][-1])
    src = torch.from_numpy(rt["perm"][:R] // wl.K).long().cuda()
    assert torch.equal(b.x_perm[:R], inp["x"].index_select(0, src))


def test_determinism_bitwise(cuda_ok):
    wl = _wl("det", T=1000, D=128, F=128, E=16, K=4, bias="zipf", seed=12)
    inp = _to_dev(make_inputs(wl, device="cpu"))
    outs = []
    for _ in range(2):
        b = Bufs(wl)
        b.run_ops(inp)
        outs.append((b.y.clone(), b.losses.clone(), b.mean_prob.clone(), b.perm.clone()))
    for a, c in zip(*outs):
        assert torch.equal(a, c)


@pytest.mark.parametrize("wl", [
    _wl("inv_tcr_pairs", T=4096, D=256, F=512, E=8, K=2, bias="zipf", seed=81),
    _wl("inv_simt_single", T=600, D=136, F=200, E=16, K=4, seed=82),
    _wl("inv_f32", T=512, D=64, F=96, E=8, K=2, dtype="f32", seed=83),
    _wl("inv_shared", T=2048, D=128, F=256, E=4, K=2, F_shared=128, seed=84),
], ids=lambda w: w.name)
def test_batch_invariance_at_a_fixed_batch_size(cuda_ok, wl):
    """Dropless layers: a token's output depends on that token alone, and the
    kernels sum every output element in an order fixed by the shape, so the
    same token gives the same bits whatever the other tokens of a batch of the
    same size are (they change every expert's row count and so the tiles its
    rows land in)."""
    inp = _to_dev(make_inputs(wl, device="cpu"))
    cfg = B.MoeConfig.make(wl.T, wl.D, wl.F, wl.E, wl.K, wl.dtype, wl.capacity_factor,
                           F_shared=wl.F_shared, **wl.routing())
    ws = torch.zeros(B.forward_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    terms = prepared_terms(cfg, inp["w_router"])
    half = wl.T // 2
    x1 = inp["x"]
    g = torch.Generator(device="cuda").manual_seed(wl.seed + 1000)
    x2 = x1.clone()
    x2[half:] = (torch.randn(wl.T - half, wl.D, generator=g, device="cuda") * 3.0).to(x1.dtype)
    x2[:half] = x1[:half].flip(0)  # the shared tokens also move to other rows
    ys = []
    for x in (x1, x2):
        y = torch.empty_like(x)
        B.moe_forward(cfg, x, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], y, ws,
                      router_bias=inp["bias"], shared=inp["shared"], w_router_terms=terms)
        ys.append(y)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(ws) == 0
    assert torch.equal(ys[1][:half].flip(0), ys[0][:half])
    assert not torch.equal(ys[1][half:], ys[0][half:])


@pytest.mark.parametrize("wl", [
    _wl("bad_offsets_pair", T=600, D=128, F=136, E=4, K=2, seed=85),
    _wl("bad_offsets_single", T=100, D=72, F=64, E=8, K=2, seed=86),
    _wl("bad_offsets_f32", T=200, D=64, F=64, E=4, K=2, dtype="f32", seed=87),
], ids=lambda w: w.name)
def test_malformed_offsets_raise_bounds_flag(cuda_ok, wl):
    """Row offsets that decrease or run past max_rows, handed straight to
    moe_expert_ffn: the GEMM kernels' own checks treat those expert blocks as
    empty and raise the bounds flag (the per-expert A maps are clamped to the
    buffer as well); after the flag is cleared a well-formed call runs clean."""
    inp = _to_dev(make_inputs(wl, device="cpu"))
    b = Bufs(wl)
    b.run_ops(inp)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(b.ws) == 0
    R = b.max_rows
    good = b.offsets.clone()
    bad = good.clone()
    bad[1] = min(int(good[2]) + 5, R)     # expert 0 runs past expert 1's start...
    bad[2] = max(int(good[1]) - 3, 0)     # ...and expert 1's block ends before it begins
    bad[wl.E - 1] = R + 77                # past the buffers
    B.moe_expert_ffn(b.cfg, b.x_perm, bad, b.perm, b.w, inp["w_gate"], inp["w_up"], inp["w_down"],
                     b.h, b.y_perm, b.ws)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(b.ws) & 0x2
    B.moe_clear_device_status(b.ws)
    B.moe_expert_ffn(b.cfg, b.x_perm, good, b.perm, b.w, inp["w_gate"], inp["w_up"], inp["w_down"],
                     b.h, b.y_perm, b.ws)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(b.ws) == 0


def test_out_of_range_ids_raise_bounds_flag(cuda_ok):
    """Corrupt ids are caught by the dispatch kernels' own bounds checks: the
    status word gets the bounds flag and nothing is written out of range."""
    wl = _wl("bad_ids", T=64, E=8, K=2)
    b = Bufs(wl)
    ids = torch.randint(0, 8, (wl.T, wl.K), dtype=torch.int32)
    ids[5, 1] = 11
    ids[9, 0] = -3
    b.ids.copy_(ids)
    B.moe_dispatch(b.cfg, None, b.ids, b.counts, b.kept, b.offsets, b.perm, b.row_of, None, b.ws)
    flags = B.moe_get_device_status(b.ws)
    assert flags & 0x2
    row_of = b.row_of.cpu().numpy().reshape(wl.T, wl.K)
    assert row_of[5, 1] == -1 and row_of[9, 0] == -1
    assert int(b.counts.sum()) == wl.T * wl.K - 2
    B.moe_clear_device_status(b.ws)
    assert B.moe_get_device_status(b.ws) == 0


# ------------------------------------------------------------- full sizes --

FULL = ["tiny_fp32", "mixtral_8x", "fine_skewed", "stmoe_capacity", "decode_e256",
        "stmoe_capacity_cf1"]


def _full_workload(name):
    if name == "stmoe_capacity_cf1":
        # the ST-MoE shape at capacity factor 1.0: C = 2048 against a hottest
        # expert of about 2290 assignments, so the token-order drop rule runs
        # on a 32768-token layer with hundreds of tiles per GEMM
        return WORKLOADS["stmoe_capacity"].with_(name=name, capacity_factor=1.0)
    return WORKLOADS[name]


@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(cuda_ok, capsys, name):
    wl = _full_workload(name)
    torch.manual_seed(0)
    inp = make_inputs(wl, device="cuda")
    b = Bufs(wl)
    b.run_ops(inp)
    rt = check_routing(wl, b, inp["sel_bias"])
    # the benchmark's call: the whole layer through moe_forward, the router
    # weight prepared once
    ws = torch.zeros(B.forward_workspace_size(b.cfg), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(b.y)
    losses = torch.empty(3, device="cuda")
    B.moe_forward(b.cfg, inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], y,
                  ws, router_bias=inp["bias"], logit_noise=inp["noise"], losses=losses,
                  w_router_terms=prepared_terms(b.cfg, inp["w_router"]))
    torch.cuda.synchronize()
    assert B.moe_get_device_status(ws) == 0
    assert torch.equal(y, b.y), "moe_forward differs from the op-by-op path"
    n_drop = int((rt["row_of"] < 0).sum())
    if wl.T <= 512:
        # the tiny fp32 layer and the decode layer: every token
        tokens, rows, blocks, tiles = list(range(wl.T)), None, None, None
    else:
        # every (expert, 128-row block) of the grouped GEMMs, each expert's first
        # and last row, and the tokens with dropped slots
        tokens, rows, blocks, tiles = full_size_tokens(wl, rt)
    err, tol, compared = check_tokens(wl, inp, rt, tokens, y, y_perm=b.y_perm, x_perm=b.x_perm)
    R = int(rt["offsets"][-1])
    if rows is not None:
        assert set(rows) <= set(compared), "a stratified row was not compared"
    else:
        assert sorted(compared) == list(range(R)), "every kept row should be compared"
    if wl.capacity_factor > 0:
        assert rt["C"] == int(np.ceil(wl.capacity_factor * wl.T * wl.K / wl.E))
    if name == "stmoe_capacity_cf1":
        assert rt["C"] == 2048 and n_drop > 0, "capacity factor 1.0 should drop assignments"
    with capsys.disabled():
        cov = (f"all {R} kept rows" if rows is None else
               f"{len(compared)} of {R} kept rows; every one of the {blocks} (expert, 128-row) "
               f"blocks = {tiles} (expert, 256-row tile) pairs")
        print(f"\n[full-size parity] {name}: {len(tokens)} tokens, {cov}; "
              f"{n_drop} dropped slots; max err {err:.3e} (tol {tol:.3e})")
    del inp
    torch.cuda.empty_cache()


def test_bounded_wait_gives_up_and_reports(cuda_ok):
    """The device failure path: a wait on a barrier nothing arrives at gives up
    after its limit (20 ms here), the status word reports the timeout and its
    location, and the context keeps working (a layer forward runs after it)."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    B.moe_selftest_wait_timeout(ws, 20_000_000)
    flags = B.moe_get_device_status(ws)
    assert flags & 0x1
    words = ws.view(torch.int32).cpu()
    assert int(words[1]) == 900 and int(words[2]) == 1
    B.moe_clear_device_status(ws)
    assert B.moe_get_device_status(ws) == 0
    wl = _wl("after_timeout", T=64, E=4, K=2, seed=21)
    b = Bufs(wl)
    b.run_ops(_to_dev(make_inputs(wl, device="cpu")))


def test_host_stream_matches_device_forward(cuda_ok):
    """MoELayer.forward_host_stream (pipelined copies in / forward / copies out)
    returns, for every batch, the same bits as the device-resident forward."""
    from mixture_experts_layer_55_b200 import MoELayer
    from workloads import make_tokens
    wl = _wl("host_stream", T=512, D=128, F=256, E=8, K=2, seed=22)
    inp = _to_dev(make_inputs(wl, device="cpu"))
    layer = MoELayer(wl.T, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], wl.K)
    xs = [make_tokens(wl, seed=100 + i) for i in range(5)]
    x_hosts = [x.pin_memory() for x in xs]
    y_hosts = [torch.empty_like(x).pin_memory() for x in xs]
    layer.forward_host_stream(x_hosts, y_hosts)
    torch.cuda.synchronize()
    for x, yh in zip(xs, y_hosts):
        y = layer.forward(x.cuda())
        torch.cuda.synchronize()
        assert torch.equal(y.cpu(), yh)


@pytest.mark.parametrize("name", ["tiny_fp32", "ragged_bf16"])
def test_cuda_graph_replay_matches_eager(cuda_ok, name):
    """MoELayer.capture: the whole forward as one CUDA graph; replays on new
    contents of the captured input give the eager forward's output bit for bit."""
    from mixture_experts_layer_55_b200 import MoELayer
    from workloads import make_tokens
    wl = WORKLOADS[name] if name in WORKLOADS else next(w for w in SMALL if w.name == name)
    inp = _to_dev(make_inputs(wl))
    layer = MoELayer(wl.T, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], wl.K,
                     wl.capacity_factor, router_bias=inp["bias"])
    x = inp["x"].clone()
    y = torch.empty_like(x)
    graph = layer.capture(x, y)
    for seed in (11, 12):
        xn = make_tokens(wl, device="cuda", seed=seed)
        x.copy_(xn)
        graph.replay()
        y_eager = layer.forward(xn)
        torch.cuda.synchronize()
        assert torch.equal(y, y_eager)
    assert B.moe_get_device_status(layer.workspace) == 0
