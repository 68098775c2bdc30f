"""Expert parallelism on the GPU path (one GPU: the exchange kernels against
their definition, and the whole layer at world size 1 over NCCL).

"Lab: build a tiny MoE in PyTorch", "From local loop to expert parallelism":
the distributed layer has the same output as the local one.  The multi-rank
exchange is covered on CPU ranks (tests/test_ep_cpu.py); here the CUDA
kernels of the receive layout and the row permutations are checked against
the definition, and the layer's product path (routing, dispatch, NCCL
all-to-all, layout, permutations, grouped experts, weighted combine) runs as
one rank against the oracle and against moe_forward_train, which weights the
expert outputs in the combine the same way.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from mixture_experts_layer_55_b200 import _binding as B
from mixture_experts_layer_55_b200.ep import ExpertParallelMoE
from workloads import WORKLOADS, Workload, make_inputs, make_tokens

from tests.test_ep_cpu import receive_layout
from tests.gpu_common import to_np

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("cuda_ok")]


@pytest.mark.parametrize("W,EL", [(4, 8), (2, 1), (8, 32)])
def test_receive_layout_and_permutation(W, EL):
    rng = np.random.default_rng(W * 100 + EL)
    recv = rng.integers(0, 40, size=(W, EL)).astype(np.int32)
    recv[0, 0] = 0          # empty segments, at the start and inside
    recv[W - 1, EL - 1] = 0
    n = int(recv.sum())
    max_rows = n + 17
    dev = "cuda"
    rc = torch.from_numpy(recv).to(dev)
    offsets = torch.empty(EL + 1, dtype=torch.int32, device=dev)
    dst_of = torch.full((max_rows,), -1, dtype=torch.int32, device=dev)
    src_of = torch.full((max_rows,), -1, dtype=torch.int32, device=dev)
    ws = torch.zeros(B.ep_workspace_size(W, EL), dtype=torch.uint8, device=dev)
    B.moe_ep_layout(W, EL, rc, max_rows, offsets, dst_of, src_of, ws)
    ref_off, ref_dst, ref_src = receive_layout(recv, W, EL)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(dst_of[:n].cpu().numpy(), ref_dst)
    np.testing.assert_array_equal(src_of[:n].cpu().numpy(), ref_src)
    # rows through both permutations come back bit-exactly
    D = 136  # 272-byte bf16 rows: 17 vectors of 16 bytes
    x = torch.randn(max(n, 1), D, device=dev).to(torch.bfloat16)
    xe = torch.empty_like(x)
    B.moe_permute_rows(x, src_of, n, xe, ws)
    back = torch.empty_like(x)
    B.moe_permute_rows(xe, dst_of, n, back, ws)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(ws) == 0
    idx = torch.from_numpy(ref_src).long().to(dev)
    assert torch.equal(xe[:n], x[idx])
    assert torch.equal(back[:n], x[:n])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("wl", [
    Workload("ep_w1", T=640, D=256, F=384, E=8, K=2),
    Workload("ep_w1_drops", T=512, D=256, F=256, E=8, K=2, capacity_factor=0.5, bias="zipf"),
], ids=lambda w: w.name)
def test_expert_parallel_one_rank(wl):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        inp = make_inputs(wl)
        g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        layer = ExpertParallelMoE(wl.T, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], wl.E,
                                  wl.K, wl.capacity_factor, router_bias=g["bias"])
        y = layer.forward(g["x"])
        torch.cuda.synchronize()
        assert layer.ops.status() == 0
        # the oracle, routed on the CUDA path's own logits
        cfg = layer.ops.cfg
        ws = torch.zeros(B.workspace_size(cfg), dtype=torch.uint8, device="cuda")
        L = torch.empty(wl.T, wl.E, device="cuda")
        ids = torch.empty(wl.T, wl.K, dtype=torch.int32, device="cuda")
        w = torch.empty(wl.T, wl.K, device="cuda")
        B.moe_route(cfg, g["x"], g["w_router"], ids, w, ws, router_bias=g["bias"], logits_out=L)
        ref = oracle.forward(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"],
                             wl.K, wl.capacity_factor, bias=inp["bias"], logits=L.cpu().numpy())
        got = to_np(y)
        m = float(np.abs(ref["y"]).max())
        assert np.abs(got - ref["y"]).max() <= 1e-2 * m + 1e-3
        # the same arithmetic as the training forward (weights applied in the combine)
        state = torch.zeros(B.train_state_size(cfg), dtype=torch.uint8, device="cuda")
        yt = torch.empty_like(g["x"])
        B.moe_forward_train(cfg, g["x"], g["w_router"], g["w_gate"], g["w_up"], g["w_down"], yt, state,
                            router_bias=g["bias"])
        torch.cuda.synchronize()
        assert np.abs(got - to_np(yt)).max() <= 1e-2 * m * 0.1 + 1e-4
    finally:
        dist.destroy_process_group()


# ------------------------------------------------ exchange over peer memory --

def _expected_remote_rows(kept_all, ids, row_of, offsets, rank, W, EL):
    """Where each slot of source `rank` lands in its owner's buffer, from the
    all-to-all path's definition: the rows for owner o leave in expert-major
    order, arrive after the rows of sources < rank, and the owner's receive
    layout moves arrival position p to expert-major row dst_of[p]."""
    E = W * EL
    K = ids.shape[1]
    out = np.full(ids.shape[0] * K, -1, np.int64)
    layouts = [receive_layout(kept_all[:, o * EL:(o + 1) * EL], W, EL) for o in range(W)]
    for t in range(ids.shape[0]):
        for k in range(K):
            r = row_of[t * K + k]
            if r < 0:
                continue
            o = ids[t, k] // EL
            recv_o = kept_all[:, o * EL:(o + 1) * EL]
            arrival = int(recv_o[:rank].sum()) + (r - offsets[o * EL])
            out[t * K + k] = layouts[o][1][arrival]
    return out, [lay[0] for lay in layouts]


def _emulated_peer_layer(wl, W, bias=None, token_seed=77, device_inputs=False):
    """W ranks of the peer-exchange layer emulated on one GPU: each rank has its
    own tokens; every rank's receive and output buffers live on this device,
    so the kernels' stores into and loads from "peer" buffers are ordinary
    device accesses.  The ranks' kernels run one after another in stream
    order; none waits on another.  device_inputs: draw the inputs on the GPU
    (full sizes; no host copies are kept)."""
    dev = "cuda"
    inp = make_inputs(wl, device=dev if device_inputs else "cpu")
    if bias is not None:
        inp["bias"] = bias
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    E, K, T, D, F = wl.E, wl.K, wl.T, wl.D, wl.F
    EL = E // W
    cfg = B.MoeConfig.make(T, D, F, E, K, wl.dtype, wl.capacity_factor)
    max_recv = W * T * K
    cfg_local = B.MoeConfig.make(max_recv, D, F, EL, 1, wl.dtype, 0.0)
    i32 = dict(dtype=torch.int32, device=dev)
    ranks = []
    for r in range(W):
        x = make_tokens(wl, device=dev if device_inputs else "cpu", seed=token_seed * 16 + r)
        st = dict(x_cpu=None if device_inputs else x, x=x.to(dev), ids=torch.empty(T, K, **i32),
                  w=torch.empty(T, K, dtype=torch.float32, device=dev),
                  counts=torch.empty(E, **i32), kept=torch.empty(E, **i32),
                  offsets=torch.empty(E + 1, **i32), perm=torch.empty(B.max_rows(cfg), **i32),
                  row_of=torch.empty(T * K, **i32), L=torch.empty(T, E, device=dev),
                  ws=torch.zeros(B.workspace_size(cfg), dtype=torch.uint8, device=dev),
                  ws_ep=torch.zeros(B.ep_workspace_size(W, EL), dtype=torch.uint8, device=dev),
                  local_offsets=torch.full((EL + 1,), -7, **i32),
                  remote_row=torch.full((T * K,), -7, **i32))
        B.moe_route(cfg, st["x"], g["w_router"], st["ids"], st["w"], st["ws"], router_bias=g["bias"],
                    logits_out=st["L"])
        B.moe_dispatch(cfg, None, st["ids"], st["counts"], st["kept"], st["offsets"], st["perm"],
                       st["row_of"], None, st["ws"])
        ranks.append(st)
    kept_all = torch.stack([st["kept"] for st in ranks]).reshape(-1).contiguous()
    recv = [torch.zeros(max_recv, D, dtype=wl.torch_dtype, device=dev) for _ in range(W)]
    outs = [torch.zeros(max_recv, D, dtype=wl.torch_dtype, device=dev) for _ in range(W)]
    recv_ptrs = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device=dev)
    out_ptrs = torch.tensor([t.data_ptr() for t in outs], dtype=torch.int64, device=dev)
    for r, st in enumerate(ranks):
        B.moe_ep_peer_dispatch(cfg, r, W, kept_all, st["x"], st["ids"], st["row_of"], st["offsets"],
                               recv_ptrs, max_recv, st["local_offsets"], st["remote_row"], st["ws_ep"])
    ws_local = torch.zeros(B.workspace_size(cfg_local), dtype=torch.uint8, device=dev)
    h = torch.empty(max_recv, F, dtype=wl.torch_dtype, device=dev)
    for o, st in enumerate(ranks):
        sl = slice(o * EL, (o + 1) * EL)
        B.moe_expert_ffn(cfg_local, recv[o], st["local_offsets"], None, None, g["w_gate"][sl],
                         g["w_up"][sl], g["w_down"][sl], h, outs[o], ws_local)
    for st in ranks:
        st["y"] = torch.empty_like(st["x"])
        B.moe_ep_peer_combine(cfg, W, st["ids"], st["remote_row"], st["w"], out_ptrs, max_recv, st["y"],
                              st["ws_ep"])
    torch.cuda.synchronize()
    for st in ranks:
        assert B.moe_get_device_status(st["ws"]) == 0
        assert B.moe_get_device_status(st["ws_ep"]) == 0
    assert B.moe_get_device_status(ws_local) == 0
    return cfg, inp, g, ranks, kept_all.view(W, E).cpu().numpy()


PEER_CASES = {
    "w2": (2, Workload("peer_w2", T=320, D=256, F=384, E=8, K=2), None),
    "w4_drops": (4, Workload("peer_w4_drops", T=256, D=256, F=256, E=8, K=2, capacity_factor=0.5,
                             bias="zipf"), None),
    "w8_one_expert_per_rank": (8, Workload("peer_w8", T=192, D=256, F=256, E=8, K=1), None),
    "w4_k4": (4, Workload("peer_w4_k4", T=160, D=256, F=256, E=16, K=4), None),
    "w2_k6": (2, Workload("peer_w2_k6", T=136, D=256, F=256, E=16, K=6), None),
    # every token prefers the last rank's experts: the other owners receive little or nothing
    "w4_skewed": (4, Workload("peer_w4_skew", T=192, D=256, F=256, E=8, K=2), "last_rank"),
}



def _random_peer_cases(n=8, seed=53):
    """Seeded random layers over emulated ranks: 2, 4 or 8 ranks, any number of local
    experts, K up to 8, ragged d_model and d_hidden, drops, a router bias."""
    import random
    rng = random.Random(seed)
    out = {}
    while len(out) < n:
        W = rng.choice([2, 4, 8])
        E = W * rng.choice([1, 2, 3, 4, 8])
        K = rng.randint(1, min(E, 8))
        T = rng.choice([1, 17, 100, 257])
        D = 8 * rng.randint(2, 48)
        F = 8 * rng.randint(2, 48)
        kw = dict(T=T, D=D, F=F, E=E, K=K, seed=700 + len(out))
        if rng.random() < 0.4:
            kw["capacity_factor"] = rng.choice([0.5, 1.0])
        if rng.random() < 0.4:
            kw["bias"] = "zipf"
        name = f"rand_w{W}_" + "_".join(f"{k}{v}" for k, v in kw.items() if k != "seed")
        out[name] = (W, Workload(name, **kw), None)
    return out


PEER_CASES.update(_random_peer_cases())


@pytest.mark.parametrize("name", sorted(PEER_CASES))
def test_peer_exchange_emulated_ranks(name):
    W, wl, skew = PEER_CASES[name]
    bias = None
    if skew == "last_rank":
        bias = torch.zeros(wl.E)
        bias[-(wl.E // W):] = 8.0
    cfg, inp, g, ranks, kept_all = _emulated_peer_layer(wl, W, bias=bias)
    EL = wl.E // W
    for r, st in enumerate(ranks):
        ids = st["ids"].cpu().numpy()
        row_of = st["row_of"].cpu().numpy()
        offsets = st["offsets"].cpu().numpy()
        exp_rows, exp_offsets = _expected_remote_rows(kept_all, ids, row_of, offsets, r, W, EL)
        np.testing.assert_array_equal(st["remote_row"].cpu().numpy(), exp_rows)
        np.testing.assert_array_equal(st["local_offsets"].cpu().numpy(), exp_offsets[r])
        # the output against the oracle's local layer on this rank's tokens
        ref = oracle.forward(st["x_cpu"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"],
                             wl.K, wl.capacity_factor, bias=inp["bias"], logits=st["L"].cpu().numpy())
        assert np.array_equal(ids, ref["ids"])
        assert np.array_equal(row_of, ref["row_of"])
        got = to_np(st["y"])
        m = float(np.abs(ref["y"]).max())
        assert np.abs(got - ref["y"]).max() <= 1e-2 * m + 1e-3
        # and against the local training forward (the same weighted combine)
        state = torch.zeros(B.train_state_size(cfg), dtype=torch.uint8, device="cuda")
        yt = torch.empty_like(st["x"])
        B.moe_forward_train(cfg, st["x"], g["w_router"], g["w_gate"], g["w_up"], g["w_down"], yt, state,
                            router_bias=g["bias"])
        torch.cuda.synchronize()
        assert np.abs(got - to_np(yt)).max() <= 1e-3 * m + 1e-4
    if name == "w4_drops":
        assert any((st["row_of"] < 0).any().item() for st in ranks), "case must drop assignments"
    if name == "w4_skewed":
        assert kept_all[:, : wl.E - EL].sum() == 0, "every row must go to the last rank"


def test_peer_exchange_full_size():
    """The Mixtral-shaped layer (T = 8192 tokens per rank, D = 4096, F = 14336,
    E = 8, K = 2) as two emulated ranks of four experts each: the receive
    layout against its definition, every output element against the local
    training forward of the same tokens (which weights the expert outputs in
    the combine the same way), and sampled tokens against the oracle (dropless
    routing makes each token's output depend on that token alone)."""
    wl = WORKLOADS["mixtral_8x"]
    W = 2
    cfg, inp, g, ranks, kept_all = _emulated_peer_layer(wl, W, device_inputs=True)
    EL = wl.E // W
    wg, wu, wd = (g[k].cpu() for k in ("w_gate", "w_up", "w_down"))
    for r, st in enumerate(ranks):
        ids = st["ids"].cpu().numpy()
        row_of = st["row_of"].cpu().numpy()
        offsets = st["offsets"].cpu().numpy()
        exp_rows, exp_offsets = _expected_remote_rows(kept_all, ids, row_of, offsets, r, W, EL)
        np.testing.assert_array_equal(st["remote_row"].cpu().numpy(), exp_rows)
        np.testing.assert_array_equal(st["local_offsets"].cpu().numpy(), exp_offsets[r])
        state = torch.zeros(B.train_state_size(cfg), dtype=torch.uint8, device="cuda")
        yt = torch.empty_like(st["x"])
        B.moe_forward_train(cfg, st["x"], g["w_router"], g["w_gate"], g["w_up"], g["w_down"], yt, state,
                            router_bias=g["bias"])
        torch.cuda.synchronize()
        assert B.moe_get_device_status(state) == 0
        got = to_np(st["y"])
        m = float(np.abs(got).max())
        assert np.abs(got - to_np(yt)).max() <= 1e-3 * m + 1e-4
        del state
        rng = np.random.default_rng(100 + r)
        tok = np.sort(rng.choice(wl.T, 3, replace=False))
        L = st["L"][torch.from_numpy(tok).cuda()].cpu().numpy()
        ref = oracle.forward(st["x"][torch.from_numpy(tok).cuda()].cpu(), g["w_router"].cpu(), wg, wu, wd,
                             wl.K, 0.0, logits=L)
        assert np.array_equal(ids[tok], ref["ids"])
        mref = float(np.abs(ref["y"]).max())
        assert np.abs(got[tok] - ref["y"]).max() <= 1e-2 * mref + 1e-3
    torch.cuda.empty_cache()


@pytest.mark.parametrize("wl", [
    Workload("peer_w1", T=640, D=256, F=384, E=8, K=2),
    Workload("peer_w1_drops", T=512, D=256, F=256, E=8, K=2, capacity_factor=0.5, bias="zipf"),
], ids=lambda w: w.name)
def test_peer_exchange_one_rank(wl):
    """The layer object with exchange='peer' at world size 1 over NCCL: the
    same output as the all-to-all exchange, twice in a row (the barriers and
    buffer reuse between steps), then the buffers released."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        inp = make_inputs(wl)
        g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        args = (wl.T, g["w_router"], g["w_gate"], g["w_up"], g["w_down"], wl.E, wl.K, wl.capacity_factor)
        peer = ExpertParallelMoE(*args, router_bias=g["bias"], exchange="peer")
        a2a = ExpertParallelMoE(*args, router_bias=g["bias"])
        for seed in (3, 4):
            x = make_tokens(wl, device="cuda", seed=seed)
            y_peer = peer.forward(x)
            y_a2a = a2a.forward(x)
            torch.cuda.synchronize()
            assert peer.ops.status() == 0 and a2a.ops.status() == 0
            m = float(y_a2a.float().abs().max())
            assert float((y_peer.float() - y_a2a.float()).abs().max()) <= 1e-3 * m + 1e-4
        peer.close()
    finally:
        dist.destroy_process_group()


def _ipc_child(handle, n, q):
    try:
        torch.cuda.set_device(0)
        from mixture_experts_layer_55_b200 import _binding as Bc
        ptr = Bc.ipc_open(handle)
        v = Bc.as_tensor(ptr, (n,), torch.int32)
        seen = bool(torch.equal(v.cpu(), torch.arange(n, dtype=torch.int32)))
        v.copy_(torch.arange(n, dtype=torch.int32, device="cuda") * 3)
        torch.cuda.synchronize()
        Bc.ipc_close(ptr)
        q.put((seen, None))
    except Exception as exc:  # pragma: no cover - reported by the parent
        q.put((False, repr(exc)))


def test_ipc_buffer_between_processes():
    """A buffer from moe_ipc_alloc, opened by another process from its handle
    (same GPU, one after the other: nothing waits on the other process)."""
    import torch.multiprocessing as mp
    n = 4096
    ptr, handle = B.ipc_alloc(n * 4)
    try:
        t = B.as_tensor(ptr, (n,), torch.int32)
        t.copy_(torch.arange(n, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        ctx = mp.get_context("spawn")
        q = ctx.Queue()
        p = ctx.Process(target=_ipc_child, args=(handle, n, q))
        p.start()
        seen, exc = q.get(timeout=240)
        p.join(timeout=60)
        assert exc is None, exc
        assert seen, "the other process read different values"
        assert torch.equal(t.cpu(), torch.arange(n, dtype=torch.int32) * 3)
    finally:
        B.ipc_free(ptr)
