"""Expert parallelism's exchange logic on CPU ranks (gloo, world sizes 2 and 4).

"Lab: build a tiny MoE in PyTorch", "From local loop to expert parallelism":
sort by owner -> exchange counts -> all-to-all -> grouped local experts ->
reverse all-to-all -> scatter-add, with the same output as the local layer.
Each rank holds E / W experts and its own tokens; the layer's device steps
(routing, dispatch, the receive layout, the experts, the combine) are given
here by the oracle and a plain statement of the receive layout, so the test
checks the data movement: every rank's output must equal the oracle's local
layer (all experts on one device) on that rank's tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


def receive_layout(recv, W, EL):
    """Expert-major offsets of the local experts and the maps between arrival
    (source-major) and expert-major order, written out from the definition."""
    recv = np.asarray(recv).reshape(W, EL)
    offsets = np.zeros(EL + 1, np.int64)
    for e in range(EL):
        offsets[e + 1] = offsets[e] + recv[:, e].sum()
    n = int(recv.sum())
    dst_of = np.zeros(n, np.int64)
    p = 0
    for s in range(W):
        for e in range(EL):
            start = offsets[e] + recv[:s, e].sum()
            for i in range(recv[s, e]):
                dst_of[p] = start + i
                p += 1
    src_of = np.zeros(n, np.int64)
    src_of[dst_of] = np.arange(n)
    return offsets, dst_of, src_of


class OracleOps:
    def __init__(self, T, E, K, cf, routing):
        self.T, self.E, self.K, self.cf, self.routing = T, E, K, cf, routing

    def route_dispatch(self, x, w_router, bias, sel_bias, noise):
        x = x.float()  # the tokens were drawn in fp32: exact
        L = oracle.router_logits(x, w_router, bias, noise)
        sb = None if sel_bias is None else sel_bias.numpy()
        ids, w, _, _ = oracle.route(L, self.K, sel_bias=sb, **self.routing)
        d = oracle.dispatch(ids, self.E, oracle.capacity(self.T, self.K, self.E, self.cf))
        self.w, self.row_of = w, d["row_of"]
        x_perm = torch.from_numpy(oracle.gather(x, d["perm"], self.K))
        return torch.from_numpy(d["kept"]), torch.from_numpy(d["offsets"]), x_perm

    def layout(self, recv_counts, W, EL):
        return receive_layout(recv_counts.numpy(), W, EL)

    def to_expert_major(self, x_recv, src_of, n):
        return x_recv[torch.from_numpy(src_of[:n])] if n else x_recv[:0]

    def to_arrival_order(self, y_loc, dst_of, n):
        return y_loc[torch.from_numpy(dst_of[:n])] if n else y_loc[:0]

    def experts(self, x_loc, offsets, wg, wu, wd):
        y = torch.zeros_like(x_loc)
        for e in range(len(offsets) - 1):
            a, b = int(offsets[e]), int(offsets[e + 1])
            if b > a:
                y[a:b] = torch.from_numpy(oracle.expert_rows(x_loc[a:b].numpy(), wg[e], wu[e], wd[e]))
        return y

    def combine(self, y_perm, x):
        return torch.from_numpy(oracle.combine(y_perm.numpy(), self.row_of, self.w, self.T, self.K))


def _inputs(T, D, F, E, seed, rank, skew):
    g = torch.Generator().manual_seed(seed)
    w_router = (torch.randn(D, E, generator=g) * 0.3).float()
    wg = (torch.randn(E, D, F, generator=g) * 0.2).float()
    wu = (torch.randn(E, D, F, generator=g) * 0.2).float()
    wd = (torch.randn(E, F, D, generator=g) * 0.2).float()
    bias = torch.zeros(E)
    if skew:  # every token prefers the experts of the last rank
        bias[-(E // 4 or 1):] = 8.0
    x = torch.randn(T, D, generator=torch.Generator().manual_seed(seed * 100 + rank)).float()
    return x, w_router, wg, wu, wd, bias


def _rank(rank, world, port, case, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        from mixture_experts_layer_55_b200.ep import ExpertParallelMoE
        T, D, F, E, K, cf, skew = case
        x, w_router, wg, wu, wd, bias = _inputs(T, D, F, E, 11, rank, skew)
        EL = E // world
        sl = slice(rank * EL, (rank + 1) * EL)
        layer = ExpertParallelMoE(T, w_router, wg[sl], wu[sl], wd[sl], E, K, cf, router_bias=bias,
                                  ops=OracleOps(T, E, K, cf, {}))
        y = layer.forward(x.double())
        ref = oracle.forward(x, w_router, wg, wu, wd, K, cf, bias=bias)
        err = float(np.abs(y.numpy() - ref["y"]).max())
        dropped = int((ref["row_of"] < 0).sum())
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, err, dropped, None))
    except Exception as exc:  # pragma: no cover - reported by the parent
        q.put((rank, None, None, repr(exc)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


CASES = {
    "even_w2": (2, (40, 16, 24, 8, 2, 0.0, False)),
    "drops_w2": (2, (48, 16, 24, 8, 2, 0.5, False)),
    "one_expert_per_rank_k2": (2, (30, 16, 24, 2, 2, 0.0, False)),
    "skewed_w4": (4, (32, 16, 24, 8, 2, 0.0, True)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_expert_parallel_equals_local_layer(name):
    world, case = CASES[name]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, err, dropped, exc in results:
        assert exc is None, f"rank {rank}: {exc}"
        assert err < 1e-12, f"rank {rank}: max error {err}"
    if name == "drops_w2":
        assert any(r[2] > 0 for r in results), "case must drop assignments"


def test_receive_layout_definition():
    """The layout's hand example: 2 sources x 2 local experts."""
    offsets, dst_of, src_of = receive_layout([[2, 1], [0, 3]], 2, 2)
    # arrival: s0e0 s0e0 s0e1 s1e1 s1e1 s1e1 -> expert-major: e0: s0,s0 | e1: s0, s1, s1, s1
    assert offsets.tolist() == [0, 2, 6]
    assert dst_of.tolist() == [0, 1, 2, 3, 4, 5]
    offsets, dst_of, src_of = receive_layout([[1, 2], [3, 0]], 2, 2)
    # arrival: s0e0 s0e1 s0e1 s1e0 s1e0 s1e0 -> e0: s0, s1, s1, s1 | e1: s0, s0
    assert offsets.tolist() == [0, 4, 6]
    assert dst_of.tolist() == [0, 4, 5, 1, 2, 3]
    assert src_of.tolist() == [0, 3, 4, 5, 1, 2]


def _peer_rows(kept_all, ids, row_of, offsets, rank, W, EL):
    """The peer exchange's placement as include/moe.h states it: slot (t, k) of
    source `rank`, routed to expert e of owner o = e // EL and kept at local row
    r, lands at  sum_{o*EL <= e' < e} sum_s kept[s][e'] + sum_{s < rank}
    kept[s][e] + (r - offsets[e])  of o's buffer."""
    out = np.full(row_of.shape, -1, np.int64)
    for i, r in enumerate(row_of):
        if r < 0:
            continue
        e = int(ids.reshape(-1)[i])
        o = e // EL
        out[i] = kept_all[:, o * EL:e].sum() + kept_all[:rank, e].sum() + (r - offsets[e])
    return out


@pytest.mark.parametrize("W,EL,seed", [(2, 4, 0), (4, 2, 1), (8, 1, 2), (3, 5, 3)])
def test_peer_placement_formula_equals_all_to_all_layout(W, EL, seed):
    """The closed-form placement of the peer exchange agrees with the all-to-all
    path's layout: rows leave each source expert-major, arrive source-major,
    and the owner's receive layout moves them to expert-major order."""
    rng = np.random.default_rng(seed)
    E, T, K = W * EL, 50, min(2, W * EL)
    kept_all = np.zeros((W, E), np.int64)
    for rank in range(W):
        ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)])
        d = oracle.dispatch(ids.astype(np.int32), E, oracle.capacity(T, K, E, 0.6))
        kept_all[rank] = d["kept"]
    # each source's own layout again, to place its slots
    rng = np.random.default_rng(seed)
    for rank in range(W):
        ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)])
        d = oracle.dispatch(ids.astype(np.int32), E, oracle.capacity(T, K, E, 0.6))
        got = _peer_rows(kept_all, ids, d["row_of"], d["offsets"], rank, W, EL)
        for i, r in enumerate(d["row_of"]):
            if r < 0:
                assert got[i] == -1
                continue
            o = int(ids.reshape(-1)[i]) // EL
            recv_o = kept_all[:, o * EL:(o + 1) * EL]
            arrival = int(recv_o[:rank].sum()) + (r - d["offsets"][o * EL])
            _, dst_of, _ = receive_layout(recv_o, W, EL)
            assert got[i] == dst_of[arrival]
