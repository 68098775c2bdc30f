"""The multi-GPU path of bench.py on the CPU: two gloo ranks run the rank
logic (process group, barrier, max over ranks, per-rank token batches,
whole-job throughput) that N replicas use on GPUs."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from workloads import Workload, make_tokens
    r, w, lr = bench.rank_info()
    dist = bench.init_dist(w, "gloo")
    try:
        dev = torch.device("cpu")
        # each rank reports a different local time; all must see the max
        local_ms = 10.0 + 5.0 * r
        ms_total, ms_step, value = bench.aggregate(local_ms, w, 1000, 4, dev)
        bench.barrier(w)
        wl = Workload("t", T=8, D=16, F=16, E=4, K=2)
        x = make_tokens(wl, seed=bench.rank_token_seed(r))
        gathered = [torch.empty_like(x) for _ in range(w)]
        dist.all_gather(gathered, x)
        q.put((r, w, lr, ms_total, ms_step, value,
               all(not torch.equal(gathered[0], g) for g in gathered[1:])))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for r, (rank, world, lr, ms_total, ms_step, value, distinct) in enumerate(out):
        assert rank == r and world == 2 and lr == r
        assert ms_total == 15.0                      # max over ranks
        assert ms_step == pytest.approx(15.0 / 4)
        assert value == pytest.approx(2 * 1000 / (15.0 / 4 / 1e3))  # whole-job tokens/s
        assert distinct                              # each replica routes its own tokens


def test_single_rank_is_identity():
    import bench
    ms_total, ms_step, value = bench.aggregate(8.0, 1, 512, 2, torch.device("cpu"))
    assert ms_total == 8.0 and ms_step == 4.0 and value == pytest.approx(512 / 4e-3)
