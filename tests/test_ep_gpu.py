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
from workloads import Workload, make_inputs

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
