"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device
memory (for example a plugin that a host framework hands only its input and
output buffers, on a fixed memory budget, where cudaMalloc would synchronise
the device and fall outside that budget).  Its scratch is a static device
array inside the library, so it takes no workspace.

The GPU test calls it through the C ABI twice in a row, on different routings,
and checks each result against moe_dispatch (with a workspace): the index
arrays and the gathered rows are integer or copy work, so they must match
bit for bit; the static array's status word must stay clear.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from mixture_experts_layer_55_b200 import _binding as B
from mixture_experts_layer_55_b200 import build as build_mod


def _cfg(**kw):
    base = dict(T=3000, D=256, F=128, E=16, K=4, dtype="bf16", capacity_factor=0.9)
    base.update(kw)
    return B.MoeConfig.make(**base)


def test_rejects_problems_beyond_the_static_scratch():
    """Host-side check, before any device work: 2*ceil(T*K/2048)*E words + 256 B
    must fit in 256 KiB."""
    build_mod.build()
    lib = B.lib()
    FAKE = 0x10000
    big = _cfg(T=2_000_000, K=8, E=256)
    st = lib.moe_dispatch_noalloc(ctypes.byref(big), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  None, None)
    assert st == B.MOE_ERR_WORKSPACE
    bad = _cfg(K=0)
    st = lib.moe_dispatch_noalloc(ctypes.byref(bad), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  None, None)
    assert st == B.MOE_ERR_ARG
    assert lib.moe_dispatch_noalloc_status(None, None) == B.MOE_ERR_ARG


def _outputs(cfg, dev):
    T, K, E, D = cfg.T, cfg.K, cfg.E, cfg.D
    R = B.max_rows(cfg)
    i32 = torch.int32
    return dict(counts=torch.full((E,), -1, dtype=i32, device=dev),
                kept=torch.full((E,), -1, dtype=i32, device=dev),
                offsets=torch.full((E + 1,), -1, dtype=i32, device=dev),
                perm=torch.full((R,), -1, dtype=i32, device=dev),
                row_of=torch.full((T * K,), -5, dtype=i32, device=dev),
                x_perm=torch.zeros(R, D, dtype=torch.bfloat16, device=dev))


@pytest.mark.gpu
def test_noalloc_dispatch_matches_workspace_dispatch_twice(cuda_ok):
    build_mod.build()
    dev = torch.device("cuda", 0)
    cfg = _cfg()
    g = torch.Generator(device=dev).manual_seed(77)
    ws = torch.zeros(B.workspace_size(cfg), dtype=torch.uint8, device=dev)
    for call in range(2):
        x = torch.randn(cfg.T, cfg.D, generator=g, device=dev).to(torch.bfloat16)
        w_router = torch.randn(cfg.D, cfg.E, generator=g, device=dev) * 0.05
        ids = torch.empty(cfg.T, cfg.K, dtype=torch.int32, device=dev)
        tw = torch.empty(cfg.T, cfg.K, device=dev)
        B.moe_route(cfg, x, w_router, ids, tw, ws)
        ref = _outputs(cfg, dev)
        B.moe_dispatch(cfg, x, ids, ref["counts"], ref["kept"], ref["offsets"], ref["perm"],
                       ref["row_of"], ref["x_perm"], ws)
        got = _outputs(cfg, dev)
        B.moe_dispatch_noalloc(cfg, x, ids, got["counts"], got["kept"], got["offsets"],
                               got["perm"], got["row_of"], got["x_perm"])
        torch.cuda.synchronize(dev)
        assert B.moe_get_device_status(ws) == 0
        assert B.moe_dispatch_noalloc_status() == 0  # the static array's own status word
        R = int(ref["offsets"][-1])
        assert R > 0 and int(ref["kept"].sum()) == R
        assert int((ref["row_of"] < 0).sum()) > 0, "the capacity factor should drop assignments"
        for k in ("counts", "kept", "offsets", "row_of"):
            assert torch.equal(got[k], ref[k]), f"call {call}: {k} differs"
        assert torch.equal(got["perm"][:R], ref["perm"][:R]), f"call {call}: perm differs"
        assert torch.equal(got["x_perm"][:R], ref["x_perm"][:R]), f"call {call}: x_perm differs"


@pytest.mark.gpu
def test_noalloc_status_reports_a_corrupt_id_and_clears(cuda_ok):
    """An expert id out of range is skipped by the device range check, which sets
    the bounds flag in the static array's status word; the next clean call starts
    from a cleared word."""
    build_mod.build()
    dev = torch.device("cuda", 0)
    cfg = _cfg(capacity_factor=0.0)
    g = torch.Generator(device=dev).manual_seed(5)
    ids = torch.randint(0, cfg.E, (cfg.T, cfg.K), generator=g, device=dev, dtype=torch.int32)
    bad = ids.clone()
    bad[17, 1] = cfg.E + 3
    out = _outputs(cfg, dev)
    B.moe_dispatch_noalloc(cfg, None, bad, out["counts"], out["kept"], out["offsets"], out["perm"],
                           out["row_of"], None)
    assert B.moe_dispatch_noalloc_status() & B.MOE_DEVFLAG_BOUNDS
    out = _outputs(cfg, dev)
    B.moe_dispatch_noalloc(cfg, None, ids, out["counts"], out["kept"], out["offsets"], out["perm"],
                           out["row_of"], None)
    assert B.moe_dispatch_noalloc_status() == 0
    assert int(out["offsets"][-1]) == cfg.T * cfg.K
