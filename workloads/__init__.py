"""Seeded synthetic inputs for the token-choice top-k MoE layer forward.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic.  Both the CUDA path and the CPU oracle are fed from here,
so that each sees the very same bytes.

Workload shapes follow the five layer shapes the library is measured on
(a tiny fp32 layer, a Mixtral-shaped layer, a fine-grained skewed layer, an
ST-MoE capacity-factor layer and a large-E decode layer).  Value recipe:

* x ~ N(0, 1); router W_r (D, E), W_gate / W_up (E, D, F), W_down (E, F, D)
  ~ N(0, 0.02^2).  Drawn in fp32, then rounded once to the layer dtype
  (bf16 layers); the router weight, bias and noise stay fp32.
* fine-grained skewed layer: fixed router bias
  b_e = 2 * (-ln(rank_e + 1) / ln 64), rank = a seeded permutation of the
  experts (CPU generator, seed 0), which makes the load Zipf-like.
* capacity layer: Gaussian logit noise of std 1/E from a second generator
  (seed 1), passed to the router as an input tensor.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    D: int
    F: int
    E: int
    K: int
    dtype: str = "bf16"          # "f32" or "bf16": x, expert weights and outputs
    capacity_factor: float = 0.0  # <= 0: dropless
    bias: str | None = None       # None or "zipf"
    noise: bool = False           # logit noise of std 1/E from a second seed
    seed: int = 0
    w_std: float = 0.02
    # router options (defaults: softmax, renormalised top-k)
    score_func: str = "softmax"
    renormalize: bool = True
    n_groups: int = 1
    topk_groups: int = 1
    route_scale: float = 1.0
    sel_bias: bool = False        # a seeded DeepSeek-V3 selection bias input
    F_shared: int = 0             # hidden size of a shared expert (0: none)

    def routing(self) -> dict:
        """Router options as keyword arguments (oracle.route / MoeConfig.make)."""
        return dict(score_func=self.score_func, renormalize=self.renormalize,
                    n_groups=self.n_groups, topk_groups=self.topk_groups,
                    route_scale=self.route_scale)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS: dict[str, Workload] = {
    # batch 4 x seq 128, fp32 throughout
    "tiny_fp32": Workload("tiny_fp32", T=512, D=256, F=512, E=8, K=2, dtype="f32"),
    # batch 2 x seq 4096, Mixtral-shaped experts
    "mixtral_8x": Workload("mixtral_8x", T=8192, D=4096, F=14336, E=8, K=2),
    # fine-grained experts with a Zipf-like router bias
    "fine_skewed": Workload("fine_skewed", T=16384, D=2048, F=1408, E=64, K=6, bias="zipf"),
    # batch 8 x seq 4096, capacity factor 1.25 and noisy logits
    "stmoe_capacity": Workload("stmoe_capacity", T=32768, D=1024, F=4096, E=32, K=2,
                               capacity_factor=1.25, noise=True),
    # decode-shaped: 128 tokens over 256 experts (about 22.5 GB of expert weights)
    "decode_e256": Workload("decode_e256", T=128, D=7168, F=2048, E=256, K=8),
}

WORKLOAD_ORDER = ["tiny_fp32", "mixtral_8x", "fine_skewed", "stmoe_capacity", "decode_e256"]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_rank(E: int, seed: int = 0) -> torch.Tensor:
    """Seeded random expert ranking (a permutation of 0..E-1), CPU generator."""
    return torch.randperm(E, generator=_gen("cpu", seed))


def zipf_bias(E: int, seed: int = 0) -> torch.Tensor:
    """Router bias b_e = 2 * (-ln(rank_e + 1) / ln 64) for a seeded ranking."""
    rank = zipf_rank(E, seed).to(torch.float64)
    return (2.0 * (-torch.log(rank + 1.0) / math.log(64.0))).to(torch.float32)


def _randn(shape, g, device, std=1.0, out_dtype=torch.float32, chunk_dim0: bool = False):
    """Draw N(0, std^2) in fp32 and round once to out_dtype.

    With chunk_dim0 the draw is made one leading slice at a time so that a very
    large bf16 tensor never needs an fp32 copy of itself (same values as one
    big draw is NOT guaranteed; the chunked recipe is the definition).
    """
    if not chunk_dim0:
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t.to(out_dtype)
    out = torch.empty(shape, device=device, dtype=out_dtype)
    for i in range(shape[0]):
        t = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out[i].copy_(t)
    return out


def make_inputs(wl: Workload | str, device="cpu", seed: int | None = None) -> dict:
    """Generate every input of one layer forward.

    Returns a dict with x (T,D), w_router (D,E) fp32, bias (E) fp32 or None,
    noise (T,E) fp32 or None, w_gate (E,D,F), w_up (E,D,F), w_down (E,F,D),
    sel_bias (E) fp32 or None (N(0, 0.5^2), generator seed + 2), shared =
    (w_gate_s (D,Fs), w_up_s (D,Fs), w_down_s (Fs,D)) or None (generator seed + 3).
    Draw order (one generator, seeded): x, w_router, w_gate, w_up, w_down.
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    seed = wl.seed if seed is None else seed
    g = _gen(device, seed)
    dt = wl.torch_dtype
    big = wl.E * wl.D * wl.F > (1 << 28)
    x = _randn((wl.T, wl.D), g, device, 1.0, dt)
    w_router = _randn((wl.D, wl.E), g, device, wl.w_std, torch.float32)
    w_gate = _randn((wl.E, wl.D, wl.F), g, device, wl.w_std, dt, chunk_dim0=big)
    w_up = _randn((wl.E, wl.D, wl.F), g, device, wl.w_std, dt, chunk_dim0=big)
    w_down = _randn((wl.E, wl.F, wl.D), g, device, wl.w_std, dt, chunk_dim0=big)
    bias = zipf_bias(wl.E, 0).to(device) if wl.bias == "zipf" else None
    noise = None
    if wl.noise:
        g2 = _gen(device, seed + 1)
        noise = _randn((wl.T, wl.E), g2, device, 1.0 / wl.E, torch.float32)
    sel_bias = None
    if wl.sel_bias:
        sel_bias = _randn((wl.E,), _gen(device, seed + 2), device, 0.5, torch.float32)
    shared = None
    if wl.F_shared:
        g3 = _gen(device, seed + 3)
        fs = wl.F_shared
        shared = (_randn((wl.D, fs), g3, device, wl.w_std, dt),
                  _randn((wl.D, fs), g3, device, wl.w_std, dt),
                  _randn((fs, wl.D), g3, device, wl.w_std, dt))
    return dict(x=x, w_router=w_router, bias=bias, noise=noise,
                w_gate=w_gate, w_up=w_up, w_down=w_down, sel_bias=sel_bias, shared=shared)


def make_tokens(wl: Workload | str, device="cpu", seed: int = 1234) -> torch.Tensor:
    """A fresh batch of activations x (T, D) for one more step of the same layer."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    g = _gen(device, seed)
    return _randn((wl.T, wl.D), g, device, 1.0, wl.torch_dtype)


def make_output_grad(wl: Workload | str, device="cpu", seed: int = 4321) -> torch.Tensor:
    """A seeded upstream gradient dY (T, D) ~ N(0, 1) in the layer dtype, for
    the backward of the layer."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    g = _gen(device, seed)
    return _randn((wl.T, wl.D), g, device, 1.0, wl.torch_dtype)
