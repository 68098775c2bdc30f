"""MoELayer: the layer's weights, configuration and workspace in one object.

A convenience over the C ABI for callers that work in PyTorch: it allocates
the device workspace once (through torch), keeps the weights resident, and
calls ``moe_forward``.  It adds no arithmetic of its own.
"""
from __future__ import annotations

import torch

from . import _binding as B


class MoELayer:
    """Token-choice top-k MoE layer forward on one CUDA device.

    weights: w_router (D, E) fp32; w_gate, w_up (E, D, F); w_down (E, F, D) in
    the layer dtype (bf16 or fp32); optional router_bias (E) fp32.
    """

    def __init__(self, T: int, w_router, w_gate, w_up, w_down, K: int, capacity_factor=0.0,
                 router_bias=None):
        E, D, F = w_gate.shape
        dtype = "bf16" if w_gate.dtype == torch.bfloat16 else "f32"
        self.cfg = B.MoeConfig.make(T, D, F, E, K, dtype, capacity_factor)
        st = B.check_config(self.cfg)
        if st != B.MOE_OK:
            raise B.MoEError(st, "MoELayer")
        self.device = w_gate.device
        self.w_router, self.w_gate, self.w_up, self.w_down = w_router, w_gate, w_up, w_down
        self.router_bias = router_bias
        nbytes = B.forward_workspace_size(self.cfg)
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.torch_dtype = w_gate.dtype
        self.losses = torch.zeros(2, dtype=torch.float32, device=self.device)
        self.mean_prob = torch.zeros(E, dtype=torch.float32, device=self.device)
        self.counts = torch.zeros(E, dtype=torch.int32, device=self.device)

    def forward(self, x, y=None, logit_noise=None, stats: bool = True, stream=None):
        """y = MoE(x) for x (T, D) on the device; returns y.  With stats the
        router's z-loss / balance loss, mean probabilities and counts are left in
        self.losses, self.mean_prob and self.counts."""
        if y is None:
            y = torch.empty_like(x)
        B.moe_forward(self.cfg, x, self.w_router, self.w_gate, self.w_up, self.w_down, y,
                      self.workspace, router_bias=self.router_bias, logit_noise=logit_noise,
                      losses=self.losses if stats else None,
                      mean_prob=self.mean_prob if stats else None,
                      counts=self.counts if stats else None, stream=stream)
        return y

    def forward_host(self, x_host, y_host, x_dev=None, y_dev=None, logit_noise=None,
                     stream=None):
        """End to end from host memory: copy x_host (pinned) in, run the layer,
        copy y out to y_host (pinned), all on one stream (asynchronous)."""
        s = stream or torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            if x_dev is None:
                x_dev = torch.empty(x_host.shape, dtype=x_host.dtype, device=self.device)
            if y_dev is None:
                y_dev = torch.empty_like(x_dev)
            x_dev.copy_(x_host, non_blocking=True)
            self.forward(x_dev, y_dev, logit_noise=logit_noise, stream=s)
            y_host.copy_(y_dev, non_blocking=True)
        return y_host
