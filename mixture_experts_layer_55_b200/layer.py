"""MoELayer: the layer's weights, configuration and workspace in one object.

A convenience over the C ABI for callers that work in PyTorch: it allocates
the device workspace once (through torch), keeps the weights resident, and
calls ``moe_forward`` (inference), or ``moe_forward_train`` and
``moe_backward`` (training).  It adds no arithmetic of its own.
"""
from __future__ import annotations

import torch

from . import _binding as B


class MoELayer:
    """Token-choice top-k MoE layer (forward and backward)
    on one CUDA device.

    weights: w_router (D, E) fp32; w_gate, w_up (E, D, F); w_down (E, F, D) in
    the layer dtype (bf16 or fp32); optional router_bias (E) fp32.
    """

    def __init__(self, T: int, w_router, w_gate, w_up, w_down, K: int, capacity_factor=0.0,
                 router_bias=None, selection_bias=None, shared=None, **router_options):
        """router_options: score_func ("softmax" | "sigmoid"), renormalize,
        n_groups, topk_groups, route_scale (see moe_config in include/moe.h).
        selection_bias (E) fp32: DeepSeek-V3 bias, for selection only.
        shared: (w_gate_s (D, Fs), w_up_s (D, Fs), w_down_s (Fs, D)), a shared
        expert every token passes through."""
        E, D, F = w_gate.shape
        dtype = "bf16" if w_gate.dtype == torch.bfloat16 else "f32"
        fs = 0 if shared is None else shared[0].shape[1]
        self.cfg = B.MoeConfig.make(T, D, F, E, K, dtype, capacity_factor, F_shared=fs,
                                    **router_options)
        self.shared = shared
        self.selection_bias = selection_bias
        st = B.check_config(self.cfg)
        if st != B.MOE_OK:
            raise B.MoEError(st, "MoELayer")
        self.device = w_gate.device
        self.w_router, self.w_gate, self.w_up, self.w_down = w_router, w_gate, w_up, w_down
        self.router_bias = router_bias
        nbytes = B.forward_workspace_size(self.cfg)
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.torch_dtype = w_gate.dtype
        self.losses = torch.zeros(3, dtype=torch.float32, device=self.device)  # z, balance, entropy
        self.mean_prob = torch.zeros(E, dtype=torch.float32, device=self.device)
        self.counts = torch.zeros(E, dtype=torch.int32, device=self.device)
        # the router weight split once into the tensor-core router's bf16 terms
        # (moe_router_prepare); split again when w_router is replaced or changed
        # in place (tracked by the tensor's version counter)
        nb = B.router_terms_size(self.cfg)
        self.router_terms = torch.empty(nb, dtype=torch.uint8, device=self.device) if nb else None
        self._terms_of = None

    def _terms(self, stream=None):
        if self.router_terms is None:
            return None
        key = (id(self.w_router), self.w_router.data_ptr(), self.w_router._version)
        if key != self._terms_of:
            B.moe_router_prepare(self.cfg, self.w_router, self.router_terms, stream=stream)
            self._terms_of = key
        return self.router_terms

    def forward(self, x, y=None, logit_noise=None, stats: bool = True, stream=None):
        """y = MoE(x) for x (T, D) on the device; returns y.  With stats the
        router's z-loss / balance loss / entropy, mean probabilities and counts are left in
        self.losses, self.mean_prob and self.counts."""
        if y is None:
            y = torch.empty_like(x)
        B.moe_forward(self.cfg, x, self.w_router, self.w_gate, self.w_up, self.w_down, y,
                      self.workspace, w_router_terms=self._terms(stream),
                      router_bias=self.router_bias, logit_noise=logit_noise,
                      selection_bias=self.selection_bias, shared=self.shared,
                      losses=self.losses if stats else None,
                      mean_prob=self.mean_prob if stats else None,
                      counts=self.counts if stats else None, stream=stream)
        return y

    def capture(self, x, y, logit_noise=None, stats: bool = True):
        """One forward over the buffers x -> y captured as a CUDA graph; returns
        the torch.cuda.CUDAGraph (graph.replay() runs the layer again on
        whatever x then holds).  The forward takes no host decision between
        its launches and never synchronises, so all of them form one graph;
        the first call runs outside the capture (one-time kernel attributes).
        Trace events must not be attached while capturing."""
        dev = self.device
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self.forward(x, y, logit_noise=logit_noise, stats=stats)
        torch.cuda.current_stream(dev).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(x, y, logit_noise=logit_noise, stats=stats)
        return graph

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

    def forward_host_stream(self, x_hosts, y_hosts, logit_noise=None, nbuf: int = 2,
                            events=None):
        """The layer over a sequence of host batches, end to end and pipelined.

        x_hosts / y_hosts: lists of pinned host tensors (T, D).  Three streams:
        the copy in of batch i+1 and the copy out of batch i-1 overlap the
        forward of batch i; device batches are double-buffered.  Returns the
        copy-out stream (synchronise on it, or on `events` when given: a pair of
        timing events recorded before the first copy in and after the last
        copy out)."""
        dev = self.device
        comp = torch.cuda.current_stream(dev)
        h2d = torch.cuda.Stream(dev)
        d2h = torch.cuda.Stream(dev)
        shape, dt = x_hosts[0].shape, x_hosts[0].dtype
        xd = [torch.empty(shape, dtype=dt, device=dev) for _ in range(nbuf)]
        yd = [torch.empty(shape, dtype=dt, device=dev) for _ in range(nbuf)]
        ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        ev_done = [torch.cuda.Event() for _ in range(nbuf)]
        ev_out = [torch.cuda.Event() for _ in range(nbuf)]
        if events is not None:
            h2d.wait_stream(comp)
            events[0].record(h2d)
        for i, (xh, yh) in enumerate(zip(x_hosts, y_hosts)):
            b = i % nbuf
            with torch.cuda.stream(h2d):
                if i >= nbuf:
                    h2d.wait_event(ev_done[b])  # the forward of batch i-nbuf read xd[b]
                xd[b].copy_(xh, non_blocking=True)
                ev_in[b].record(h2d)
            comp.wait_event(ev_in[b])
            if i >= nbuf:
                comp.wait_event(ev_out[b])      # the copy out of batch i-nbuf read yd[b]
            self.forward(xd[b], yd[b], logit_noise=logit_noise, stream=comp)
            ev_done[b].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_done[b])
                yh.copy_(yd[b], non_blocking=True)
                ev_out[b].record(d2h)
        if events is not None:
            events[1].record(d2h)
        comp.wait_stream(d2h)
        return d2h

    # ----------------------------------------------------------- training
    def forward_train(self, x, y=None, logit_noise=None, stream=None):
        """forward() that keeps the activations moe_backward reads; the state
        buffer is allocated on first use."""
        if getattr(self, "state", None) is None:
            self.state = torch.zeros(B.train_state_size(self.cfg), dtype=torch.uint8,
                                     device=self.device)
        if y is None:
            y = torch.empty_like(x)
        B.moe_forward_train(self.cfg, x, self.w_router, self.w_gate, self.w_up, self.w_down, y,
                            self.state, router_bias=self.router_bias, logit_noise=logit_noise,
                            selection_bias=self.selection_bias, shared=self.shared,
                            losses=self.losses, mean_prob=self.mean_prob, counts=self.counts,
                            stream=stream)
        self._train_x = x
        return y

    def backward(self, dy, c_balance: float = 0.0, c_z: float = 0.0, grads=None, stream=None):
        """Gradients of sum(dy * y) + c_balance * balance + c_z * z for the
        last forward_train.  Returns a dict of dx (layer dtype) and fp32
        dw_router, db_router (when the layer has a router bias), dw_gate,
        dw_up, dw_down (and dshared); ``grads`` may pass that dict back to
        reuse its buffers."""
        x = getattr(self, "_train_x", None)
        if x is None:
            raise RuntimeError("backward() needs a forward_train() first")
        if getattr(self, "bwd_workspace", None) is None:
            self.bwd_workspace = torch.zeros(B.backward_workspace_size(self.cfg),
                                             dtype=torch.uint8, device=self.device)
        if grads is None:
            f32 = dict(dtype=torch.float32, device=self.device)
            grads = dict(dx=torch.empty_like(x),
                         dw_router=torch.empty(self.w_router.shape, **f32),
                         dw_gate=torch.empty(self.w_gate.shape, **f32),
                         dw_up=torch.empty(self.w_up.shape, **f32),
                         dw_down=torch.empty(self.w_down.shape, **f32))
            if self.router_bias is not None:
                grads["db_router"] = torch.empty(self.router_bias.shape, **f32)
            if self.shared is not None:
                grads["dshared"] = tuple(torch.empty(w.shape, **f32) for w in self.shared)
        B.moe_backward(self.cfg, x, self.w_router, self.w_gate, self.w_up, self.w_down, self.state,
                       dy, grads["dx"], grads["dw_router"], grads["dw_gate"], grads["dw_up"],
                       grads["dw_down"], self.bwd_workspace, c_balance=c_balance, c_z=c_z,
                       db_router=grads.get("db_router"), shared=self.shared,
                       dshared=grads.get("dshared"), stream=stream)
        return grads

    def update_selection_bias(self, gamma: float, stream=None):
        """One DeepSeek-V3 balancing step from the last forward's counts."""
        if self.selection_bias is None:
            raise ValueError("the layer has no selection bias")
        B.moe_update_selection_bias(self.cfg, self.counts, gamma, self.selection_bias, stream=stream)
