"""Expert parallelism: the MoE layer with its experts sharded across ranks.

"Lab: build a tiny MoE in PyTorch", "From local loop to expert parallelism":

    sort by owner -> exchange counts -> all-to-all dispatch
    -> grouped local experts -> reverse all-to-all -> scatter-add

with the same mathematical output as the local layer ("2.9 Mixture-of-Experts
(MoE) Architectures", "Expert Parallelism: A Systems Preview": experts sharded
across devices, every token sent to the device holding its expert and its
result sent back).  Rank r of W holds the contiguous experts r*EL .. r*EL+EL-1
(EL = E / W) and its own batch of tokens; each rank's output equals the local
layer's on that batch (routing, capacity and combine are the batch's own).

Two exchanges are built:

- ``exchange="all_to_all"``: the exchanges are collectives of
  ``torch.distributed`` (NCCL over NVLink on GPUs; all-to-all with per-rank
  sizes, which needs the counts on the host, one device-to-host read per
  forward).  Every other step is a kernel of the CUDA library, through its C
  ABI: routing and the owner-sorted (expert-major) dispatch, the receive
  layout and the row permutations, the grouped experts, the weighted combine.
  ``ops`` can replace those steps (the CPU tests of the exchange logic pass
  the oracle's).
- ``exchange="peer"``: every rank's receive and expert-output buffers are
  mapped into every rank (CUDA IPC), and the library's kernels move the rows
  themselves: the dispatch kernel stores each kept token row straight into its
  owner's buffer at its expert-major row, the owner's grouped experts run in
  place, and the combine kernel loads each slot's result from its owner and
  adds it, weighted, at home.  The communication library only all-gathers the
  kept counts (world x E int32) and provides two stream-ordered barriers (a
  one-element all-reduce): no host read, no all-to-all, no permutation.

The default ops are the CUDA library, which fails loudly when it is not built.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding as B


class CudaOps:
    """The layer's device steps, through the C ABI (no host arithmetic)."""

    def __init__(self, T, D, F, E, K, EL, W, dtype, capacity_factor, router_options, device):
        self.cfg = B.MoeConfig.make(T, D, F, E, K, dtype, capacity_factor, **router_options)
        # the owner's grouped experts: EL experts over at most W * T * K arriving rows
        self.max_recv = W * T * K
        self.cfg_local = B.MoeConfig.make(self.max_recv, D, F, EL, 1, dtype, 0.0)
        self.device = device
        self.ws = torch.zeros(B.forward_workspace_size(self.cfg), dtype=torch.uint8, device=device)
        self.ws_local = torch.zeros(B.workspace_size(self.cfg_local), dtype=torch.uint8, device=device)
        self.ws_ep = torch.zeros(B.ep_workspace_size(W, EL), dtype=torch.uint8, device=device)
        self.max_rows = B.max_rows(self.cfg)
        i32 = dict(dtype=torch.int32, device=device)
        self.ids = torch.empty((T, K), **i32)
        self.w = torch.empty((T, K), dtype=torch.float32, device=device)
        self.counts = torch.empty(E, **i32)
        self.kept = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.perm = torch.empty(self.max_rows, **i32)
        self.row_of = torch.empty(T * K, **i32)
        self.offsets_local = torch.empty(EL + 1, **i32)
        self.dst_of = torch.empty(self.max_recv, **i32)
        self.src_of = torch.empty(self.max_recv, **i32)
        self.remote_row = None  # peer exchange: row of each slot in its owner's buffer
        self.h_local = None     # peer exchange: the local experts' hidden activations
        # the router weight's bf16 terms (moe_router_prepare), split again when the
        # weight is replaced or changed in place (its version counter)
        nb = B.router_terms_size(self.cfg)
        self.router_terms = torch.empty(nb, dtype=torch.uint8, device=device) if nb else None
        self._terms_of = None

    def _terms(self, w_router):
        if self.router_terms is None:
            return None
        key = (id(w_router), w_router.data_ptr(), w_router._version)
        if key != self._terms_of:
            B.moe_router_prepare(self.cfg, w_router, self.router_terms)
            self._terms_of = key
        return self.router_terms

    def route_dispatch(self, x, w_router, router_bias, selection_bias, logit_noise):
        x_perm = torch.empty((self.max_rows, x.shape[1]), dtype=x.dtype, device=x.device)
        B.moe_route(self.cfg, x, w_router, self.ids, self.w, self.ws, router_bias=router_bias,
                    logit_noise=logit_noise, selection_bias=selection_bias,
                    w_router_terms=self._terms(w_router))
        B.moe_dispatch(self.cfg, x, self.ids, self.counts, self.kept, self.offsets, self.perm,
                       self.row_of, x_perm, self.ws)
        return self.kept, self.offsets, x_perm

    def layout(self, recv_counts, W, EL):
        B.moe_ep_layout(W, EL, recv_counts, self.max_recv, self.offsets_local, self.dst_of,
                        self.src_of, self.ws_ep)
        return self.offsets_local, self.dst_of, self.src_of

    def to_expert_major(self, x_recv, src_of, n):
        # the grouped GEMM's operand maps cover max_recv rows (its tiles read
        # past an expert's last row), so the buffer has all of them
        x_loc = torch.empty((self.max_recv, x_recv.shape[1]), dtype=x_recv.dtype, device=x_recv.device)
        B.moe_permute_rows(x_recv, src_of, n, x_loc, self.ws_ep)
        return x_loc

    def to_arrival_order(self, y_loc, dst_of, n):
        y_back = torch.empty((max(n, 1), y_loc.shape[1]), dtype=y_loc.dtype, device=y_loc.device)
        B.moe_permute_rows(y_loc, dst_of, n, y_back, self.ws_ep)
        return y_back

    def experts(self, x_loc, offsets_local, w_gate, w_up, w_down):
        R = self.max_recv
        h = torch.empty((R, w_gate.shape[2]), dtype=x_loc.dtype, device=x_loc.device)
        y = torch.empty((R, x_loc.shape[1]), dtype=x_loc.dtype, device=x_loc.device)
        B.moe_expert_ffn(self.cfg_local, x_loc, offsets_local, None, None, w_gate, w_up, w_down, h,
                         y, self.ws_local)
        return y

    def combine(self, y_perm, x):
        y = torch.empty_like(x)
        B.moe_combine_weighted(self.cfg, y_perm, self.row_of, self.w, y)
        return y

    def status(self):
        flags = 0
        for ws in (self.ws, self.ws_local, self.ws_ep):
            flags |= B.moe_get_device_status(ws)
        return flags

    # ---- peer exchange: routing and the dispatch index only (no local gather),
    # rows stored into the owners' buffers, experts in place, combine from the owners

    def route_index(self, x, w_router, router_bias, selection_bias, logit_noise):
        B.moe_route(self.cfg, x, w_router, self.ids, self.w, self.ws, router_bias=router_bias,
                    logit_noise=logit_noise, selection_bias=selection_bias,
                    w_router_terms=self._terms(w_router))
        B.moe_dispatch(self.cfg, None, self.ids, self.counts, self.kept, self.offsets, self.perm,
                       self.row_of, None, self.ws)
        return self.kept

    def peer_dispatch(self, x, kept_all, rank, W, peer):
        if self.remote_row is None:
            self.remote_row = torch.empty_like(self.row_of)
        B.moe_ep_peer_dispatch(self.cfg, rank, W, kept_all, x, self.ids, self.row_of, self.offsets,
                               peer.recv_ptrs, peer.rows, self.offsets_local, self.remote_row,
                               self.ws_ep)

    def peer_experts(self, peer, w_gate, w_up, w_down):
        if self.h_local is None:
            self.h_local = torch.empty((self.max_recv, w_gate.shape[2]), dtype=w_gate.dtype,
                                       device=self.device)
        B.moe_expert_ffn(self.cfg_local, peer.recv_x, self.offsets_local, None, None, w_gate, w_up,
                         w_down, self.h_local, peer.y_loc, self.ws_local)

    def peer_combine(self, x, W, peer):
        y = torch.empty_like(x)
        B.moe_ep_peer_combine(self.cfg, W, self.ids, self.remote_row, self.w, peer.out_ptrs,
                              peer.rows, y, self.ws_ep)
        return y


class PeerBuffers:
    """Every rank's receive buffer and expert-output buffer (rows x D elements
    each), mapped into this process: this rank's own from moe_ipc_alloc, the
    others' opened from the handles all ranks exchange at construction.
    recv_ptrs / out_ptrs: int64 device tensors of the W addresses, indexed by
    rank.  close() unmaps and frees them (collective: every rank calls it)."""

    def __init__(self, rows: int, D: int, elem_bytes: int, group, device):
        self.group = group
        self.rows = int(rows)
        W, rank = dist.get_world_size(group), dist.get_rank(group)
        nbytes = self.rows * D * elem_bytes
        self.recv_x, hx = B.ipc_alloc(nbytes)
        self.y_loc, hy = B.ipc_alloc(nbytes)
        handles = [None] * W
        dist.all_gather_object(handles, (hx, hy), group=group)
        self._opened = []
        xs, ys = [], []
        for r, (px_h, py_h) in enumerate(handles):
            if r == rank:
                xs.append(self.recv_x)
                ys.append(self.y_loc)
            else:
                px, py = B.ipc_open(px_h), B.ipc_open(py_h)
                self._opened += [px, py]
                xs.append(px)
                ys.append(py)
        self.recv_ptrs = torch.tensor(xs, dtype=torch.int64, device=device)
        self.out_ptrs = torch.tensor(ys, dtype=torch.int64, device=device)

    def close(self):
        if self.recv_x is None:
            return
        torch.cuda.synchronize()
        dist.barrier(group=self.group)  # nobody reads a peer's buffer any more
        for p in self._opened:
            B.ipc_close(p)
        self._opened = []
        dist.barrier(group=self.group)  # every mapping of this rank's buffers is gone
        B.ipc_free(self.recv_x)
        B.ipc_free(self.y_loc)
        self.recv_x = self.y_loc = None


class ExpertParallelMoE:
    """One rank's share of an expert-parallel MoE layer.

    w_router (D, E) fp32 and router_bias (E) are the whole router (every rank
    routes its own tokens over all E experts); w_gate_local, w_up_local
    (EL, D, F) and w_down_local (EL, F, D) are this rank's experts
    rank*EL .. rank*EL + EL - 1.  router_options as for MoELayer.
    """

    def __init__(self, T: int, w_router, w_gate_local, w_up_local, w_down_local, E: int, K: int,
                 capacity_factor: float = 0.0, router_bias=None, selection_bias=None, group=None,
                 ops=None, exchange: str = "all_to_all", **router_options):
        if exchange not in ("all_to_all", "peer"):
            raise ValueError("exchange is 'all_to_all' or 'peer'")
        if exchange == "peer" and ops is not None:
            raise ValueError("the peer exchange runs on the CUDA library's kernels only")
        self.exchange = exchange
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.W != 0:
            raise ValueError("the experts must divide evenly among the ranks")
        self.E, self.K, self.T = E, K, T
        self.EL = E // self.W
        if w_gate_local.shape[0] != self.EL:
            raise ValueError(f"this rank holds {self.EL} experts, got {w_gate_local.shape[0]}")
        self.D, self.F = w_gate_local.shape[1], w_gate_local.shape[2]
        self.w_router, self.router_bias, self.selection_bias = w_router, router_bias, selection_bias
        self.w_gate, self.w_up, self.w_down = w_gate_local, w_up_local, w_down_local
        if ops is None:
            dtype = "bf16" if w_gate_local.dtype == torch.bfloat16 else "f32"
            ops = CudaOps(T, self.D, self.F, E, K, self.EL, self.W, dtype, capacity_factor,
                          router_options, w_gate_local.device)
        self.ops = ops
        # optional CUDA events recorded on the current stream at the step
        # boundaries of forward() (stage_names() + 1 of them), for stage timing
        self.trace_events = None
        self.peer = None
        if exchange == "peer":
            dev = w_gate_local.device
            self.kept_all = torch.empty(self.W * E, dtype=torch.int32, device=dev)
            self._sync = torch.zeros(1, dtype=torch.int32, device=dev)
            self.peer = PeerBuffers(ops.max_recv, self.D, w_gate_local.element_size(), group, dev)

    def close(self):
        """Release the peer buffers (collective for the peer exchange)."""
        if self.peer is not None:
            self.peer.close()
            self.peer = None

    PEER_STAGES = ("route", "counts_allgather", "dispatch", "barrier_rows", "experts",
                   "barrier_results", "combine")
    A2A_STAGES = ("route_dispatch", "counts_exchange", "rows_all_to_all", "to_expert_major",
                  "experts", "results_all_to_all", "combine")

    def stage_names(self):
        return self.PEER_STAGES if self.exchange == "peer" else self.A2A_STAGES

    def _mark(self, i):
        if self.trace_events is not None:
            self.trace_events[i].record()

    def _barrier(self):
        # stream-ordered: the next kernel on this stream starts after every
        # rank's kernels before its own all-reduce have finished
        dist.all_reduce(self._sync, group=self.group)

    def _forward_peer(self, x, logit_noise):
        ops = self.ops
        self._mark(0)
        kept = ops.route_index(x, self.w_router, self.router_bias, self.selection_bias, logit_noise)
        self._mark(1)
        dist.all_gather_into_tensor(self.kept_all, kept, group=self.group)
        self._mark(2)
        ops.peer_dispatch(x, self.kept_all, self.rank, self.W, self.peer)
        self._mark(3)
        self._barrier()  # every rank's rows are in their owners' buffers
        self._mark(4)
        ops.peer_experts(self.peer, self.w_gate, self.w_up, self.w_down)
        self._mark(5)
        self._barrier()  # every owner's results are ready
        self._mark(6)
        y = ops.peer_combine(x, self.W, self.peer)
        self._mark(7)
        return y

    def forward(self, x, logit_noise=None):
        if self.exchange == "peer":
            return self._forward_peer(x, logit_noise)
        W, EL = self.W, self.EL
        ops = self.ops
        self._mark(0)
        # route this rank's tokens and sort their rows by expert (so by owner)
        kept, offsets, x_perm = ops.route_dispatch(x, self.w_router, self.router_bias,
                                                   self.selection_bias, logit_noise)
        self._mark(1)
        # exchange the per-expert row counts: recv[s, e] = rows source s sends for my expert e
        send_counts = kept.reshape(W, EL).contiguous()
        recv_counts = torch.empty_like(send_counts)
        dist.all_to_all_single(recv_counts, send_counts, group=self.group)
        # the all-to-all sizes (host values: one device-to-host read of 2 W numbers)
        owner_bounds = offsets[::EL].to(torch.int64)
        send_rows = (owner_bounds[1:] - owner_bounds[:-1]).cpu().tolist()
        recv_rows = recv_counts.sum(1).cpu().tolist()
        n_send, n_recv = sum(send_rows), sum(recv_rows)
        self._mark(2)
        # rows to their owners
        x_recv = torch.empty((max(n_recv, 1), self.D), dtype=x.dtype, device=x.device)
        dist.all_to_all_single(x_recv[:n_recv], x_perm[:n_send].contiguous(), recv_rows, send_rows,
                               group=self.group)
        self._mark(3)
        # arrived source-major; the grouped experts want expert-major
        offsets_local, dst_of, src_of = ops.layout(recv_counts, W, EL)
        x_loc = ops.to_expert_major(x_recv, src_of, n_recv)
        self._mark(4)
        y_loc = ops.experts(x_loc, offsets_local, self.w_gate, self.w_up, self.w_down)
        self._mark(5)
        # results back in arrival order, then to the tokens' home ranks
        y_back = ops.to_arrival_order(y_loc, dst_of, n_recv)
        y_perm = torch.empty((max(n_send, 1), self.D), dtype=x.dtype, device=x.device)
        dist.all_to_all_single(y_perm[:n_send], y_back[:n_recv].contiguous(), send_rows, recv_rows,
                               group=self.group)
        self._mark(6)
        # weighted scatter-add at home
        y = ops.combine(y_perm, x)
        self._mark(7)
        return y
