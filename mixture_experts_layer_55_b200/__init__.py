"""B200-native token-choice top-k Mixture-of-Experts layer: forward, backward
and expert parallelism.

The compute lives in ``libmoe_b200.so`` (hand-written CUDA for sm_100a behind
the C ABI of ``include/moe.h``); this package is its thin Python binding plus
``MoELayer`` (a holder of one GPU's weights and workspaces) and
``ExpertParallelMoE`` (the layer with its experts sharded across ranks, the
exchanges through ``torch.distributed`` all-to-all or through the library's
own kernels over peer-mapped buffers).  PyTorch serves only for device
memory, streams and collectives.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    MOE_BF16, MOE_F32, MoeConfig, MoEError, backward_kernel_count, backward_workspace_size,
    capacity, check_config, ep_workspace_size, forward_kernel_count, forward_workspace_size,
    header_symbols, ipc_alloc, ipc_close, ipc_free, ipc_open, lib, max_rows, moe_backward, moe_clear_device_status, moe_combine,
    moe_combine_weighted, moe_dispatch, moe_dispatch_noalloc, moe_ep_layout, moe_ep_peer_combine,
    moe_ep_peer_dispatch, moe_expert_ffn,
    moe_forward, moe_forward_train, moe_get_device_status, moe_permute_rows, moe_route,
    moe_selftest_wait_timeout, moe_trace_attach, moe_trace_attach_backward,
    moe_update_selection_bias, status_string, trace_backward_stage_names, trace_stage_names,
    train_state_size, workspace_size)
from .ep import ExpertParallelMoE, PeerBuffers  # noqa: F401
from .layer import MoELayer  # noqa: F401
