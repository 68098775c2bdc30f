"""B200-native forward pass of a token-choice top-k Mixture-of-Experts layer.

The compute lives in ``libmoe_b200.so`` (hand-written CUDA for sm_100a behind
the C ABI of ``include/moe.h``); this package is its thin Python binding plus
``MoELayer``, a convenience holder of the layer's weights and workspace.
PyTorch serves only for device memory and streams.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    MOE_BF16, MOE_F32, MoeConfig, MoEError, capacity, check_config, forward_kernel_count,
    forward_workspace_size, header_symbols, lib, max_rows, moe_clear_device_status, moe_combine,
    moe_dispatch, moe_dispatch_noalloc, moe_expert_ffn, moe_forward, moe_get_device_status,
    moe_route, moe_selftest_wait_timeout, moe_trace_attach, moe_update_selection_bias,
    status_string, trace_stage_names, workspace_size)
from .layer import MoELayer  # noqa: F401
