"""ctypes binding of libmoe_b200.so (the C ABI declared in include/moe.h).

Argument marshalling only: tensors become device pointers, the current torch
stream becomes the cudaStream_t, and a non-OK status becomes MoEError.  Every
step of the layer runs in the library's CUDA kernels; nothing here computes.
"""
from __future__ import annotations

import ctypes
import os
import re

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "moe.h")

MOE_OK = 0
MOE_ERR_ARG = -1
MOE_ERR_SHAPE = -2
MOE_ERR_UNSUPPORTED = -3
MOE_ERR_ALIGN = -4
MOE_ERR_CUDA = -5
MOE_ERR_DEVICE_TIMEOUT = -6
MOE_ERR_DEVICE_BOUNDS = -7
MOE_ERR_WORKSPACE = -8
MOE_DEVFLAG_TIMEOUT = 0x1  # device status word bits (include/moe.h)
MOE_DEVFLAG_BOUNDS = 0x2

MOE_F32 = 0
MOE_BF16 = 1
MOE_SCORE_SOFTMAX = 0
MOE_SCORE_SIGMOID = 1
SCORE_FUNCS = {"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID}


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class MoeConfig(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("D", ctypes.c_int32),
        ("F", ctypes.c_int32),
        ("E", ctypes.c_int32),
        ("K", ctypes.c_int32),
        ("capacity_factor", ctypes.c_float),
        ("score_func", ctypes.c_int32),
        ("renormalize", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("n_groups", ctypes.c_int32),
        ("topk_groups", ctypes.c_int32),
        ("route_scale", ctypes.c_float),
        ("F_shared", ctypes.c_int32),
    ]

    @classmethod
    def make(cls, T, D, F, E, K, dtype="bf16", capacity_factor=0.0, score_func="softmax",
             renormalize=True, n_groups=1, topk_groups=1, route_scale=1.0, F_shared=0):
        dt = {"bf16": MOE_BF16, "f32": MOE_F32, MOE_BF16: MOE_BF16, MOE_F32: MOE_F32}[dtype]
        sf = SCORE_FUNCS.get(score_func, score_func)
        return cls(int(T), int(D), int(F), int(E), int(K), float(capacity_factor), int(sf),
                   int(bool(renormalize)), dt, int(n_groups), int(topk_groups), float(route_scale),
                   int(F_shared))


_lib = None

_P = ctypes.c_void_p
_SIG = {
    "moe_status_string": ([ctypes.c_int32], ctypes.c_char_p),
    "moe_version": ([], ctypes.c_int32),
    "moe_check_config": ([_P], ctypes.c_int32),
    "moe_capacity": ([_P, _P], ctypes.c_int32),
    "moe_max_rows": ([_P, _P], ctypes.c_int32),
    "moe_workspace_size": ([_P, _P], ctypes.c_int32),
    "moe_forward_workspace_size": ([_P, _P], ctypes.c_int32),
    "moe_router_terms_size": ([_P, _P], ctypes.c_int32),
    "moe_router_prepare": ([_P] * 4, ctypes.c_int32),
    "moe_route": ([_P] * 15 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_dispatch": ([_P] * 10 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_dispatch_noalloc": ([_P] * 10, ctypes.c_int32),
    "moe_dispatch_noalloc_status": ([_P, _P], ctypes.c_int32),
    "moe_expert_ffn": ([_P] * 11 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_combine": ([_P] * 6, ctypes.c_int32),
    "moe_forward": ([_P] * 20 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_update_selection_bias": ([_P, _P, ctypes.c_float, _P, _P], ctypes.c_int32),
    "moe_get_device_status": ([_P, _P, _P], ctypes.c_int32),
    "moe_clear_device_status": ([_P, _P], ctypes.c_int32),
    "moe_forward_kernel_count": ([_P, ctypes.c_int32], ctypes.c_int32),
    "moe_selftest_wait_timeout": ([_P, ctypes.c_size_t, ctypes.c_int64, _P], ctypes.c_int32),
    "moe_trace_attach": ([_P, ctypes.c_int32], ctypes.c_int32),
    "moe_trace_boundary_count": ([], ctypes.c_int32),
    "moe_trace_stage_name": ([ctypes.c_int32], ctypes.c_char_p),
    "moe_train_state_size": ([_P, _P], ctypes.c_int32),
    "moe_forward_train": ([_P] * 19 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_backward_workspace_size": ([_P, _P], ctypes.c_int32),
    "moe_backward": ([_P] * 10 + [ctypes.c_size_t, _P, ctypes.c_float, ctypes.c_float]
                     + [_P] * 10 + [ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_backward_kernel_count": ([_P], ctypes.c_int32),
    "moe_trace_attach_backward": ([_P, ctypes.c_int32], ctypes.c_int32),
    "moe_trace_backward_boundary_count": ([], ctypes.c_int32),
    "moe_trace_backward_stage_name": ([ctypes.c_int32], ctypes.c_char_p),
    "moe_ep_workspace_size": ([ctypes.c_int32, ctypes.c_int32, _P], ctypes.c_int32),
    "moe_ep_layout": ([ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int64, _P, _P, _P, _P,
                       ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_permute_rows": ([_P, ctypes.c_int64, _P, ctypes.c_int64, ctypes.c_int64, _P, _P, _P],
                         ctypes.c_int32),
    "moe_combine_weighted": ([_P] * 7, ctypes.c_int32),
    "moe_ipc_alloc": ([ctypes.c_size_t, _P, _P], ctypes.c_int32),
    "moe_ipc_open": ([_P, _P], ctypes.c_int32),
    "moe_ipc_close": ([_P], ctypes.c_int32),
    "moe_ipc_free": ([_P], ctypes.c_int32),
    "moe_ep_peer_dispatch": ([_P, ctypes.c_int32, ctypes.c_int32] + [_P] * 6
                             + [ctypes.c_int64, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int32),
    "moe_ep_peer_combine": ([_P, ctypes.c_int32] + [_P] * 4 + [ctypes.c_int64, _P, _P, _P,
                                                               ctypes.c_size_t, _P], ctypes.c_int32),
}


def header_symbols() -> list[str]:
    """Names of every function include/moe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"^MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)


def lib() -> ctypes.CDLL:
    """Load the library (fails loudly when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build the CUDA library first "
                "(python -m mixture_experts_layer_55_b200.build or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIG.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().moe_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - library unavailable
        return "unknown"


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


# ----------------------------------------------------------- marshalling --

def _ptr(t):
    """Device (or host) address of a tensor, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        return torch.cuda.current_stream().cuda_stream
    return None


def _cfg(cfg: MoeConfig):
    return ctypes.byref(cfg)


def check_config(cfg: MoeConfig) -> int:
    return int(lib().moe_check_config(_cfg(cfg)))


def capacity(cfg: MoeConfig) -> int:
    v = ctypes.c_int64()
    _check(lib().moe_capacity(_cfg(cfg), ctypes.byref(v)), "moe_capacity")
    return v.value


def max_rows(cfg: MoeConfig) -> int:
    v = ctypes.c_int64()
    _check(lib().moe_max_rows(_cfg(cfg), ctypes.byref(v)), "moe_max_rows")
    return v.value


def workspace_size(cfg: MoeConfig) -> int:
    v = ctypes.c_size_t()
    _check(lib().moe_workspace_size(_cfg(cfg), ctypes.byref(v)), "moe_workspace_size")
    return v.value


def forward_workspace_size(cfg: MoeConfig) -> int:
    v = ctypes.c_size_t()
    _check(lib().moe_forward_workspace_size(_cfg(cfg), ctypes.byref(v)),
           "moe_forward_workspace_size")
    return v.value


def router_terms_size(cfg: MoeConfig) -> int:
    """Bytes of the prepared router weight (0: this layer's router takes none)."""
    v = ctypes.c_size_t()
    _check(lib().moe_router_terms_size(_cfg(cfg), ctypes.byref(v)), "moe_router_terms_size")
    return int(v.value)


def moe_router_prepare(cfg, w_router, w_router_terms, stream=None):
    """Split w_router into the three bf16 terms the tensor-core router reads."""
    _check(lib().moe_router_prepare(_cfg(cfg), _ptr(w_router), _ptr(w_router_terms),
                                    _stream(stream)), "moe_router_prepare")


def moe_route(cfg, x, w_router, topk_ids, topk_w, workspace, router_bias=None, logit_noise=None,
              logits_in=None, logits_out=None, probs_out=None, mean_prob=None, losses=None,
              selection_bias=None, w_router_terms=None, stream=None):
    st = lib().moe_route(_cfg(cfg), _ptr(x), _ptr(w_router), _ptr(w_router_terms),
                         _ptr(router_bias),
                         _ptr(selection_bias), _ptr(logit_noise), _ptr(logits_in),
                         _ptr(logits_out), _ptr(probs_out),
                         _ptr(topk_ids), _ptr(topk_w), _ptr(mean_prob), _ptr(losses),
                         _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(st, "moe_route")


def moe_dispatch(cfg, x, topk_ids, counts, kept, offsets, perm, row_of, x_perm, workspace,
                 stream=None):
    st = lib().moe_dispatch(_cfg(cfg), _ptr(x), _ptr(topk_ids), _ptr(counts), _ptr(kept),
                            _ptr(offsets), _ptr(perm), _ptr(row_of), _ptr(x_perm), _ptr(workspace),
                            _nbytes(workspace), _stream(stream))
    _check(st, "moe_dispatch")


def moe_dispatch_noalloc(cfg, x, topk_ids, counts, kept, offsets, perm, row_of, x_perm,
                         stream=None):
    """moe_dispatch with its scratch in the library's static device array (no
    workspace argument; for callers that cannot allocate device memory)."""
    st = lib().moe_dispatch_noalloc(_cfg(cfg), _ptr(x), _ptr(topk_ids), _ptr(counts), _ptr(kept),
                                    _ptr(offsets), _ptr(perm), _ptr(row_of), _ptr(x_perm),
                                    _stream(stream))
    _check(st, "moe_dispatch_noalloc")


def moe_dispatch_noalloc_status(stream=None) -> int:
    """Flags word of the last moe_dispatch_noalloc on the current device
    (synchronises the stream)."""
    flags = ctypes.c_int32()
    st = lib().moe_dispatch_noalloc_status(_stream(stream), ctypes.byref(flags))
    if st not in (MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BOUNDS):
        _check(st, "moe_dispatch_noalloc_status")
    return flags.value


def moe_expert_ffn(cfg, x_perm, offsets, perm, topk_w, w_gate, w_up, w_down, h, y_perm, workspace,
                   stream=None):
    st = lib().moe_expert_ffn(_cfg(cfg), _ptr(x_perm), _ptr(offsets), _ptr(perm), _ptr(topk_w),
                              _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(h), _ptr(y_perm),
                              _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(st, "moe_expert_ffn")


def moe_combine(cfg, y_perm, row_of, y, y_add=None, stream=None):
    st = lib().moe_combine(_cfg(cfg), _ptr(y_perm), _ptr(row_of), _ptr(y_add), _ptr(y),
                           _stream(stream))
    _check(st, "moe_combine")


def moe_forward(cfg, x, w_router, w_gate, w_up, w_down, y, workspace, router_bias=None,
                logit_noise=None, losses=None, mean_prob=None, counts=None, topk_ids=None,
                topk_w=None, selection_bias=None, shared=None, w_router_terms=None, stream=None):
    """shared = (w_gate_s, w_up_s, w_down_s) when cfg.F_shared > 0."""
    sg, su, sd = shared if shared is not None else (None, None, None)
    st = lib().moe_forward(_cfg(cfg), _ptr(x), _ptr(w_router), _ptr(w_router_terms),
                           _ptr(router_bias),
                           _ptr(selection_bias), _ptr(logit_noise), _ptr(w_gate), _ptr(w_up),
                           _ptr(w_down), _ptr(sg), _ptr(su), _ptr(sd), _ptr(y),
                           _ptr(losses), _ptr(mean_prob), _ptr(counts), _ptr(topk_ids),
                           _ptr(topk_w), _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(st, "moe_forward")


def train_state_size(cfg: MoeConfig) -> int:
    v = ctypes.c_size_t()
    _check(lib().moe_train_state_size(_cfg(cfg), ctypes.byref(v)), "moe_train_state_size")
    return v.value


def backward_workspace_size(cfg: MoeConfig) -> int:
    v = ctypes.c_size_t()
    _check(lib().moe_backward_workspace_size(_cfg(cfg), ctypes.byref(v)),
           "moe_backward_workspace_size")
    return v.value


def moe_forward_train(cfg, x, w_router, w_gate, w_up, w_down, y, state, router_bias=None,
                      logit_noise=None, losses=None, mean_prob=None, counts=None, topk_ids=None,
                      topk_w=None, selection_bias=None, shared=None, stream=None):
    """moe_forward that keeps the backward's activations in ``state``."""
    sg, su, sd = shared if shared is not None else (None, None, None)
    st = lib().moe_forward_train(_cfg(cfg), _ptr(x), _ptr(w_router), _ptr(router_bias),
                                 _ptr(selection_bias), _ptr(logit_noise), _ptr(w_gate), _ptr(w_up),
                                 _ptr(w_down), _ptr(sg), _ptr(su), _ptr(sd), _ptr(y),
                                 _ptr(losses), _ptr(mean_prob), _ptr(counts), _ptr(topk_ids),
                                 _ptr(topk_w), _ptr(state), _nbytes(state), _stream(stream))
    _check(st, "moe_forward_train")


def moe_backward(cfg, x, w_router, w_gate, w_up, w_down, state, dy, dx, dw_router, dw_gate, dw_up,
                 dw_down, workspace, c_balance: float = 0.0, c_z: float = 0.0, db_router=None,
                 shared=None, dshared=None, stream=None):
    """shared = (w_gate_s, w_up_s, w_down_s) and dshared = their fp32
    gradient buffers when cfg.F_shared > 0."""
    sg, su, sd = shared if shared is not None else (None, None, None)
    dg, du, dd = dshared if dshared is not None else (None, None, None)
    st = lib().moe_backward(_cfg(cfg), _ptr(x), _ptr(w_router), _ptr(w_gate), _ptr(w_up),
                            _ptr(w_down), _ptr(sg), _ptr(su), _ptr(sd), _ptr(state), _nbytes(state),
                            _ptr(dy), float(c_balance), float(c_z), _ptr(dx), _ptr(dw_router),
                            _ptr(db_router), _ptr(dw_gate), _ptr(dw_up), _ptr(dw_down), _ptr(dg),
                            _ptr(du), _ptr(dd), _ptr(workspace), _nbytes(workspace),
                            _stream(stream))
    _check(st, "moe_backward")


def backward_kernel_count(cfg: MoeConfig) -> int:
    """Kernels one moe_backward launches for this configuration."""
    return int(lib().moe_backward_kernel_count(_cfg(cfg)))


def moe_update_selection_bias(cfg, counts, gamma: float, selection_bias, stream=None):
    """selection_bias += gamma * sign(mean(counts) - counts), on the device."""
    _check(lib().moe_update_selection_bias(_cfg(cfg), _ptr(counts), float(gamma),
                                           _ptr(selection_bias), _stream(stream)),
           "moe_update_selection_bias")


def moe_get_device_status(workspace, stream=None) -> int:
    """Flags word of a workspace (synchronises the stream); raises on a set flag."""
    flags = ctypes.c_int32()
    st = lib().moe_get_device_status(_ptr(workspace), _stream(stream), ctypes.byref(flags))
    if st not in (MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BOUNDS):
        _check(st, "moe_get_device_status")
    return flags.value


def moe_clear_device_status(workspace, stream=None):
    _check(lib().moe_clear_device_status(_ptr(workspace), _stream(stream)),
           "moe_clear_device_status")


def moe_selftest_wait_timeout(workspace, limit_ns: int, stream=None):
    _check(lib().moe_selftest_wait_timeout(_ptr(workspace), _nbytes(workspace), int(limit_ns),
                                           _stream(stream)), "moe_selftest_wait_timeout")


def forward_kernel_count(cfg: MoeConfig, router_terms_given: bool = False) -> int:
    """Kernels one moe_forward launches for this configuration."""
    return int(lib().moe_forward_kernel_count(_cfg(cfg), int(bool(router_terms_given))))


def moe_trace_attach(events):
    """Attach torch.cuda.Event objects (or raw cudaEvent_t ints); [] detaches.

    torch creates an event's CUDA handle lazily, at its first record; events
    without a handle are recorded once here so that one exists."""
    handles = []
    for e in events:
        if not isinstance(e, int) and not e.cuda_event:
            e.record()
        handles.append(e if isinstance(e, int) else e.cuda_event)
    arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
    _check(lib().moe_trace_attach(arr if handles else None, len(handles)), "moe_trace_attach")


def trace_stage_names() -> list[str]:
    n = lib().moe_trace_boundary_count()
    return [lib().moe_trace_stage_name(i).decode() for i in range(n)]


def _event_handles(events):
    handles = []
    for e in events:
        if not isinstance(e, int) and not e.cuda_event:
            e.record()
        handles.append(e if isinstance(e, int) else e.cuda_event)
    return handles


def moe_trace_attach_backward(events):
    """moe_trace_attach for moe_backward's boundaries."""
    handles = _event_handles(events)
    arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
    _check(lib().moe_trace_attach_backward(arr if handles else None, len(handles)),
           "moe_trace_attach_backward")


def trace_backward_stage_names() -> list[str]:
    n = lib().moe_trace_backward_boundary_count()
    return [lib().moe_trace_backward_stage_name(i).decode() for i in range(n)]


def _nbytes(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        raise ValueError("pass the workspace as a tensor so its size is known")
    return t.numel() * t.element_size()


# ------------------------------------------------------- expert parallelism

def ep_workspace_size(world: int, experts_per_rank: int) -> int:
    v = ctypes.c_size_t()
    _check(lib().moe_ep_workspace_size(int(world), int(experts_per_rank), ctypes.byref(v)),
           "moe_ep_workspace_size")
    return v.value


def moe_ep_layout(world: int, experts_per_rank: int, recv_counts, max_rows: int, offsets, dst_of,
                  src_of, workspace, stream=None):
    _check(lib().moe_ep_layout(int(world), int(experts_per_rank), _ptr(recv_counts), int(max_rows),
                               _ptr(offsets), _ptr(dst_of), _ptr(src_of), _ptr(workspace),
                               _nbytes(workspace), _stream(stream)), "moe_ep_layout")


def moe_permute_rows(inp, idx, n: int, out, workspace, stream=None):
    """out[:n] = inp[idx[:n]] (rows), on the device."""
    row_bytes = inp.stride(0) * inp.element_size()
    _check(lib().moe_permute_rows(_ptr(inp), int(inp.shape[0]), _ptr(idx), int(n), int(row_bytes),
                                  _ptr(out), _ptr(workspace), _stream(stream)), "moe_permute_rows")


def moe_combine_weighted(cfg, y_perm, row_of, topk_w, y, y_add=None, stream=None):
    _check(lib().moe_combine_weighted(_cfg(cfg), _ptr(y_perm), _ptr(row_of), _ptr(topk_w),
                                      _ptr(y_add), _ptr(y), _stream(stream)), "moe_combine_weighted")


# ------------------------------------------ expert parallelism over peer memory

IPC_HANDLE_BYTES = 64


def ipc_alloc(nbytes: int):
    """(device address, handle bytes) of a new peer-mappable buffer."""
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(lib().moe_ipc_alloc(int(nbytes), ctypes.byref(ptr), handle), "moe_ipc_alloc")
    return ptr.value, handle.raw


def ipc_open(handle: bytes) -> int:
    """Device address of another process's buffer, from its handle."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle has 64 bytes")
    ptr = ctypes.c_void_p()
    buf = ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES)
    _check(lib().moe_ipc_open(buf, ctypes.byref(ptr)), "moe_ipc_open")
    return ptr.value


def ipc_close(ptr: int):
    _check(lib().moe_ipc_close(ptr), "moe_ipc_close")


def ipc_free(ptr: int):
    _check(lib().moe_ipc_free(ptr), "moe_ipc_free")


class DeviceBuffer:
    """A raw device buffer seen as a tensor (no copy), through the CUDA array
    interface; keeps nothing alive but the address."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(int(v) for v in shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def as_tensor(ptr: int, shape, dtype):
    """Tensor view of `shape` elements of `dtype` at device address ptr."""
    import torch
    if dtype == torch.bfloat16:  # the array interface has no bf16: view int16 as bf16
        return torch.as_tensor(DeviceBuffer(ptr, shape, "<i2"), device="cuda").view(torch.bfloat16)
    typestr = {torch.float32: "<f4", torch.int32: "<i4", torch.uint8: "|u1"}[dtype]
    return torch.as_tensor(DeviceBuffer(ptr, shape, typestr), device="cuda")


def moe_ep_peer_dispatch(cfg, rank: int, world: int, kept_all, x, topk_ids, row_of, offsets,
                         recv_bufs, recv_rows: int, local_offsets, remote_row, workspace, stream=None):
    """recv_bufs: int64 device tensor of `world` receive-buffer addresses."""
    _check(lib().moe_ep_peer_dispatch(_cfg(cfg), int(rank), int(world), _ptr(kept_all), _ptr(x),
                                      _ptr(topk_ids), _ptr(row_of), _ptr(offsets), _ptr(recv_bufs),
                                      int(recv_rows), _ptr(local_offsets), _ptr(remote_row),
                                      _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "moe_ep_peer_dispatch")


def moe_ep_peer_combine(cfg, world: int, topk_ids, remote_row, topk_w, y_bufs, recv_rows: int, y,
                        workspace, y_add=None, stream=None):
    """y_bufs: int64 device tensor of `world` expert-output buffer addresses."""
    _check(lib().moe_ep_peer_combine(_cfg(cfg), int(world), _ptr(topk_ids), _ptr(remote_row),
                                     _ptr(topk_w), _ptr(y_bufs), int(recv_rows), _ptr(y_add), _ptr(y),
                                     _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "moe_ep_peer_combine")
