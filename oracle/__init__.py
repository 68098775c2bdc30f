"""CPU fp64 oracle of the token-choice top-k MoE layer: forward and backward.

TEST INFRASTRUCTURE ONLY: this package is the checker the CUDA library is
compared against.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the library itself never does, and
it imports nothing from the library.

The arithmetic lives in ``moe_oracle.c`` (plain loops, double precision); this
module builds it with gcc, marshals numpy arrays in and out through ctypes, and
strings the steps together in the order the pages give them
("Lab: build a tiny MoE in PyTorch", section "Full implementation" and
"Add a capacity limit").

Inputs may be numpy arrays or CPU torch tensors: fp32 arrays, or bf16 data
given either as a torch bfloat16 tensor or as raw uint16 words.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_moe.so")
_lib = None
_lock = threading.Lock()

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle_moe.so (gcc, OpenMP, -O2)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
            lib.oracle_router_logits.argtypes = [i64, i32, i32, P, i32, P, P, P, P]
            lib.oracle_router_logits.restype = None
            lib.oracle_route.argtypes = [i64, i32, i32, P, i32, i32, P, i32, i32, f64, P, P, P, P, P]
            lib.oracle_route.restype = i32
            lib.oracle_update_bias.argtypes = [i32, P, f64, P]
            lib.oracle_update_bias.restype = None
            lib.oracle_router_stats.argtypes = [i64, i32, i32, P, P, P, P, P, P, P]
            lib.oracle_router_stats.restype = None
            lib.oracle_capacity.argtypes = [i64, i32, i32, f64]
            lib.oracle_capacity.restype = i64
            lib.oracle_dispatch.argtypes = [i64, i32, i32, P, i64, P, P, P, P, P]
            lib.oracle_dispatch.restype = None
            lib.oracle_gather.argtypes = [i64, i32, i32, P, i32, P, P]
            lib.oracle_gather.restype = None
            lib.oracle_expert_rows.argtypes = [i64, i32, i32, P, P, P, P, i32, P]
            lib.oracle_expert_rows.restype = None
            lib.oracle_combine.argtypes = [i64, i32, i32, P, P, P, P]
            lib.oracle_combine.restype = None
            lib.oracle_router_backward.argtypes = [i64, i32, i32, P, P, P, P, i32, i32, f64, f64,
                                                   f64, P]
            lib.oracle_router_backward.restype = None
            lib.oracle_router_linear_backward.argtypes = [i64, i32, i32, P, i32, P, P, P, P, P]
            lib.oracle_router_linear_backward.restype = None
            lib.oracle_expert_backward_rows.argtypes = [i64, P, P, P, i32, i32, P, i32, P, P, P, P,
                                                        i32, P, P, P, P, P]
            lib.oracle_expert_backward_rows.restype = None
            lib.oracle_expert_backward_cols.argtypes = [i64, P, P, P, i32, i32, i32, P, P, i32, P,
                                                        P, P, P, i32, P, P, P]
            lib.oracle_expert_backward_cols.restype = None
            lib.oracle_expert_wgrad.argtypes = [i64, P, P, i32, i32, P, i32, P, P, P, P, P, P, P]
            lib.oracle_expert_wgrad.restype = None
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = i32
            lib.oracle_set_num_threads.argtypes = [i32]
            lib.oracle_set_num_threads.restype = None
            _lib = lib
    return _lib


def _elem_array(a):
    """Return (contiguous numpy array, element-type code) for fp32 / bf16 data."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach()
            if a.device.type != "cpu":
                raise ValueError("oracle inputs must be CPU tensors")
            if a.dtype == torch.bfloat16:
                return np.ascontiguousarray(a.contiguous().view(torch.int16).numpy().view(np.uint16)), BF16
            a = a.contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a), BF16
    if a.dtype == np.float32:
        return np.ascontiguousarray(a), F32
    raise TypeError(f"unsupported element type {a.dtype}")


def _f32(a):
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(np.asarray(a))
    if a.dtype != np.float32:
        raise TypeError("expected fp32 data")
    return a


def _i32(a):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _f64(a):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu()
            if a.dtype == torch.bfloat16:
                a = a.double()  # exact widening
            a = a.contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's parallel loops from now on (results do not
    depend on it)."""
    _load().oracle_set_num_threads(int(n))


def router_logits(x, w_router, bias=None, noise=None) -> np.ndarray:
    """L[t,e] = x[t] . W_r[:, e] (+ b[e]) (+ noise[t,e]) in fp64, shape (T, E)."""
    lib = _load()
    xa, xd = _elem_array(x)
    w = _f32(w_router)
    b, nz = _f32(bias), _f32(noise)
    T, D = xa.shape
    E = w.shape[1]
    out = np.empty((T, E), dtype=np.float64)
    lib.oracle_router_logits(T, D, E, _ptr(xa), xd, _ptr(w), _ptr(b), _ptr(nz), _ptr(out))
    return out


SCORE_FUNCS = {"softmax": 0, "sigmoid": 1}


def route(logits, K: int, score_func: str = "softmax", renormalize: bool = True, sel_bias=None,
          n_groups: int = 1, topk_groups: int = 1, route_scale: float = 1.0,
          with_entropy: bool = False):
    """Scores, (group-limited) top-K on (logit + selection bias desc, id asc),
    and the weights of the selected experts.

    ``logits`` is (T, E), any real type (fp32 logits convert exactly).
    Returns ids (T,K) int32, weights (T,K) f64, probs (T,E) f64 (the scores
    normalised per token), lse (T,) f64, and with ``with_entropy`` the
    per-token entropy (T,) of the softmax probabilities.
    """
    lib = _load()
    L = _f64(logits)
    T, E = L.shape
    if not 1 <= K <= E:
        raise ValueError("top_k must be in [1, n_experts]")
    if n_groups > 1 and (E % n_groups or not 1 <= topk_groups <= n_groups
                         or topk_groups * (E // n_groups) < K):
        raise ValueError("invalid expert groups")
    b = None if sel_bias is None else _f64(sel_bias)
    ids = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float64)
    probs = np.empty((T, E), dtype=np.float64)
    lse = np.empty((T,), dtype=np.float64)
    ent = np.empty((T,), dtype=np.float64)
    rc = lib.oracle_route(T, E, K, _ptr(L), SCORE_FUNCS[score_func], int(bool(renormalize)),
                          _ptr(b), int(n_groups), int(topk_groups), float(route_scale), _ptr(ids),
                          _ptr(w), _ptr(probs), _ptr(lse), _ptr(ent))
    if rc != 0:
        raise ValueError("non-finite router logit")
    if with_entropy:
        return ids, w, probs, lse, ent
    return ids, w, probs, lse


def update_bias(bias, counts, gamma: float) -> np.ndarray:
    """DeepSeek-V3 selection-bias step: b_e += gamma * sign(mean(counts) - counts_e)."""
    lib = _load()
    b = _f64(bias).copy()
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.int64))
    lib.oracle_update_bias(b.shape[0], _ptr(c), float(gamma), _ptr(b))
    return b


def router_stats(ids, probs, lse, E: int):
    """counts (E,) int64, mean_prob (E,), z_loss, balance_loss."""
    lib = _load()
    ids = _i32(ids)
    probs, lse = _f64(probs), _f64(lse)
    T, K = ids.shape
    counts = np.empty((E,), dtype=np.int64)
    mp = np.empty((E,), dtype=np.float64)
    z = ctypes.c_double()
    bal = ctypes.c_double()
    lib.oracle_router_stats(T, E, K, _ptr(ids), _ptr(probs), _ptr(lse), _ptr(counts), _ptr(mp),
                            ctypes.byref(z), ctypes.byref(bal))
    return counts, mp, z.value, bal.value


def capacity(T: int, K: int, E: int, capacity_factor: float) -> int:
    return int(_load().oracle_capacity(T, K, E, float(capacity_factor)))


def dispatch(ids, E: int, C: int) -> dict:
    """counts, kept, offsets (E+1), perm (sum kept), row_of (T*K) -- all int32."""
    lib = _load()
    ids = _i32(ids)
    T, K = ids.shape
    counts = np.empty((E,), np.int32)
    kept = np.empty((E,), np.int32)
    offsets = np.empty((E + 1,), np.int32)
    perm = np.full((T * K,), -1, np.int32)
    row_of = np.empty((T * K,), np.int32)
    lib.oracle_dispatch(T, K, E, _ptr(ids), int(C), _ptr(counts), _ptr(kept), _ptr(offsets),
                        _ptr(perm), _ptr(row_of))
    R = int(offsets[-1])
    return dict(counts=counts, kept=kept, offsets=offsets, perm=perm[:R].copy(), row_of=row_of)


def gather(x, perm, K: int) -> np.ndarray:
    lib = _load()
    xa, xd = _elem_array(x)
    perm = _i32(perm)
    R = perm.shape[0]
    D = xa.shape[1]
    out = np.empty((R, D), np.float64)
    lib.oracle_gather(R, D, K, _ptr(xa), xd, _ptr(perm), _ptr(out))
    return out


def expert_rows(rows, w_gate_e, w_up_e, w_down_e) -> np.ndarray:
    """Unweighted SwiGLU expert output for each row of ``rows`` (n, D)."""
    lib = _load()
    rows = _f64(rows)
    wg, wdt = _elem_array(w_gate_e)
    wu, wdt2 = _elem_array(w_up_e)
    wd, wdt3 = _elem_array(w_down_e)
    if not (wdt == wdt2 == wdt3):
        raise TypeError("expert weights must share one element type")
    n, D = rows.shape
    F = wg.shape[1]
    assert wg.shape == (D, F) and wu.shape == (D, F) and wd.shape == (F, D)
    out = np.empty((n, D), np.float64)
    if n:
        lib.oracle_expert_rows(n, D, F, _ptr(rows), _ptr(wg), _ptr(wu), _ptr(wd), wdt, _ptr(out))
    return out


def combine(o, row_of, weights, T: int, K: int) -> np.ndarray:
    lib = _load()
    o = _f64(o)
    row_of = _i32(row_of)
    w = _f64(weights)
    D = o.shape[1] if o.ndim == 2 and o.shape[0] else None
    if D is None:
        raise ValueError("combine needs the row width: pass o with shape (R, D), R >= 1")
    y = np.empty((T, D), np.float64)
    lib.oracle_combine(T, K, D, _ptr(o), _ptr(row_of), _ptr(w), _ptr(y))
    return y


def _expert_slice(w, e):
    return w[e]


def forward(x, w_router, w_gate, w_up, w_down, K: int, capacity_factor: float = 0.0,
            bias=None, noise=None, logits=None, shared=None, **routing) -> dict:
    """The whole layer: route -> dispatch -> experts -> combine.

    When ``logits`` is given (T, E) the router GEMM is skipped and the layer is
    routed from those logits (parity mode: the CUDA path's fp32 logits).
    ``routing`` passes the router options of ``route`` (score_func,
    renormalize, sel_bias, n_groups, topk_groups, route_scale).
    ``shared`` = (w_gate_s (D, Fs), w_up_s (D, Fs), w_down_s (Fs, D)) adds a
    shared SwiGLU expert that every token passes through ("Lab: build a tiny
    MoE in PyTorch", "Add a shared expert": routed + shared_expert(x)).
    Returns every intermediate: logits, ids, weights, probs, lse, entropy,
    counts, mean_prob, z_loss, balance_loss, capacity, kept, offsets, perm,
    row_of, o (unweighted expert outputs per row), row_weight (w per row), y.
    """
    xa, _ = _elem_array(x)
    T, D = xa.shape
    E = _f32(w_router).shape[1]
    L = router_logits(x, w_router, bias, noise) if logits is None else _f64(logits)
    ids, w, probs, lse, ent = route(L, K, with_entropy=True, **routing)
    counts64, mean_prob, z, bal = router_stats(ids, probs, lse, E)
    C = capacity(T, K, E, capacity_factor)
    dsp = dispatch(ids, E, C)
    perm, offsets = dsp["perm"], dsp["offsets"]
    x_perm = gather(x, perm, K)
    R = perm.shape[0]
    o = np.zeros((R, D), np.float64)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            o[a:b] = expert_rows(x_perm[a:b], _expert_slice(w_gate, e), _expert_slice(w_up, e),
                                 _expert_slice(w_down, e))
    wflat = w.reshape(-1)
    row_weight = wflat[perm] if R else np.zeros((0,), np.float64)
    y = combine(o, dsp["row_of"], w, T, K) if R else np.zeros((T, D), np.float64)
    y_shared = None
    if shared is not None:
        y_shared = expert_rows(_f64(x), shared[0], shared[1], shared[2])
        y = y + y_shared
    return dict(logits=L, ids=ids, weights=w, probs=probs, lse=lse, entropy=float(ent.mean()),
                counts=dsp["counts"],
                mean_prob=mean_prob, z_loss=z, balance_loss=bal, capacity=C, kept=dsp["kept"],
                offsets=offsets, perm=perm, row_of=dsp["row_of"], x_perm=x_perm, o=o,
                row_weight=row_weight, y_shared=y_shared, y=y)


def slot_outputs(x_rows, slot_ids, slot_kept, get_expert) -> np.ndarray:
    """Unweighted expert output of every kept (token, slot) of a few tokens.

    x_rows (n, D); slot_ids / slot_kept (n, K); get_expert(e) -> (w_gate_e,
    w_up_e, w_down_e) host arrays of one expert.  Returns (n, K, D), zero rows
    for dropped slots.  Experts are visited one at a time so a caller can
    stream large weights.
    """
    xr = _f64(x_rows)
    n, D = xr.shape
    ids = np.asarray(slot_ids)
    kp = np.asarray(slot_kept, dtype=bool)
    K = ids.shape[1]
    outs = np.zeros((n, K, D), np.float64)
    for e in sorted(set(int(v) for v in ids[kp].reshape(-1))):
        sel = [(i, k) for i in range(n) for k in range(K) if kp[i, k] and int(ids[i, k]) == e]
        wg, wu, wd = get_expert(e)
        o = expert_rows(xr[[i for i, _ in sel]], wg, wu, wd)
        for j, (i, k) in enumerate(sel):
            outs[i, k] = o[j]
    return outs


def token_outputs(x_rows, slot_ids, slot_weights, slot_kept, get_expert, outs=None) -> np.ndarray:
    """Direct per-token layer output for a few tokens ("Trace one token by hand").

    y[i] = sum over kept slots, in slot order, of w * expert(x_i).  ``outs``
    may pass precomputed slot_outputs.
    """
    ws = np.asarray(slot_weights, dtype=np.float64)
    kp = np.asarray(slot_kept, dtype=bool)
    if outs is None:
        outs = slot_outputs(x_rows, slot_ids, kp, get_expert)
    n, K, D = outs.shape
    y = np.zeros((n, D), np.float64)
    for i in range(n):
        for k in range(K):
            if kp[i, k]:
                y[i] += ws[i, k] * outs[i, k]
    return y


# ----------------------------------------------------------------- backward
#
# The gradient of  loss = sum <dY, y> + c_bal * balance + c_z * z  ("Lab: build
# a tiny MoE in PyTorch", "Smoke test and backward pass"), with the top-k
# decision as a stop-gradient ("2.9 Mixture-of-Experts (MoE) Architectures",
# "The Router").  The arithmetic is in moe_oracle.c; these wrappers marshal.


def router_backward(logits, ids, dw, counts, c_bal: float = 0.0, c_z: float = 0.0,
                     score_func: str = "softmax", renormalize: bool = True,
                     route_scale: float = 1.0) -> np.ndarray:
    """dL (T, E): gradient of the router logits from the gate-weight
    gradients dw (T, K), the balance loss (coefficient c_bal, counts fixed) and
    the z-loss (coefficient c_z)."""
    lib = _load()
    L = _f64(logits)
    ids = _i32(ids)
    T, E = L.shape
    K = ids.shape[1]
    dw = _f64(dw).reshape(T, K)
    cnt = np.ascontiguousarray(np.asarray(counts, dtype=np.int64))
    out = np.empty((T, E), np.float64)
    lib.oracle_router_backward(T, E, K, _ptr(L), _ptr(ids), _ptr(dw), _ptr(cnt),
                               SCORE_FUNCS[score_func], int(bool(renormalize)), float(route_scale),
                               float(c_bal), float(c_z), _ptr(out))
    return out


def router_linear_backward(x, w_router, dlogits):
    """(dW_r (D, E), db (E,), dx_r (T, D)) of L = x W_r + b."""
    lib = _load()
    xa, xd = _elem_array(x)
    w = _f32(w_router)
    dL = _f64(dlogits)
    T, D = xa.shape
    E = w.shape[1]
    dw = np.empty((D, E), np.float64)
    db = np.empty((E,), np.float64)
    dx = np.empty((T, D), np.float64)
    lib.oracle_router_linear_backward(T, D, E, _ptr(xa), xd, _ptr(w), _ptr(dL), _ptr(dw), _ptr(db),
                                      _ptr(dx))
    return dw, db, dx


def _weights3(w_gate, w_up, w_down):
    wg, t1 = _elem_array(w_gate)
    wu, t2 = _elem_array(w_up)
    wd, t3 = _elem_array(w_down)
    if not (t1 == t2 == t3):
        raise TypeError("expert weights must share one element type")
    if wg.ndim == 2:  # one expert (a shared expert): (D, F), (D, F), (F, D)
        wg, wu, wd = wg[None], wu[None], wd[None]
    return np.ascontiguousarray(wg), np.ascontiguousarray(wu), np.ascontiguousarray(wd), t1


def expert_backward_rows(tok, ex, wt, x, dy, w_gate, w_up, w_down, intermediates: bool = False):
    """Per-row expert backward: dw (n,), dx (n, D) and, with ``intermediates``,
    h, dg, du (n, F).  Row r is token tok[r] through expert ex[r] with gate
    weight wt[r]; weights (E, D, F), (E, D, F), (E, F, D) or one expert's 2-D
    matrices."""
    lib = _load()
    xa, xd = _elem_array(x)
    wg, wu, wd, wdt = _weights3(w_gate, w_up, w_down)
    dyd = _f64(dy)
    tok, ex, wt = _i32(tok), _i32(ex), _f64(wt)
    n = tok.shape[0]
    D, F = wg.shape[1], wg.shape[2]
    dw = np.zeros((n,), np.float64)
    dx = np.zeros((n, D), np.float64)
    h = np.zeros((n, F), np.float64) if intermediates else None
    dg = np.zeros((n, F), np.float64) if intermediates else None
    du = np.zeros((n, F), np.float64) if intermediates else None
    if n:
        lib.oracle_expert_backward_rows(n, _ptr(tok), _ptr(ex), _ptr(wt), D, F, _ptr(xa), xd,
                                        _ptr(dyd), _ptr(wg), _ptr(wu), _ptr(wd), wdt, _ptr(dw),
                                        _ptr(dx), _ptr(h), _ptr(dg), _ptr(du))
    if intermediates:
        return dw, dx, h, dg, du
    return dw, dx


def expert_backward_cols(tok, ex, wt, fcols, x, dy, w_gate, w_up, w_down):
    """h, dg, du (n, len(fcols)) of the given rows at hidden columns fcols."""
    lib = _load()
    xa, xd = _elem_array(x)
    wg, wu, wd, wdt = _weights3(w_gate, w_up, w_down)
    dyd = _f64(dy)
    tok, ex, wt, fc = _i32(tok), _i32(ex), _f64(wt), _i32(fcols)
    n, nf = tok.shape[0], fc.shape[0]
    D, F = wg.shape[1], wg.shape[2]
    h = np.zeros((n, nf), np.float64)
    dg = np.zeros((n, nf), np.float64)
    du = np.zeros((n, nf), np.float64)
    if n:
        lib.oracle_expert_backward_cols(n, _ptr(tok), _ptr(ex), _ptr(wt), D, F, nf, _ptr(fc),
                                        _ptr(xa), xd, _ptr(dyd), _ptr(wg), _ptr(wu), _ptr(wd), wdt,
                                        _ptr(h), _ptr(dg), _ptr(du))
    return h, dg, du


def expert_wgrad(tok, wt, x, dy, h, dg, du):
    """(dWg (D, F'), dWu (D, F'), dWd (F', D)) of one expert from its rows in
    row order; F' = h.shape[1] (all hidden columns, or a sampled subset)."""
    lib = _load()
    xa, xd = _elem_array(x)
    dyd = _f64(dy)
    tok, wt = _i32(tok), _f64(wt)
    h, dg, du = _f64(h), _f64(dg), _f64(du)
    n = tok.shape[0]
    D = xa.shape[1]
    F = h.shape[1] if h.ndim == 2 else 0
    dWg = np.zeros((D, F), np.float64)
    dWu = np.zeros((D, F), np.float64)
    dWd = np.zeros((F, D), np.float64)
    lib.oracle_expert_wgrad(n, _ptr(tok), _ptr(wt), D, F, _ptr(xa), xd, _ptr(dyd), _ptr(h),
                            _ptr(dg), _ptr(du), _ptr(dWg), _ptr(dWu), _ptr(dWd))
    return dWg, dWu, dWd


def backward(x, w_router, w_gate, w_up, w_down, dy, K: int, capacity_factor: float = 0.0,
             bias=None, noise=None, logits=None, shared=None, c_bal: float = 0.0,
             c_z: float = 0.0, **routing) -> dict:
    """Gradients of the whole layer for upstream gradient dy (T, D) of y and
    loss coefficients c_bal (balance) and c_z (z-loss).

    Runs the oracle forward first (same arguments as ``forward``), then: each
    kept row's expert backward (dw, dx, h, dg, du); the gate-weight gradient
    of every slot (0 for a dropped one); the router-logit gradient; the
    router's linear map; the experts' weight gradients (rows in order); the
    shared expert.  dx = sum over kept slots (slot order) of the rows' dx,
    plus the shared expert's, plus the router's.
    Returns dx, dw_router, db_router, dw_gate, dw_up, dw_down, dlogits,
    dw_slot, dshared (tuple or None) and fwd (the forward's dict).
    """
    fwd = forward(x, w_router, w_gate, w_up, w_down, K, capacity_factor, bias=bias, noise=noise,
                  logits=logits, shared=shared, **routing)
    xa, _ = _elem_array(x)
    T, D = xa.shape
    wg_all, _, _, _ = _weights3(w_gate, w_up, w_down)
    E, F = wg_all.shape[0], wg_all.shape[2]
    dyd = _f64(dy)
    perm, offsets, row_of = fwd["perm"], fwd["offsets"], fwd["row_of"]
    R = perm.shape[0]
    tok = (perm // K).astype(np.int32)
    ex = np.repeat(np.arange(E, dtype=np.int32), np.diff(offsets))
    wt = fwd["row_weight"]
    dw_rows, dx_rows, h, dg, du = expert_backward_rows(tok, ex, wt, x, dyd, w_gate, w_up, w_down,
                                                       intermediates=True)
    dw_slot = np.zeros((T * K,), np.float64)
    dw_slot[perm] = dw_rows
    counts = np.asarray(fwd["counts"], dtype=np.int64)
    sf = routing.get("score_func", "softmax")
    dL = router_backward(fwd["logits"], fwd["ids"], dw_slot.reshape(T, K), counts, c_bal, c_z,
                         score_func=sf, renormalize=routing.get("renormalize", True),
                         route_scale=routing.get("route_scale", 1.0))
    dWr, db, dx_r = router_linear_backward(x, w_router, dL)
    dx = (combine(dx_rows, row_of, np.ones((T, K)), T, K) if R
          else np.zeros((T, D), np.float64))
    dWg = np.zeros((E, D, F), np.float64)
    dWu = np.zeros((E, D, F), np.float64)
    dWd = np.zeros((E, F, D), np.float64)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        dWg[e], dWu[e], dWd[e] = expert_wgrad(tok[a:b], wt[a:b], x, dyd, h[a:b], dg[a:b], du[a:b])
    dshared = None
    if shared is not None:
        ts = np.arange(T, dtype=np.int32)
        _, dx_s, hs, dgs, dus = expert_backward_rows(ts, np.zeros(T, np.int32), np.ones(T), x, dyd,
                                                     shared[0], shared[1], shared[2],
                                                     intermediates=True)
        dx = dx + dx_s
        dshared = expert_wgrad(ts, np.ones(T), x, dyd, hs, dgs, dus)
    dx = dx + dx_r
    return dict(dx=dx, dw_router=dWr, db_router=db, dw_gate=dWg, dw_up=dWu, dw_down=dWd,
                dlogits=dL, dw_slot=dw_slot.reshape(T, K), dshared=dshared, fwd=fwd)
