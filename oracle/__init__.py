"""CPU oracle for MoE dispatch/combine — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product path never does.

This is a thin ctypes shim over ``moe_oracle.c`` (the plain single-threaded
definition of each step; see the header comment there for the sources and the
precision of every step).  Arrays are numpy; bf16 tensors are carried as
``uint16`` bit patterns and FP8 codes as ``uint8``.  Nothing here shares code
with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, EINVAL, EINDEX, EOVERFLOW = 0, 1, 2, 3
DTYPE_F32, DTYPE_BF16 = 0, 1
QUANT_NONE, QUANT_FP8_E4M3_B128 = 0, 1

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_int64
        lib.oracle_route_topk.argtypes = [P, I, I, I, P, P]
        lib.oracle_layout.argtypes = [P, I, I, I, I, I, L, P, P, P, P, P]
        lib.oracle_dispatch.argtypes = [P, I, I, I, I, P, I, L, P, P]
        lib.oracle_combine.argtypes = [P, I, I, I, I, L, P, P, P, P, P, P]
        lib.oracle_route_sigmoid_grouped.argtypes = [P, P, I, I, I, I, I, I, ctypes.c_float, P, P]
        lib.oracle_route_exp.argtypes = [ctypes.c_float]
        lib.oracle_route_exp.restype = ctypes.c_float
        lib.oracle_route_sigmoid.argtypes = [ctypes.c_float]
        lib.oracle_route_sigmoid.restype = ctypes.c_float
        lib.oracle_combine_fp8.argtypes = [P, P, I, I, I, I, L, P, P, P, P, P, P]
        lib.oracle_combine_backward.argtypes = [P, P, P, I, I, I, I, L, P, P, P, P, P]
        lib.oracle_dispatch_backward.argtypes = [P, I, I, I, I, L, P, P]
        lib.oracle_route_backward.argtypes = [P, P, P, I, I, I, P]
        lib.oracle_route_weights_dispatched.argtypes = [P, P, I, I, L, P]
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_float
        lib.oracle_bf16_round.argtypes = [ctypes.c_float]
        lib.oracle_bf16_round.restype = ctypes.c_uint16
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    def __init__(self, name: str, rc: int):
        super().__init__(f"{name} returned {rc}")
        self.rc = rc


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def _dtype_code(a) -> int:
    if a.dtype == np.float32:
        return DTYPE_F32
    if a.dtype == np.uint16:
        return DTYPE_BF16
    raise TypeError(f"activation arrays must be float32 or uint16 (bf16 bits), got {a.dtype}")


def route_topk(logits: np.ndarray, K: int):
    """Top-K experts per token and their gating weights. logits: float32 [S,E]."""
    logits = _c(logits, np.float32)
    S, E = logits.shape
    idx = np.empty((S, K), np.int32)
    w = np.empty((S, K), np.float32)
    rc = _load().oracle_route_topk(_ptr(logits), S, E, K, _ptr(idx), _ptr(w))
    if rc:
        raise OracleError("oracle_route_topk", rc)
    return idx, w


def route_sigmoid_grouped(logits, K: int, bias=None, n_group: int = 1, topk_group: int = 1,
                          normalize: bool = True, scale: float = 1.0):
    """Sigmoid scores, selection-only bias, group-limited top-K; see moe_oracle.c."""
    logits = _c(logits, np.float32)
    S, E = logits.shape
    bias = None if bias is None else _c(bias, np.float32)
    idx = np.empty((S, K), np.int32)
    w = np.empty((S, K), np.float32)
    rc = _load().oracle_route_sigmoid_grouped(_ptr(logits), _ptr(bias), S, E, K, n_group, topk_group,
                                              int(normalize), float(scale), _ptr(idx), _ptr(w))
    if rc:
        raise OracleError("oracle_route_sigmoid_grouped", rc)
    return idx, w


def route_exp(x: np.ndarray) -> np.ndarray:
    f = _load().oracle_route_exp
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()], np.float32)


def route_sigmoid(x: np.ndarray) -> np.ndarray:
    f = _load().oracle_route_sigmoid
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()], np.float32)


def capacity(S: int, E: int, K: int, P: int) -> int:
    """Row capacity that always fits the padded layout: S*K + E*max(P-1, 0)."""
    return S * K + E * max(P - 1, 0)


def layout(topk_idx: np.ndarray, E: int, R: int, P: int, cap: int | None = None):
    """Counts, padded offsets, rank offsets, slot_of [S,K] and row_src [cap]."""
    topk_idx = _c(topk_idx, np.int32)
    S, K = topk_idx.shape
    if cap is None:
        cap = capacity(S, E, K, P)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    rank_offsets = np.empty(R + 1, np.int32)
    slot_of = np.empty((S, K), np.int32)
    row_src = np.empty(cap, np.int32)
    rc = _load().oracle_layout(_ptr(topk_idx), S, E, K, R, P, cap, _ptr(counts), _ptr(offsets),
                               _ptr(rank_offsets), _ptr(slot_of), _ptr(row_src))
    if rc:
        raise OracleError("oracle_layout", rc)
    return dict(counts=counts, offsets=offsets, rank_offsets=rank_offsets, slot_of=slot_of,
                row_src=row_src, cap=cap)


def dispatch(x: np.ndarray, slot_of: np.ndarray, cap: int, quant: int = QUANT_NONE,
             xd: np.ndarray | None = None, xs: np.ndarray | None = None):
    """Scatter rows of x [S,H] to xd [cap,H]; with FP8 also the scales xs [cap,H/128].

    Rows that no pair maps to keep whatever ``xd``/``xs`` held (zeros if not given)."""
    x = np.ascontiguousarray(x)
    slot_of = _c(slot_of, np.int32)
    S, H = x.shape
    K = slot_of.shape[1]
    if quant == QUANT_FP8_E4M3_B128:
        if xd is None:
            xd = np.zeros((cap, H), np.uint8)
        if xs is None:
            xs = np.zeros((cap, H // 128), np.float32)
    elif xd is None:
        xd = np.zeros((cap, H), x.dtype)
    rc = _load().oracle_dispatch(_ptr(x), _dtype_code(x), S, H, K, _ptr(slot_of), quant, cap,
                                 _ptr(xd), _ptr(xs))
    if rc:
        raise OracleError("oracle_dispatch", rc)
    return xd, xs


def combine(y: np.ndarray, slot_of: np.ndarray, topk_w: np.ndarray, shared=None, residual=None,
            want_no_routed: bool = True):
    """Weighted gather back to token order, fused with the dual residual.

    Returns (out, out_no_routed); out_no_routed is None unless both shared and
    residual are given and want_no_routed is true."""
    y = np.ascontiguousarray(y)
    slot_of = _c(slot_of, np.int32)
    topk_w = _c(topk_w, np.float32)
    S, K = slot_of.shape
    cap, H = y.shape
    for a in (shared, residual):
        if a is not None:
            assert a.dtype == y.dtype and a.shape == (S, H)
    shared = None if shared is None else np.ascontiguousarray(shared)
    residual = None if residual is None else np.ascontiguousarray(residual)
    out = np.empty((S, H), y.dtype)
    rnr = np.empty((S, H), y.dtype) if (want_no_routed and shared is not None
                                         and residual is not None) else None
    rc = _load().oracle_combine(_ptr(y), _dtype_code(y), S, H, K, cap, _ptr(slot_of), _ptr(topk_w),
                                _ptr(shared), _ptr(residual), _ptr(out), _ptr(rnr))
    if rc:
        raise OracleError("oracle_combine", rc)
    return out, rnr


def combine_fp8(yq, ys, slot_of, topk_w, shared=None, residual=None, dtype="bf16",
                want_no_routed: bool = True):
    """Combine over e4m3 expert outputs yq [cap,H] (uint8) with scales ys [cap,H/128].

    The outputs (and shared/residual, if given) are in ``dtype`` ("bf16" or "f32")."""
    yq = _c(yq, np.uint8)
    ys = _c(ys, np.float32)
    slot_of = _c(slot_of, np.int32)
    topk_w = _c(topk_w, np.float32)
    S, K = slot_of.shape
    cap, H = yq.shape
    code = DTYPE_BF16 if dtype == "bf16" else DTYPE_F32
    npdt = np.uint16 if dtype == "bf16" else np.float32
    shared = None if shared is None else _c(shared, npdt)
    residual = None if residual is None else _c(residual, npdt)
    out = np.empty((S, H), npdt)
    rnr = np.empty((S, H), npdt) if (want_no_routed and shared is not None and residual is not None) else None
    rc = _load().oracle_combine_fp8(_ptr(yq), _ptr(ys), code, S, H, K, cap, _ptr(slot_of), _ptr(topk_w),
                                    _ptr(shared), _ptr(residual), _ptr(out), _ptr(rnr))
    if rc:
        raise OracleError("oracle_combine_fp8", rc)
    return out, rnr


def combine_backward(g, y, slot_of, topk_w, gn=None, grad_y=None, want_skip=True):
    """Backward of combine: (grad_y [cap,H], grad_w [S,K] fp32, grad_skip [S,H] or None).

    grad_y rows that no pair maps to keep what ``grad_y`` held (zeros if not given)."""
    g = np.ascontiguousarray(g)
    y = np.ascontiguousarray(y)
    slot_of = _c(slot_of, np.int32)
    topk_w = _c(topk_w, np.float32)
    S, K = slot_of.shape
    cap, H = y.shape
    assert g.dtype == y.dtype and g.shape == (S, H)
    if gn is not None:
        gn = np.ascontiguousarray(gn)
        assert gn.dtype == y.dtype and gn.shape == (S, H)
    if grad_y is None:
        grad_y = np.zeros((cap, H), y.dtype)
    grad_w = np.empty((S, K), np.float32)
    skip = np.empty((S, H), y.dtype) if want_skip else None
    rc = _load().oracle_combine_backward(_ptr(g), _ptr(gn), _ptr(y), _dtype_code(y), S, H, K, cap,
                                         _ptr(slot_of), _ptr(topk_w), _ptr(grad_y), _ptr(grad_w),
                                         _ptr(skip))
    if rc:
        raise OracleError("oracle_combine_backward", rc)
    return grad_y, grad_w, skip


def dispatch_backward(grad_xd, slot_of, S=None):
    """Backward of the plain dispatch: grad_x [S,H] = sum of the K copies' gradients."""
    grad_xd = np.ascontiguousarray(grad_xd)
    slot_of = _c(slot_of, np.int32)
    S, K = slot_of.shape
    cap, H = grad_xd.shape
    grad_x = np.empty((S, H), grad_xd.dtype)
    rc = _load().oracle_dispatch_backward(_ptr(grad_xd), _dtype_code(grad_xd), S, H, K, cap,
                                          _ptr(slot_of), _ptr(grad_x))
    if rc:
        raise OracleError("oracle_dispatch_backward", rc)
    return grad_x


def route_backward(topk_idx, topk_w, grad_w, E: int):
    """Backward of the gating softmax: grad_logits [S,E] fp32."""
    topk_idx = _c(topk_idx, np.int32)
    topk_w = _c(topk_w, np.float32)
    grad_w = _c(grad_w, np.float32)
    S, K = topk_idx.shape
    out = np.empty((S, E), np.float32)
    rc = _load().oracle_route_backward(_ptr(topk_idx), _ptr(topk_w), _ptr(grad_w), S, E, K, _ptr(out))
    if rc:
        raise OracleError("oracle_route_backward", rc)
    return out


def route_weights_dispatched(topk_w, slot_of, cap: int):
    """Routing weights in dispatched order: float32 [cap], 0 on rows no pair fills."""
    topk_w = _c(topk_w, np.float32)
    slot_of = _c(slot_of, np.int32)
    S, K = slot_of.shape
    out = np.empty(cap, np.float32)
    rc = _load().oracle_route_weights_dispatched(_ptr(topk_w), _ptr(slot_of), S, K, cap, _ptr(out))
    if rc:
        raise OracleError("oracle_route_weights_dispatched", rc)
    return out


def e4m3_encode(v: float) -> int:
    return int(_load().oracle_e4m3_encode(float(v)))


def e4m3_decode(q: int) -> float:
    return float(_load().oracle_e4m3_decode(int(q)))


def bf16_round(v: float) -> int:
    return int(_load().oracle_bf16_round(float(v)))
