"""Thin Python binding over the C ABI in ``include/moe_route.h``.

Argument marshalling only: each function checks tensor dtypes/devices,
allocates outputs the caller did not pass, and calls the C entry point of the
same name on the current CUDA stream.  All arithmetic runs in the CUDA kernels
of ``libmoe_route.so``; there is no CPU fallback, and a missing or unloadable
library raises immediately.
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_route.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_CUDA, MOE_ERR_SCRATCH_TOO_SMALL = 0, 1, 2, 3
MOE_STATIC_LAYOUT_SCRATCH_BYTES = 1 << 20
MOE_DTYPE_F32, MOE_DTYPE_BF16 = 0, 1
MOE_QUANT_NONE, MOE_QUANT_FP8_E4M3_B128 = 0, 1
MOE_STATUS_BAD_INDEX, MOE_STATUS_OVERFLOW, MOE_STATUS_BAD_SLOT, MOE_STATUS_TIMEOUT = 1, 2, 4, 8
MOE_MAX_EXPERTS, MOE_MAX_TOPK = 1024, 32

_P, _I, _L, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t

# name -> (restype, argtypes), the exact C signatures
SIGNATURES = {
    "moe_route_topk": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_dispatch_layout_kernels": (_I, [_I, _I, _I]),
    "moe_selftest_wait_timeout": (_I, [_I, ctypes.c_ulonglong, _P, _P, _P]),
    "moe_dispatch_route_weights": (_I, [_P, _P, _I, _I, _L, _P, _P, _P]),
    "moe_route_sigmoid_grouped": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P, _P]),
    "moe_dispatch_layout_workspace": (_Z, [_I, _I, _I]),
    "moe_dispatch_layout": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _L, _P, _Z, _P, _P]),
    "moe_dispatch": (_I, [_P, _I, _I, _I, _I, _P, _I, _P, _P, _L, _P, _P]),
    "moe_combine_dual_residual": (_I, [_P, _I, _I, _I, _I, _L, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch_layout_static": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _L, _P, _P]),
    "moe_combine_fp8_dual_residual": (_I, [_P, _P, _I, _I, _I, _I, _L, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_combine_dual_residual_backward": (_I, [_P, _P, _P, _I, _I, _I, _I, _L, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch_backward": (_I, [_P, _I, _I, _I, _I, _L, _P, _P, _P, _P]),
    "moe_route_topk_backward": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "moe_route_dispatch_workspace": (_Z, [_I, _I, _I]),
    "moe_route_dispatch_kernels": (_I, [_I, _I, _I, _I, _I, _I]),
    "moe_route_dispatch": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _L,
                                _P, _Z, _P, _P]),
    "moe_ep_plan": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_error_string": (ctypes.c_char_p, [_I]),
    "moe_capacity": (_L, [_I, _I, _I, _I]),
}

_lib = None


class MoeError(RuntimeError):
    def __init__(self, fn: str, rc: int):
        msg = lib().moe_error_string(rc).decode()
        super().__init__(f"{fn} failed: {msg} (code {rc})")
        self.rc = rc


def lib() -> ctypes.CDLL:
    """Load libmoe_route.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library missing: {LIB_PATH}; build it with "
                               "`python -m combine_moe_route_09_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device) -> ctypes.c_void_p:
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def _dev(t: torch.Tensor, name: str, dtypes, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    return t


def _dtype_code_of(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return MOE_DTYPE_F32
    if dt == torch.bfloat16:
        return MOE_DTYPE_BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {dt}")


def _dtype_code(t: torch.Tensor) -> int:
    return MOE_DTYPE_F32 if t.dtype == torch.float32 else MOE_DTYPE_BF16


_ACT = (torch.float32, torch.bfloat16)
_FP8 = (torch.float8_e4m3fn, torch.uint8)


def moe_capacity(S: int, E: int, K: int, token_padding: int) -> int:
    return int(lib().moe_capacity(S, E, K, token_padding))


def moe_route_topk(logits: torch.Tensor, K: int, topk_idx=None, topk_w=None, stream=None):
    """Top-K experts per token (descending logit, ties to the lower id) and softmax weights."""
    _dev(logits, "logits", (torch.float32,))
    S, E = logits.shape
    if topk_idx is None:
        topk_idx = torch.empty((S, K), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((S, K), dtype=torch.float32, device=logits.device)
    _dev(topk_idx, "topk_idx", (torch.int32,), (S, K))
    _dev(topk_w, "topk_w", (torch.float32,), (S, K))
    _check("moe_route_topk", lib().moe_route_topk(_ptr(logits), S, E, K, _ptr(topk_idx), _ptr(topk_w),
                                                   _stream(stream, logits.device)))
    return topk_idx, topk_w


def moe_selftest_wait_timeout(which: int, limit_ns: int, status: torch.Tensor, flag=None, stream=None):
    """Runs one bounded wait that nothing completes (0: mbarrier, 1: flag poll); it sets the
    timeout bit in `status` (device int32 [1]) and returns."""
    _dev(status, "status", (torch.int32,), (1,))
    if flag is not None:
        _dev(flag, "flag", (torch.int32,), (1,))
    _check("moe_selftest_wait_timeout", lib().moe_selftest_wait_timeout(
        which, limit_ns, _ptr(status), _ptr(flag), _stream(stream, status.device)))


def moe_dispatch_layout_kernels(S: int, E: int, K: int) -> int:
    """Kernels moe_dispatch_layout launches for these sizes on the current device (1 or 2)."""
    n = lib().moe_dispatch_layout_kernels(S, E, K)
    if n < 0:
        raise MoeError("moe_dispatch_layout_kernels", MOE_ERR_CUDA)
    return n


def moe_dispatch_route_weights(topk_w: torch.Tensor, row_src: torch.Tensor, out=None, status=None, stream=None):
    """Routing weights in dispatched order: out[r] = topk_w.flat[row_src[r]], 0 where row_src < 0."""
    _dev(topk_w, "topk_w", (torch.float32,))
    _dev(row_src, "row_src", (torch.int32,))
    S, K = topk_w.shape
    cap = row_src.shape[0]
    if out is None:
        out = torch.empty(cap, dtype=torch.float32, device=row_src.device)
    _dev(out, "route_weights", (torch.float32,), (cap,))
    _check("moe_dispatch_route_weights", lib().moe_dispatch_route_weights(
        _ptr(topk_w), _ptr(row_src), S, K, cap, _ptr(out), _ptr(status), _stream(stream, row_src.device)))
    return out


def moe_route_sigmoid_grouped(logits: torch.Tensor, K: int, bias=None, n_group: int = 1,
                              topk_group: int = 1, normalize: bool = True, scale: float = 1.0,
                              topk_idx=None, topk_w=None, stream=None):
    """Sigmoid scores, selection-only bias, group-limited top-K (see include/moe_route.h)."""
    _dev(logits, "logits", (torch.float32,))
    S, E = logits.shape
    if bias is not None:
        _dev(bias, "bias", (torch.float32,), (E,))
    if topk_idx is None:
        topk_idx = torch.empty((S, K), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((S, K), dtype=torch.float32, device=logits.device)
    _dev(topk_idx, "topk_idx", (torch.int32,), (S, K))
    _dev(topk_w, "topk_w", (torch.float32,), (S, K))
    _check("moe_route_sigmoid_grouped", lib().moe_route_sigmoid_grouped(
        _ptr(logits), _ptr(bias), S, E, K, n_group, topk_group, int(normalize), float(scale), _ptr(topk_idx),
        _ptr(topk_w), _stream(stream, logits.device)))
    return topk_idx, topk_w


def moe_dispatch_layout_workspace(S: int, E: int, K: int) -> int:
    return int(lib().moe_dispatch_layout_workspace(S, E, K))


class Layout(NamedTuple):
    counts: torch.Tensor        # [E]    tokens_per_expert
    offsets: torch.Tensor       # [E+1]  cu_seqlens of the padded groups
    rank_offsets: torch.Tensor  # [R+1]
    slot_of: torch.Tensor       # [S,K]
    row_src: torch.Tensor       # [cap]
    cap: int


def moe_dispatch_layout(topk_idx: torch.Tensor, E: int, R: int, token_padding: int = 0,
                        cap: Optional[int] = None, *, workspace=None, status=None, out=None,
                        stream=None) -> Layout:
    """Histogram + prefix scan into the padded expert-contiguous layout.

    ``workspace`` (uint8, >= moe_dispatch_layout_workspace bytes) must be zero-filled
    before its first use; each call leaves it ready for the next.  A fresh zeroed
    one is allocated when it is not given.  ``out`` may carry a Layout to write into."""
    _dev(topk_idx, "topk_idx", (torch.int32,))
    S, K = topk_idx.shape
    dev = topk_idx.device
    if cap is None:
        cap = moe_capacity(S, E, K, token_padding)
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                     torch.empty((S, K), **i32), torch.empty(max(cap, 0), **i32), cap)
    need = moe_dispatch_layout_workspace(S, E, K)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", (torch.uint8,))
    if status is not None:
        _dev(status, "status", (torch.int32,))
    _check("moe_dispatch_layout", lib().moe_dispatch_layout(
        _ptr(topk_idx), S, E, K, R, token_padding, _ptr(out.counts), _ptr(out.offsets),
        _ptr(out.rank_offsets), _ptr(out.slot_of), _ptr(out.row_src), cap, _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream, dev)))
    return out._replace(cap=cap)


def moe_dispatch_layout_static(topk_idx: torch.Tensor, E: int, R: int, token_padding: int = 0,
                               cap: Optional[int] = None, *, status=None, out=None,
                               stream=None) -> Layout:
    """moe_dispatch_layout without a workspace, for callers that may not allocate
    device memory where they call it: the scratch is an array built into the
    library (MOE_STATIC_LAYOUT_SCRATCH_BYTES per GPU).  Outputs are allocated here
    only when ``out`` is not given.  Calls that may overlap on the GPU share that
    array and must be serialised; the first call on a device should precede any
    stream capture."""
    _dev(topk_idx, "topk_idx", (torch.int32,))
    S, K = topk_idx.shape
    dev = topk_idx.device
    if cap is None:
        cap = moe_capacity(S, E, K, token_padding)
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                     torch.empty((S, K), **i32), torch.empty(max(cap, 0), **i32), cap)
    if status is not None:
        _dev(status, "status", (torch.int32,))
    _check("moe_dispatch_layout_static", lib().moe_dispatch_layout_static(
        _ptr(topk_idx), S, E, K, R, token_padding, _ptr(out.counts), _ptr(out.offsets),
        _ptr(out.rank_offsets), _ptr(out.slot_of), _ptr(out.row_src), cap, _ptr(status),
        _stream(stream, dev)))
    return out._replace(cap=cap)


def moe_route_dispatch_workspace(S: int, E: int, K: int) -> int:
    return int(lib().moe_route_dispatch_workspace(S, E, K))


def moe_route_dispatch_kernels(S: int, H: int, E: int, K: int, dtype: torch.dtype = torch.bfloat16,
                               quant: int = MOE_QUANT_NONE) -> int:
    """1 when moe_route_dispatch runs as one fused kernel for these sizes on the
    current device, else the number of separate kernels (3 or 4)."""
    return int(lib().moe_route_dispatch_kernels(S, H, E, K, _dtype_code_of(dtype), quant))


def moe_route_dispatch(logits: torch.Tensor, x: torch.Tensor, K: int, R: int, token_padding: int = 0,
                       quant: int = MOE_QUANT_NONE, cap: Optional[int] = None, *, topk_idx=None, topk_w=None,
                       layout: Optional[Layout] = None, xd=None, xs=None, workspace=None, status=None,
                       stream=None):
    """Router top-K, dispatch layout and dispatch in one call (one kernel when the
    batch fits).  Returns (topk_idx, topk_w, layout, xd, xs), exactly what
    moe_route_topk, moe_dispatch_layout and moe_dispatch would return.

    ``workspace`` (uint8, >= moe_route_dispatch_workspace bytes) must be
    zero-filled before its first use; a fresh one is allocated if not given."""
    _dev(logits, "logits", (torch.float32,))
    _dev(x, "x", _ACT)
    S, E = logits.shape
    H = x.shape[1]
    _dev(x, "x", _ACT, (S, H))
    dev = x.device
    if cap is None:
        cap = moe_capacity(S, E, K, token_padding)
    i32 = dict(dtype=torch.int32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty((S, K), **i32)
    if topk_w is None:
        topk_w = torch.empty((S, K), dtype=torch.float32, device=dev)
    _dev(topk_idx, "topk_idx", (torch.int32,), (S, K))
    _dev(topk_w, "topk_w", (torch.float32,), (S, K))
    if layout is None:
        layout = Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                        torch.empty((S, K), **i32), torch.empty(max(cap, 0), **i32), cap)
    if quant == MOE_QUANT_FP8_E4M3_B128:
        if xd is None:
            xd = torch.empty((cap, H), dtype=torch.float8_e4m3fn, device=dev)
        if xs is None:
            xs = torch.empty((cap, H // 128), dtype=torch.float32, device=dev)
        _dev(xd, "xd", (torch.float8_e4m3fn, torch.uint8), (cap, H))
        _dev(xs, "xs", (torch.float32,), (cap, H // 128))
    else:
        if xd is None:
            xd = torch.empty((cap, H), dtype=x.dtype, device=dev)
        _dev(xd, "xd", (x.dtype,), (cap, H))
    need = moe_route_dispatch_workspace(S, E, K)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", (torch.uint8,))
    if status is not None:
        _dev(status, "status", (torch.int32,))
    _check("moe_route_dispatch", lib().moe_route_dispatch(
        _ptr(logits), _ptr(x), _dtype_code(x), S, H, E, K, R, token_padding, quant, _ptr(topk_idx), _ptr(topk_w),
        _ptr(layout.counts), _ptr(layout.offsets), _ptr(layout.rank_offsets), _ptr(layout.slot_of),
        _ptr(layout.row_src), _ptr(xd), _ptr(xs), cap, _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream, dev)))
    return topk_idx, topk_w, layout._replace(cap=cap), xd, xs


def moe_dispatch(x: torch.Tensor, slot_of: torch.Tensor, cap: int, quant: int = MOE_QUANT_NONE,
                 xd=None, xs=None, status=None, stream=None):
    """Scatter rows of x [S,H] into xd [cap,H]; with FP8 also scales xs [cap,H/128]."""
    _dev(x, "x", _ACT)
    S, H = x.shape
    K = slot_of.shape[1]
    _dev(slot_of, "slot_of", (torch.int32,), (S, K))
    if quant == MOE_QUANT_FP8_E4M3_B128:
        if xd is None:
            xd = torch.empty((cap, H), dtype=torch.float8_e4m3fn, device=x.device)
        if xs is None:
            xs = torch.empty((cap, H // 128), dtype=torch.float32, device=x.device)
        _dev(xd, "xd", _FP8, (cap, H))
        _dev(xs, "xs", (torch.float32,), (cap, H // 128))
    else:
        if xd is None:
            xd = torch.empty((cap, H), dtype=x.dtype, device=x.device)
        _dev(xd, "xd", (x.dtype,), (cap, H))
    if status is not None:
        _dev(status, "status", (torch.int32,))
    _check("moe_dispatch", lib().moe_dispatch(_ptr(x), _dtype_code(x), S, H, K, _ptr(slot_of), quant,
                                               _ptr(xd), _ptr(xs), cap, _ptr(status),
                                               _stream(stream, x.device)))
    return xd, xs


def moe_combine_dual_residual(y: torch.Tensor, slot_of: torch.Tensor, topk_w: torch.Tensor,
                              shared_out=None, residual=None, residual_out=None,
                              residual_no_routed_out=None, want_no_routed: bool = True,
                              status=None, stream=None):
    """Weighted gather back to token order with the FarSkip dual-residual epilogue.

    Returns (residual_out, residual_no_routed_out); the second is None unless both
    shared_out and residual are given (and want_no_routed)."""
    _dev(y, "y", _ACT)
    cap, H = y.shape
    S, K = slot_of.shape
    _dev(slot_of, "slot_of", (torch.int32,))
    _dev(topk_w, "topk_w", (torch.float32,), (S, K))
    for name, t in (("shared_out", shared_out), ("residual", residual)):
        if t is not None:
            _dev(t, name, (y.dtype,), (S, H))
    if residual_out is None:
        residual_out = torch.empty((S, H), dtype=y.dtype, device=y.device)
    _dev(residual_out, "residual_out", (y.dtype,), (S, H))
    if residual_no_routed_out is None and want_no_routed and shared_out is not None \
            and residual is not None:
        residual_no_routed_out = torch.empty((S, H), dtype=y.dtype, device=y.device)
    if residual_no_routed_out is not None:
        _dev(residual_no_routed_out, "residual_no_routed_out", (y.dtype,), (S, H))
    if status is not None:
        _dev(status, "status", (torch.int32,))
    _check("moe_combine_dual_residual", lib().moe_combine_dual_residual(
        _ptr(y), _dtype_code(y), S, H, K, cap, _ptr(slot_of), _ptr(topk_w), _ptr(shared_out),
        _ptr(residual), _ptr(residual_out), _ptr(residual_no_routed_out), _ptr(status),
        _stream(stream, y.device)))
    return residual_out, residual_no_routed_out


def moe_combine_fp8_dual_residual(yq: torch.Tensor, ys: torch.Tensor, slot_of: torch.Tensor,
                                  topk_w: torch.Tensor, shared_out=None, residual=None, residual_out=None,
                                  residual_no_routed_out=None, want_no_routed: bool = True,
                                  dtype: torch.dtype = torch.bfloat16, status=None, stream=None):
    """moe_combine_dual_residual over FP8 expert outputs: yq [cap,H] e4m3 codes and
    ys [cap,H/128] fp32 block scales; outputs (and shared_out/residual) in ``dtype``."""
    _dev(yq, "yq", _FP8)
    cap, H = yq.shape
    S, K = slot_of.shape
    _dev(ys, "ys", (torch.float32,), (cap, H // 128))
    _dev(slot_of, "slot_of", (torch.int32,))
    _dev(topk_w, "topk_w", (torch.float32,), (S, K))
    for name, t in (("shared_out", shared_out), ("residual", residual)):
        if t is not None:
            _dev(t, name, (dtype,), (S, H))
    if residual_out is None:
        residual_out = torch.empty((S, H), dtype=dtype, device=yq.device)
    _dev(residual_out, "residual_out", (dtype,), (S, H))
    if residual_no_routed_out is None and want_no_routed and shared_out is not None and residual is not None:
        residual_no_routed_out = torch.empty((S, H), dtype=dtype, device=yq.device)
    if residual_no_routed_out is not None:
        _dev(residual_no_routed_out, "residual_no_routed_out", (dtype,), (S, H))
    if status is not None:
        _dev(status, "status", (torch.int32,))
    code = MOE_DTYPE_F32 if dtype == torch.float32 else MOE_DTYPE_BF16
    _check("moe_combine_fp8_dual_residual", lib().moe_combine_fp8_dual_residual(
        _ptr(yq), _ptr(ys), code, S, H, K, cap, _ptr(slot_of), _ptr(topk_w), _ptr(shared_out), _ptr(residual),
        _ptr(residual_out), _ptr(residual_no_routed_out), _ptr(status), _stream(stream, yq.device)))
    return residual_out, residual_no_routed_out


# ----------------------------------------------------------------------------------------------
# backward (training): the transposes of the forward steps, through the same layout
# ----------------------------------------------------------------------------------------------

def moe_combine_dual_residual_backward(grad_out: torch.Tensor, y: torch.Tensor, slot_of: torch.Tensor,
                                       topk_w: torch.Tensor, grad_no_routed=None, grad_y=None,
                                       grad_w=None, grad_skip=None, want_skip: bool = True,
                                       status=None, stream=None):
    """Returns (grad_y [cap,H], grad_w [S,K] fp32, grad_skip [S,H] or None).

    grad_skip is the gradient of both ``residual`` and ``shared_out``.  grad_y
    rows that no pair maps to are not written (allocated with zeros here)."""
    _dev(y, "y", _ACT)
    cap, H = y.shape
    S, K = slot_of.shape
    _dev(grad_out, "grad_out", (y.dtype,), (S, H))
    _dev(slot_of, "slot_of", (torch.int32,))
    _dev(topk_w, "topk_w", (torch.float32,), (S, K))
    if grad_no_routed is not None:
        _dev(grad_no_routed, "grad_no_routed", (y.dtype,), (S, H))
    if grad_y is None:
        grad_y = torch.zeros((cap, H), dtype=y.dtype, device=y.device)
    if grad_w is None:
        grad_w = torch.empty((S, K), dtype=torch.float32, device=y.device)
    if grad_skip is None and want_skip:
        grad_skip = torch.empty((S, H), dtype=y.dtype, device=y.device)
    _dev(grad_y, "grad_y", (y.dtype,), (cap, H))
    _dev(grad_w, "grad_w", (torch.float32,), (S, K))
    if grad_skip is not None:
        _dev(grad_skip, "grad_skip", (y.dtype,), (S, H))
    if status is not None:
        _dev(status, "status", (torch.int32,))
    _check("moe_combine_dual_residual_backward", lib().moe_combine_dual_residual_backward(
        _ptr(grad_out), _ptr(grad_no_routed), _ptr(y), _dtype_code(y), S, H, K, cap, _ptr(slot_of),
        _ptr(topk_w), _ptr(grad_y), _ptr(grad_w), _ptr(grad_skip), _ptr(status), _stream(stream, y.device)))
    return grad_y, grad_w, grad_skip


def moe_dispatch_backward(grad_xd: torch.Tensor, slot_of: torch.Tensor, grad_x=None, status=None,
                          stream=None):
    """grad_x [S,H] = sum of the K copies' gradients (straight through for FP8)."""
    _dev(grad_xd, "grad_xd", _ACT)
    cap, H = grad_xd.shape
    S, K = slot_of.shape
    _dev(slot_of, "slot_of", (torch.int32,))
    if grad_x is None:
        grad_x = torch.empty((S, H), dtype=grad_xd.dtype, device=grad_xd.device)
    _dev(grad_x, "grad_x", (grad_xd.dtype,), (S, H))
    if status is not None:
        _dev(status, "status", (torch.int32,))
    _check("moe_dispatch_backward", lib().moe_dispatch_backward(
        _ptr(grad_xd), _dtype_code(grad_xd), S, H, K, cap, _ptr(slot_of), _ptr(grad_x), _ptr(status),
        _stream(stream, grad_xd.device)))
    return grad_x


def moe_route_topk_backward(topk_idx: torch.Tensor, topk_w: torch.Tensor, grad_w: torch.Tensor, E: int,
                            grad_logits=None, stream=None):
    """grad_logits [S,E] fp32 through the gating softmax over the selected logits."""
    _dev(topk_idx, "topk_idx", (torch.int32,))
    S, K = topk_idx.shape
    _dev(topk_w, "topk_w", (torch.float32,), (S, K))
    _dev(grad_w, "grad_w", (torch.float32,), (S, K))
    if grad_logits is None:
        grad_logits = torch.empty((S, E), dtype=torch.float32, device=topk_idx.device)
    _dev(grad_logits, "grad_logits", (torch.float32,), (S, E))
    _check("moe_route_topk_backward", lib().moe_route_topk_backward(
        _ptr(topk_idx), _ptr(topk_w), _ptr(grad_w), S, E, K, _ptr(grad_logits),
        _stream(stream, topk_idx.device)))
    return grad_logits
