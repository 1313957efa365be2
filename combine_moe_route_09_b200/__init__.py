"""B200-native (sm_100a) MoE token dispatch and combine.

The four calls of one MoE routing pass, each a C-ABI entry point of
``libmoe_route.so`` with a thin binding of the same name:

* :func:`moe_route_topk` — router top-K gating
* :func:`moe_dispatch_layout` — per-expert histogram + prefix scan into the
  padded expert-contiguous layout
* :func:`moe_dispatch` — row scatter, optionally FP8 e4m3 per 128 channels
* :func:`moe_combine_dual_residual` — weighted gather with the FarSkip
  dual-residual epilogue

:func:`moe_route_dispatch` runs the first three as one call (one kernel when
that is faster); :class:`buffer.MoeBuffer` preallocates one pass;
:mod:`ep` runs the pass with experts spread over several GPUs.

Importing the package does not load the library; the first call does, and
raises if it is missing.
"""
from .binding import (  # noqa: F401
    MOE_DTYPE_BF16,
    MOE_DTYPE_F32,
    MOE_ERR_CUDA,
    MOE_ERR_INVALID_ARG,
    MOE_ERR_SCRATCH_TOO_SMALL,
    MOE_MAX_EXPERTS,
    MOE_MAX_TOPK,
    MOE_OK,
    MOE_QUANT_FP8_E4M3_B128,
    MOE_QUANT_NONE,
    MOE_STATIC_LAYOUT_SCRATCH_BYTES,
    MOE_STATUS_BAD_INDEX,
    MOE_STATUS_BAD_SLOT,
    MOE_STATUS_OVERFLOW,
    MOE_STATUS_TIMEOUT,
    Layout,
    MoeError,
    lib,
    moe_capacity,
    moe_combine_dual_residual,
    moe_combine_dual_residual_backward,
    moe_combine_fp8_dual_residual,
    moe_dispatch,
    moe_dispatch_backward,
    moe_dispatch_layout,
    moe_dispatch_layout_kernels,
    moe_dispatch_layout_static,
    moe_dispatch_layout_workspace,
    moe_dispatch_route_weights,
    moe_route_dispatch,
    moe_route_dispatch_kernels,
    moe_route_dispatch_workspace,
    moe_route_sigmoid_grouped,
    moe_route_topk,
    moe_route_topk_backward,
    moe_selftest_wait_timeout,
)
