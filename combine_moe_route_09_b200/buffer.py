"""Preallocated buffers for one MoE routing pass, in the shape of MoonEP's
``Buffer(S, H, K, E, num_ep_ranks)`` ("MoonEP developer guide", core API
example): construct once, then dispatch/combine every layer through the same
device memory.

All device memory is allocated here, once, by PyTorch; the C entry points only
read and write it.  One pass is four calls on one stream, with no host
synchronisation:

    route_topk -> dispatch_layout -> dispatch -> (experts) -> combine_dual_residual
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class MoeBuffer:
    """Device buffers and the four calls of one routing pass.

    S tokens (all logical ranks), hidden H, K experts per token, E experts, R
    logical ranks, token_padding P (0 = none); dtype of activations (float32
    or bfloat16); fp8 = dispatch quantised to e4m3 with 128-channel scales.
    """

    def __init__(self, S: int, H: int, K: int, E: int, R: int = 1, token_padding: int = 0,
                 dtype: torch.dtype = torch.bfloat16, fp8: bool = False, device="cuda"):
        self.S, self.H, self.K, self.E, self.R, self.P = S, H, K, E, R, token_padding
        self.dtype, self.fp8, self.device = dtype, fp8, torch.device(device)
        self.cap = B.moe_capacity(S, E, K, token_padding)
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_idx = torch.empty((S, K), **i32)
        self.topk_w = torch.empty((S, K), dtype=torch.float32, device=dev)
        self.layout = B.Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32),
                               torch.empty(R + 1, **i32), torch.empty((S, K), **i32),
                               torch.empty(self.cap, **i32), self.cap)
        ws = B.moe_dispatch_layout_workspace(S, E, K)
        self.workspace = torch.zeros(max(ws, 256), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, **i32)
        if fp8:
            self.xd = torch.empty((self.cap, H), dtype=torch.float8_e4m3fn, device=dev)
            self.xs = torch.empty((self.cap, H // 128), dtype=torch.float32, device=dev)
        else:
            self.xd = torch.empty((self.cap, H), dtype=dtype, device=dev)
            self.xs = None
        self.out = torch.empty((S, H), dtype=dtype, device=dev)
        self.out_no_routed = torch.empty((S, H), dtype=dtype, device=dev)

    @property
    def quant(self) -> int:
        return B.MOE_QUANT_FP8_E4M3_B128 if self.fp8 else B.MOE_QUANT_NONE

    # -- the four calls ---------------------------------------------------------------
    def route(self, logits: torch.Tensor, stream=None):
        return B.moe_route_topk(logits, self.K, self.topk_idx, self.topk_w, stream=stream)

    def plan(self, topk_idx: Optional[torch.Tensor] = None, stream=None) -> B.Layout:
        idx = self.topk_idx if topk_idx is None else topk_idx
        return B.moe_dispatch_layout(idx, self.E, self.R, self.P, self.cap, workspace=self.workspace,
                                     status=self.status, out=self.layout, stream=stream)

    def dispatch(self, x: torch.Tensor, stream=None):
        return B.moe_dispatch(x, self.layout.slot_of, self.cap, self.quant, self.xd, self.xs,
                              status=self.status, stream=stream)

    def combine(self, y: torch.Tensor, shared_out=None, residual=None, topk_w=None, stream=None):
        fused = shared_out is not None and residual is not None
        return B.moe_combine_dual_residual(
            y, self.layout.slot_of, self.topk_w if topk_w is None else topk_w, shared_out, residual,
            self.out, self.out_no_routed if fused else None, want_no_routed=fused,
            status=self.status, stream=stream)

    def step(self, logits, x, y, shared_out=None, residual=None, stream=None):
        """One full pass: route, layout, dispatch, combine (y = expert outputs)."""
        self.route(logits, stream)
        self.plan(stream=stream)
        self.dispatch(x, stream)
        return self.combine(y, shared_out, residual, stream=stream)

    # kernels one step launches (route 1, layout 2, dispatch 1, combine 1)
    KERNELS_PER_STEP = 5

    def read_status(self) -> int:
        """Reads and clears the device status word (synchronises)."""
        v = int(self.status.item())
        self.status.zero_()
        return v
