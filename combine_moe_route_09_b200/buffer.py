"""Preallocated buffers for one MoE routing pass, in the shape of MoonEP's
``Buffer(S, H, K, E, num_ep_ranks)`` ("MoonEP developer guide", core API
example): construct once, then dispatch/combine every layer through the same
device memory.

All device memory is allocated here, once, by PyTorch; the C entry points only
read and write it.  One pass is four calls on one stream, with no host
synchronisation:

    route_topk -> dispatch_layout -> dispatch -> (experts) -> combine_dual_residual

The per-call argument lists for the buffers owned here are built once; an
input tensor is validated the first time it is seen (and again whenever its
storage, shape or dtype changes), so a steady-state step costs four C calls.
"""
from __future__ import annotations

import ctypes
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
                 dtype: torch.dtype = torch.bfloat16, fp8: bool = False, device="cuda",
                 fused: Optional[bool] = None):
        if dtype not in (torch.float32, torch.bfloat16):
            raise TypeError("activations must be float32 or bfloat16")
        self.S, self.H, self.K, self.E, self.R, self.P = S, H, K, E, R, token_padding
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.dtype, self.fp8, self.device = dtype, fp8, dev
        self.cap = B.moe_capacity(S, E, K, token_padding)
        if self.cap < 0:
            raise ValueError("invalid sizes")
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_idx = torch.empty((S, K), **i32)
        self.topk_w = torch.empty((S, K), dtype=torch.float32, device=dev)
        self.layout = B.Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32),
                               torch.empty(R + 1, **i32), torch.empty((S, K), **i32),
                               torch.empty(self.cap, **i32), self.cap)
        ws = max(B.moe_dispatch_layout_workspace(S, E, K), B.moe_route_dispatch_workspace(S, E, K))
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
        self._lib = B.lib()
        self._seen = {}
        self._dt = B.MOE_DTYPE_F32 if dtype == torch.float32 else B.MOE_DTYPE_BF16
        p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        L = self.layout
        self._p_idx, self._p_w, self._p_status = p(self.topk_idx), p(self.topk_w), p(self.status)
        self._layout_args = (p(self.topk_idx), S, E, K, R, token_padding, p(L.counts), p(L.offsets),
                             p(L.rank_offsets), p(L.slot_of), p(L.row_src), self.cap,
                             p(self.workspace), self.workspace.numel(), p(self.status))
        self._p_slot, self._p_xd = p(L.slot_of), p(self.xd)
        self._p_xs = p(self.xs) if fp8 else None
        self._p_out, self._p_rnr = p(self.out), p(self.out_no_routed)
        self._rd_args = (S, H, E, K, R, token_padding, self.quant, p(self.topk_idx), p(self.topk_w), p(L.counts),
                         p(L.offsets), p(L.rank_offsets), p(L.slot_of), p(L.row_src), self._p_xd, self._p_xs,
                         self.cap, p(self.workspace), self.workspace.numel(), p(self.status))
        # route + layout + dispatch as one fused kernel when it applies to these sizes
        # on this device: fused=True forces it, False never uses it, None (default)
        # times both plans once (they give identical outputs) and keeps the faster
        with torch.cuda.device(self.device):
            applies = B.moe_route_dispatch_kernels(S, H, E, K, dtype, self.quant) == 1
        self.fused = applies and fused is not False
        self.plan_timings_us = None
        if applies and fused is None:
            self._choose_plan()

    @property
    def kernels_per_step(self) -> int:
        """Kernels one step launches: fused route + layout + dispatch 1, combine 1; or
        route 1, layout 1 or 2, dispatch 1, combine 1."""
        if self.fused:
            return 2
        with torch.cuda.device(self.device):
            return 3 + B.moe_dispatch_layout_kernels(self.S, self.E, self.K)

    @property
    def quant(self) -> int:
        return B.MOE_QUANT_FP8_E4M3_B128 if self.fp8 else B.MOE_QUANT_NONE

    def _in(self, t: torch.Tensor, name: str, dtypes, shape) -> ctypes.c_void_p:
        key = (name, t.data_ptr(), tuple(t.shape), t.dtype, t.is_contiguous())
        ptr = self._seen.get(name)
        if ptr is None or ptr[0] != key:
            B._dev(t, name, dtypes, shape)
            if t.device != self.device:
                raise ValueError(f"{name} is on {t.device}, buffers are on {self.device}")
            ptr = (key, ctypes.c_void_p(t.data_ptr()))
            self._seen[name] = ptr
        return ptr[1]

    def _stream(self, stream) -> ctypes.c_void_p:
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        return ctypes.c_void_p(s.cuda_stream)

    # -- the four calls ---------------------------------------------------------------
    def route(self, logits: torch.Tensor, stream=None):
        pl = self._in(logits, "logits", (torch.float32,), (self.S, self.E))
        B._check("moe_route_topk", self._lib.moe_route_topk(pl, self.S, self.E, self.K, self._p_idx,
                                                             self._p_w, self._stream(stream)))
        return self.topk_idx, self.topk_w

    def plan(self, topk_idx: Optional[torch.Tensor] = None, stream=None) -> B.Layout:
        """Layout of self.topk_idx (or of the given ids, written to this buffer's layout)."""
        args = self._layout_args
        if topk_idx is not None:
            args = (self._in(topk_idx, "topk_idx", (torch.int32,), (self.S, self.K)),) + args[1:]
        B._check("moe_dispatch_layout", self._lib.moe_dispatch_layout(*args, self._stream(stream)))
        return self.layout

    def route_dispatch(self, logits: torch.Tensor, x: torch.Tensor, stream=None):
        """route + plan + dispatch as one call (one kernel when the batch fits)."""
        pl = self._in(logits, "logits", (torch.float32,), (self.S, self.E))
        px = self._in(x, "x", (self.dtype,), (self.S, self.H))
        a = self._rd_args
        B._check("moe_route_dispatch", self._lib.moe_route_dispatch(
            pl, px, self._dt, *a, self._stream(stream)))
        return self.xd, self.xs

    def dispatch(self, x: torch.Tensor, stream=None):
        px = self._in(x, "x", (self.dtype,), (self.S, self.H))
        B._check("moe_dispatch", self._lib.moe_dispatch(px, self._dt, self.S, self.H, self.K, self._p_slot,
                                                         self.quant, self._p_xd, self._p_xs, self.cap,
                                                         self._p_status, self._stream(stream)))
        return self.xd, self.xs

    def combine(self, y: torch.Tensor, shared_out=None, residual=None, topk_w=None, stream=None):
        py = self._in(y, "y", (self.dtype,), (self.cap, self.H))
        ps = None if shared_out is None else self._in(shared_out, "shared_out", (self.dtype,), (self.S, self.H))
        pr = None if residual is None else self._in(residual, "residual", (self.dtype,), (self.S, self.H))
        pw = self._p_w if topk_w is None else self._in(topk_w, "topk_w", (torch.float32,), (self.S, self.K))
        fused = ps is not None and pr is not None
        B._check("moe_combine_dual_residual", self._lib.moe_combine_dual_residual(
            py, self._dt, self.S, self.H, self.K, self.cap, self._p_slot, pw, ps, pr, self._p_out,
            self._p_rnr if fused else None, self._p_status, self._stream(stream)))
        return self.out, (self.out_no_routed if fused else None)

    def step_phases(self, logits, x, y, shared_out=None, residual=None, stream=None):
        """The calls of one full pass, in order, as (phase name, zero-argument call)
        pairs; running them in order is one step (y = expert outputs)."""
        if self.fused:
            return [
                ("route_dispatch", lambda: self.route_dispatch(logits, x, stream)),
                ("combine", lambda: self.combine(y, shared_out, residual, stream=stream)),
            ]
        return [
            ("route", lambda: self.route(logits, stream)),
            ("layout", lambda: self.plan(stream=stream)),
            ("dispatch", lambda: self.dispatch(x, stream)),
            ("combine", lambda: self.combine(y, shared_out, residual, stream=stream)),
        ]

    def step(self, logits, x, y, shared_out=None, residual=None, stream=None):
        """One full pass: route, layout, dispatch, combine (y = expert outputs)."""
        for _, call in self.step_phases(logits, x, y, shared_out, residual, stream):
            call()
        return self.out, (self.out_no_routed if (shared_out is not None and residual is not None) else None)

    def capture(self, logits, x, y, shared_out=None, residual=None, steps: int = 1):
        """Records `steps` consecutive steps into a CUDA graph and returns it
        (``graph.replay()`` reruns them).  The graph reads the given input tensors
        and writes this buffer's outputs at fixed addresses: refill the inputs in
        place between replays.  Run one eager step first (kernel attributes are set
        on first use)."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(steps):
                self.step(logits, x, y, shared_out, residual)
        return g

    def _choose_plan(self, calls: int = 10, reps: int = 5):
        """Times whole steps both ways -- route + layout + dispatch as the fused
        kernel or as the separate kernels, then the combine -- on synthetic inputs
        of this buffer's shapes (expert outputs, shared and residual rows drawn
        for the purpose and freed after), each as a CUDA graph of `calls` steps,
        and keeps the faster plan (median of `reps`).  The combine is timed too
        because the plan changes what it finds in L2.  Both plans write identical
        outputs; only the speed differs."""
        dev = self.device
        gen = torch.Generator(device=dev).manual_seed(0)
        logits = torch.randn((self.S, self.E), generator=gen, device=dev)
        x = torch.randn((self.S, self.H), generator=gen, device=dev).to(self.dtype)
        y = torch.randn((self.cap, self.H), generator=gen, device=dev).to(self.dtype)
        sh = torch.randn((self.S, self.H), generator=gen, device=dev).to(self.dtype)
        rs = torch.randn((self.S, self.H), generator=gen, device=dev).to(self.dtype)
        side = torch.cuda.Stream(dev)
        times = {}
        with torch.cuda.device(dev):
            for fused in (True, False):
                self.fused = fused
                self.step(logits, x, y, sh, rs)
                torch.cuda.synchronize(dev)
                g = torch.cuda.CUDAGraph()
                side.wait_stream(torch.cuda.current_stream(dev))
                with torch.cuda.graph(g, stream=side):
                    for _ in range(calls):
                        self.step(logits, x, y, sh, rs)
                g.replay()
                torch.cuda.synchronize(dev)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                ts = []
                for _ in range(reps):
                    a.record()
                    g.replay()
                    b.record()
                    torch.cuda.synchronize(dev)
                    ts.append(a.elapsed_time(b) * 1e3 / calls)
                del g
                times["fused" if fused else "separate"] = sorted(ts)[len(ts) // 2]
        del logits, x, y, sh, rs
        self.fused = times["fused"] <= times["separate"]
        self.plan_timings_us = times
        self._seen.clear()
        self.read_status()

    def read_status(self) -> int:
        """Reads and clears the device status word (synchronises).  After a
        timeout the workspace is zeroed again, as its contract asks."""
        v = int(self.status.item())
        self.status.zero_()
        if v & B.MOE_STATUS_TIMEOUT:
            self.workspace.zero_()
        return v
