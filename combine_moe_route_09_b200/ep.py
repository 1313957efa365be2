"""Expert parallelism over W ranks, one GPU (one process) per rank.

"Efficient and portable mixture-of-experts communication": experts are split
over the ranks in blocks of E/W (Portable Kernels); a dispatch sends each
token's rows to the ranks owning its experts, which receive the rows of one
expert contiguously (Dispatch); the combine returns the expert outputs to the
token's rank and takes the router-weighted sum there (Combine).  "MoonEP
developer guide", core API example: Buffer(S, H, K, E, num_ep_ranks).

How this library does it, rank s holding S_s tokens:

1. route its tokens and build its local layout with R = W logical ranks and no
   padding (moe_route_topk, moe_dispatch_layout): the layout is the send
   buffer, rank-major, expert-contiguous, and moe_dispatch scatters (and, with
   FP8, quantises) the rows into it;
2. exchange the [E] expert counts (an all-gather), after which every rank
   computes the same receive plan on the host (moe_ep_plan, C);
3. move the rows: for each (peer, expert) one point-to-point segment, from the
   sender's send buffer straight into its place in the receiver's buffer
   (NCCL send/recv grouped in one batch; a rank's own segments are device
   copies).  Rank d's receive buffer then holds its experts' rows expert-major,
   each expert's rows in (source rank, token) order, padded to token_padding:
   exactly rank d's part of the single-GPU layout of all tokens;
4. after the experts, the combine moves the output rows back along the same
   segments into the source rank's send-order buffer and runs
   moe_combine_dual_residual there with the local layout and weights.

The exchange needs the counts on the host (the segment sizes), so step 2
synchronises each rank's stream once per dispatch.  No load here uses cluster
multicast, and no kernel reads another GPU's memory: rows cross between GPUs
only through NCCL.  The segment bookkeeping (`segments`, `exchange`) works with
any torch.distributed backend, so it runs on CPU tensors with gloo too.
"""
from __future__ import annotations

import ctypes
from typing import List, NamedTuple, Optional, Sequence, Tuple

import numpy as np
import torch

from . import binding as B


class EpPlan(NamedTuple):
    counts: np.ndarray          # [W, E] int32: counts[s][e], pairs of rank s routed to expert e
    expert_offsets: np.ndarray  # [E + 1] int32: padded offsets of the whole batch, rank-major
    recv_offsets: np.ndarray    # [W, W, E/W] int32: [d][s][j] first row of s's rows of expert d*E/W + j in d's buffer
    recv_rows: np.ndarray       # [W] int32: rows of each rank's receive buffer
    send_offsets: np.ndarray    # [W, E + 1] int32: exclusive scan of counts[s] (each rank's send layout)
    W: int
    E: int
    token_padding: int

    @property
    def Eloc(self) -> int:
        return self.E // self.W

    def rank_base(self, d: int) -> int:
        """Row of the whole-batch layout where rank d's receive buffer starts."""
        return int(self.expert_offsets[d * self.Eloc])


def ep_plan(counts: np.ndarray, token_padding: int = 0) -> EpPlan:
    """The receive plan for the all-gathered counts [W, E] (moe_ep_plan, host C)."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    W, E = counts.shape
    eo = np.empty(E + 1, np.int32)
    ro = np.empty((W, W, E // max(W, 1)), np.int32)
    rr = np.empty(W, np.int32)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    B._check("moe_ep_plan", B.lib().moe_ep_plan(p(counts), W, E, token_padding, p(eo), p(ro), p(rr)))
    so = np.zeros((W, E + 1), np.int32)
    so[:, 1:] = np.cumsum(counts, axis=1)
    return EpPlan(counts, eo, ro, rr, so, W, E, token_padding)


def segments(plan: EpPlan, src: int, dst: int) -> List[Tuple[int, int, int]]:
    """(row in src's send buffer, row in dst's receive buffer, rows) of every
    non-empty segment from rank src to rank dst, in local-expert order."""
    out = []
    for j in range(plan.Eloc):
        e = dst * plan.Eloc + j
        n = int(plan.counts[src, e])
        if n:
            out.append((int(plan.send_offsets[src, e]), int(plan.recv_offsets[dst, src, j]), n))
    return out


def exchange(plan: EpPlan, rank: int, send: Sequence[torch.Tensor], recv: Sequence[torch.Tensor],
             group=None, reverse: bool = False):
    """Moves every segment of the plan between this rank's buffers and its peers'.

    dispatch (reverse=False): rows of `send` (this rank's send buffers, send
    layout order) go to the owning ranks' `recv` buffers; reverse=True: the
    combine direction, rows of the owners' buffers (here `send` holds this
    rank's receive-side buffers) come back into the source ranks' send-order
    buffers (`recv`).  Several tensors (for example FP8 codes and their scales)
    move together, one per entry, with the same rows.  Point-to-point segments
    are posted in one batch, in (peer, local expert) order on both sides so
    that each pair's sends and receives match; a rank's own segments are local
    copies."""
    import torch.distributed as dist

    ops = []
    for peer in range(plan.W):
        if reverse:
            # my receive rows (b) back to peer's send layout (a); my send rows (a) from peer's buffer
            out = [(b, n) for (a, b, n) in segments(plan, peer, rank)]
            inc = [(a, n) for (a, b, n) in segments(plan, rank, peer)]
        else:
            out = [(a, n) for (a, b, n) in segments(plan, rank, peer)]
            inc = [(b, n) for (a, b, n) in segments(plan, peer, rank)]
        if peer == rank:
            for (r_out, n), (r_in, _) in zip(out, inc):
                for s_t, r_t in zip(send, recv):
                    r_t[r_in:r_in + n].copy_(s_t[r_out:r_out + n])
            continue
        for (r_out, n) in out:
            for s_t in send:
                ops.append(dist.P2POp(dist.isend, s_t[r_out:r_out + n], peer, group))
        for (r_in, n) in inc:
            for r_t in recv:
                ops.append(dist.P2POp(dist.irecv, r_t[r_in:r_in + n], peer, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def exchange_local(plan: EpPlan, send: Sequence[Sequence[torch.Tensor]], recv: Sequence[Sequence[torch.Tensor]],
                   reverse: bool = False):
    """The same segment moves for W ranks held by one process (send[s], recv[d]
    are rank s's and rank d's buffer lists): device copies instead of messages.
    For tests and single-GPU emulation of W ranks."""
    W = plan.W
    for s in range(W):
        for d in range(W):
            for (a, b, n) in segments(plan, s, d):
                if reverse:  # owner d's rows back into source s's send layout
                    for x_t, y_t in zip(send[d], recv[s]):
                        y_t[a:a + n].copy_(x_t[b:b + n])
                else:
                    for x_t, y_t in zip(send[s], recv[d]):
                        y_t[b:b + n].copy_(x_t[a:a + n])


def global_slots(plan: EpPlan, rank: int, slot_of_local: np.ndarray) -> np.ndarray:
    """Where rank `rank`'s pairs sit in the whole-batch layout: for a pair of
    expert e with local slot l, base(d) + recv_offsets[d][rank][j] + (l - send_offsets[rank][e])
    (d, j the owner and local index of e); -1 stays -1."""
    sl = np.asarray(slot_of_local, np.int64)
    out = np.full(sl.shape, -1, np.int64)
    so = plan.send_offsets[rank]
    valid = sl >= 0
    e = np.searchsorted(so, sl[valid], side="right") - 1  # expert of each local slot
    d, j = e // plan.Eloc, e % plan.Eloc
    base = plan.expert_offsets[d * plan.Eloc]
    out[valid] = base + plan.recv_offsets[d, rank, j] + (sl[valid] - so[e])
    return out.astype(np.int32)


class EpRank:
    """One rank of an expert-parallel MoE routing pass (one process per GPU).

    S tokens on this rank, hidden H, K experts per token, E experts over W
    ranks (E % W == 0), token_padding P for the receive buffers, activations
    bf16 or fp32, optional FP8 dispatch.  `dispatch` returns this rank's expert
    inputs (expert-major, padded) and keeps what `combine` needs."""

    def __init__(self, S: int, H: int, K: int, E: int, W: int, rank: int, token_padding: int = 0,
                 dtype: torch.dtype = torch.bfloat16, fp8: bool = False, device="cuda", group=None):
        if E % W:
            raise ValueError("E must be a multiple of the number of ranks")
        self.S, self.H, self.K, self.E, self.W, self.rank, self.P = S, H, K, E, W, rank, token_padding
        self.dtype, self.fp8, self.device, self.group = dtype, fp8, torch.device(device), group
        self.quant = B.MOE_QUANT_FP8_E4M3_B128 if fp8 else B.MOE_QUANT_NONE
        i32 = dict(dtype=torch.int32, device=self.device)
        self.cap = S * K  # the send layout has no padding
        self.layout = B.Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(W + 1, **i32),
                               torch.empty((S, K), **i32), torch.empty(self.cap, **i32), self.cap)
        self.workspace = torch.zeros(max(B.moe_dispatch_layout_workspace(S, E, K), 256), dtype=torch.uint8,
                                     device=self.device)
        self.status = torch.zeros(1, **i32)
        if fp8:
            self.send = [torch.empty((self.cap, H), dtype=torch.uint8, device=self.device),
                         torch.empty((self.cap, H // 128), dtype=torch.float32, device=self.device)]
        else:
            self.send = [torch.empty((self.cap, H), dtype=dtype, device=self.device)]
        self.plan: Optional[EpPlan] = None
        self.topk_idx = self.topk_w = None

    def local_dispatch(self, logits: torch.Tensor, x: torch.Tensor):
        """Route this rank's tokens, build the send layout and fill the send buffers (GPU)."""
        self.topk_idx, self.topk_w = B.moe_route_topk(logits, self.K)
        B.moe_dispatch_layout(self.topk_idx, self.E, self.W, 0, self.cap, workspace=self.workspace,
                              status=self.status, out=self.layout)
        xd = self.send[0].view(torch.float8_e4m3fn) if self.fp8 else self.send[0]
        B.moe_dispatch(x, self.layout.slot_of, self.cap, self.quant, xd, self.send[1] if self.fp8 else None,
                       status=self.status)

    def make_plan(self, counts_all: np.ndarray) -> EpPlan:
        self.plan = ep_plan(counts_all, self.P)
        return self.plan

    def new_recv(self, rows: int) -> List[torch.Tensor]:
        if self.fp8:
            return [torch.empty((rows, self.H), dtype=torch.uint8, device=self.device),
                    torch.empty((rows, self.H // 128), dtype=torch.float32, device=self.device)]
        return [torch.empty((rows, self.H), dtype=self.dtype, device=self.device)]

    def dispatch(self, logits: torch.Tensor, x: torch.Tensor) -> Tuple[List[torch.Tensor], np.ndarray]:
        """Whole dispatch over the process group: returns (receive buffers, this
        rank's expert offsets within them [E/W + 1])."""
        import torch.distributed as dist

        self.local_dispatch(logits, x)
        gathered = [torch.empty(self.E, dtype=torch.int32, device=self.device) for _ in range(self.W)]
        dist.all_gather(gathered, self.layout.counts, group=self.group)
        counts_all = torch.stack(gathered).cpu().numpy()  # synchronises: the segment sizes go to the host
        plan = self.make_plan(counts_all)
        recv = self.new_recv(int(plan.recv_rows[self.rank]))
        exchange(plan, self.rank, self.send, recv, self.group)
        lo = self.rank * plan.Eloc
        offs = plan.expert_offsets[lo:lo + plan.Eloc + 1] - plan.expert_offsets[lo]
        return recv, offs

    def combine(self, y_recv: torch.Tensor, shared_out=None, residual=None):
        """Expert outputs of this rank's receive buffer back to their source
        ranks, then the weighted sum (and the dual residual) of this rank's
        tokens with the local layout."""
        y_send = torch.empty((self.cap, self.H), dtype=y_recv.dtype, device=self.device)
        exchange(self.plan, self.rank, [y_recv], [y_send], self.group, reverse=True)
        return self.local_combine(y_send, shared_out, residual)

    def local_combine(self, y_send: torch.Tensor, shared_out=None, residual=None):
        return B.moe_combine_dual_residual(y_send, self.layout.slot_of, self.topk_w, shared_out, residual,
                                           status=self.status)
