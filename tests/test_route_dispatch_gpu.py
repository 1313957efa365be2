"""GPU parity of moe_route_dispatch, the one-call route + layout + dispatch.

Every output is compared with the CPU oracle (top-K ids, layout, dispatched
bytes and FP8 scales bit-exact; gating weights within 1e-5 relative) and,
bit for bit, with the three separate entry points on the same inputs.  The
cases cover the workloads that run as one fused kernel, the ragged and
maximum shares per CTA, the fallback to separate kernels, scale rows that are
not whole 16-byte units, two quantisation passes, fp32 input, K = E, padding,
a capacity smaller than the layout, heavy ties, graph replay and a workspace
shared with moe_dispatch_layout.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import synth

from .helpers import assert_f32_close

pytestmark = pytest.mark.gpu


def dev(a):
    return synth.to_torch(a, device="cuda")


def host(t):
    return synth.from_torch(t)


def _wl(S, H, E, K, R, P, dtype="bf16", quant="fp8", seed=11, bias="none"):
    return synth.Workload(f"case_{S}_{H}_{E}_{K}", S, H, E, K, R, P, dtype, quant, False, bias=bias, seed=seed)


def _qcode(w):
    return B.MOE_QUANT_FP8_E4M3_B128 if w.quant == "fp8" else B.MOE_QUANT_NONE


def _sentinels(w, cap):
    if w.quant == "fp8":
        return (torch.full((cap, w.H), 0x5A, dtype=torch.uint8, device="cuda"),
                torch.full((cap, w.H // 128), -7.0, dtype=torch.float32, device="cuda"))
    t = torch.float32 if w.dtype == "f32" else torch.bfloat16
    return torch.full((cap, w.H), -7.0, dtype=t, device="cuda"), None


def _fused(w, logits, x, cap=None, status=None):
    cap = B.moe_capacity(w.S, w.E, w.K, w.P) if cap is None else cap
    xd, xs = _sentinels(w, cap)
    idx, wt, lay, xd, xs = B.moe_route_dispatch(logits, x, w.K, w.R, w.P, _qcode(w), cap, xd=xd, xs=xs,
                                                status=status)
    return idx, wt, lay, xd, xs


def _separate(w, logits, x, cap=None, status=None):
    cap = B.moe_capacity(w.S, w.E, w.K, w.P) if cap is None else cap
    idx, wt = B.moe_route_topk(logits, w.K)
    lay = B.moe_dispatch_layout(idx, w.E, w.R, w.P, cap, status=status)
    xd, xs = _sentinels(w, cap)
    B.moe_dispatch(x, lay.slot_of, cap, _qcode(w), xd, xs, status=status)
    return idx, wt, lay, xd, xs


LAYOUT_KEYS = ("counts", "offsets", "rank_offsets", "slot_of", "row_src")


def _assert_same_gpu(a, b):
    for i, name in enumerate(("topk_idx", "topk_w")):
        assert torch.equal(a[i], b[i]), name
    for k in LAYOUT_KEYS:
        assert torch.equal(getattr(a[2], k), getattr(b[2], k)), k
    assert torch.equal(a[3].view(torch.uint8), b[3].view(torch.uint8)), "xd"
    if a[4] is not None:
        assert torch.equal(a[4], b[4]), "xs"


def _assert_oracle(w, logits_h, x_h, got, cap=None):
    idx, wt = oracle.route_topk(logits_h, w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P, cap)
    q = oracle.QUANT_FP8_E4M3_B128 if w.quant == "fp8" else oracle.QUANT_NONE
    xd, xs = oracle.dispatch(x_h, lay["slot_of"], lay["cap"], quant=q)
    np.testing.assert_array_equal(host(got[0]), idx)
    assert_f32_close(host(got[1]), wt, 1e-5, "topk_w")
    for k in LAYOUT_KEYS:
        np.testing.assert_array_equal(host(getattr(got[2], k)), lay[k], err_msg=k)
    valid = lay["row_src"] >= 0
    gxd = host(got[3])
    np.testing.assert_array_equal(gxd[valid], xd[valid])
    if w.quant == "fp8":
        gxs = host(got[4])
        np.testing.assert_array_equal(gxs[valid], xs[valid])
        assert np.all(gxd[~valid] == 0x5A) and np.all(gxs[~valid] == -7.0)  # padding rows untouched


def _run_case(w, expect_fused=None, cap=None):
    lg, x = synth.logits(w), synth.activations(w)
    dl, dx = dev(lg), dev(x)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    n = B.moe_route_dispatch_kernels(w.S, w.H, w.E, w.K, dt, _qcode(w))
    if expect_fused is not None:
        assert (n == 1) == expect_fused, n
    st1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _fused(w, dl, dx, cap, st1)
    ref = _separate(w, dl, dx, cap, st2)
    torch.cuda.synchronize()
    _assert_same_gpu(got, ref)
    assert st1.item() == st2.item()
    _assert_oracle(w, lg, x, got, cap)
    return st1.item()


@pytest.mark.parametrize("key", ["1", "2", "2b", "3"])
def test_workloads_run_fused_and_match(key):
    w = synth.WORKLOADS[key]
    w = w.replace(fused=False)
    assert _run_case(w, expect_fused=True) == 0


@pytest.mark.parametrize("key", ["4", "5"])
def test_workloads_on_separate_kernels_match(key):
    # 4: 28 FP8 tokens per SM are quantised faster by the separate dispatch kernel;
    # 5: 16384 tokens of 2048 bf16 channels do not fit in shared memory per SM
    assert _run_case(synth.WORKLOADS[key].replace(fused=False), expect_fused=False) == 0


EDGE = [
    # S, H, E, K, R, P, dtype, quant, expect_fused
    (1, 7168, 256, 8, 8, 0, "bf16", "fp8", True),        # one token, one CTA
    (149, 7168, 256, 8, 8, 0, "bf16", "fp8", True),      # one CTA with two tokens
    (300, 7168, 256, 8, 8, 0, "bf16", "fp8", True),      # three tokens per CTA (two quantiser groups)
    (592, 7168, 256, 8, 8, 0, "bf16", "fp8", True),      # 4 FP8 tokens per CTA: the most the fused kernel takes
    (593, 7168, 256, 8, 8, 0, "bf16", "fp8", False),     # one token more: separate kernels
    (2220, 7168, 256, 8, 8, 0, "bf16", "none", True),    # 15 bf16 rows of 14 KB per CTA fit in shared memory
    (2400, 7168, 256, 8, 8, 0, "bf16", "none", False),   # 17 do not
    (300, 512, 33, 3, 3, 16, "bf16", "fp8", True),       # E not a multiple of 4, padding
    (200, 384, 64, 6, 4, 0, "bf16", "fp8", True),        # 3 scale blocks: scales stored per element
    (100, 16384, 64, 4, 2, 0, "bf16", "fp8", False),     # rows too long for the fused quantiser: separate kernels
    (150, 8192, 64, 4, 2, 0, "bf16", "fp8", True),       # the longest FP8 row the fused quantiser takes
    (500, 7168, 256, 8, 8, 0, "f32", "fp8", True),       # fp32 input: a raw row covers 4 slots
    (500, 1024, 512, 32, 8, 128, "bf16", "none", True),  # E = 512, K = 32, bf16 copy
    (256, 256, 8, 8, 1, 0, "f32", "none", True),         # K = E, fp32 copy
    (3000, 2048, 128, 8, 4, 64, "bf16", "none", True),   # copy rows resident, padding
]


@pytest.mark.parametrize("S,H,E,K,R,P,dt,q,fused", EDGE)
def test_edge_shapes(S, H, E, K, R, P, dt, q, fused):
    w = _wl(S, H, E, K, R, P, dt, q, seed=S + H + E)
    assert _run_case(w, expect_fused=fused) == 0


def test_capacity_smaller_than_the_layout():
    """Pairs whose slot would be >= cap get slot -1 and are not dispatched; the
    overflow is flagged; everything else is the full layout's."""
    w = _wl(512, 512, 64, 4, 4, 0, "bf16", "fp8", seed=5)
    lg, x = synth.logits(w), synth.activations(w)
    dl, dx = dev(lg), dev(x)
    cap = w.S * w.K - 100
    st1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _fused(w, dl, dx, cap, st1)
    ref = _separate(w, dl, dx, cap, st2)
    torch.cuda.synchronize()
    _assert_same_gpu(got, ref)
    assert st1.item() & B.MOE_STATUS_OVERFLOW and st1.item() == st2.item()
    idx, _ = oracle.route_topk(lg, w.K)
    full = oracle.layout(idx, w.E, w.R, w.P)
    np.testing.assert_array_equal(host(got[2].counts), full["counts"])
    np.testing.assert_array_equal(host(got[2].offsets), full["offsets"])
    s_ref, s_got = full["slot_of"], host(got[2].slot_of)
    np.testing.assert_array_equal(s_got[s_ref < cap], s_ref[s_ref < cap])
    assert np.all(s_got[s_ref >= cap] == -1)
    np.testing.assert_array_equal(host(got[2].row_src), full["row_src"][:cap])
    xd, xs = oracle.dispatch(x, np.where(s_ref < cap, s_ref, -1), cap, quant=oracle.QUANT_FP8_E4M3_B128)
    valid = full["row_src"][:cap] >= 0
    np.testing.assert_array_equal(host(got[3])[valid], xd[valid])
    np.testing.assert_array_equal(host(got[4])[valid], xs[valid])


def test_heavy_ties_follow_the_lower_expert_id():
    w = _wl(500, 512, 64, 8, 8, 0, "bf16", "fp8", seed=9)
    rng = np.random.default_rng(9)
    lg = rng.integers(-2, 3, size=(w.S, w.E)).astype(np.float32)  # few distinct values
    lg[::7, :] = 0.0
    lg[1::7, ::3] = -0.0
    x = synth.activations(w)
    dl, dx = dev(lg), dev(x)
    got = _fused(w, dl, dx)
    ref = _separate(w, dl, dx)
    torch.cuda.synchronize()
    _assert_same_gpu(got, ref)
    _assert_oracle(w, lg, x, got)


def test_repeated_calls_and_graph_replay_with_new_inputs():
    """The workspace header is left ready by every call: repeated calls, then a
    captured call replayed after its inputs were refilled with another draw."""
    w = synth.WORKLOADS["3"].replace(fused=False)
    w2 = w.replace(seed=w.seed + 77)
    lg1, x1 = synth.logits(w), synth.activations(w)
    lg2, x2 = synth.logits(w2), synth.activations(w2)
    dl, dx = dev(lg1), dev(x1)
    cap = B.moe_capacity(w.S, w.E, w.K, w.P)
    ws = torch.zeros(B.moe_route_dispatch_workspace(w.S, w.E, w.K), dtype=torch.uint8, device="cuda")
    idx = torch.empty((w.S, w.K), dtype=torch.int32, device="cuda")
    wt = torch.empty((w.S, w.K), dtype=torch.float32, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    lay = B.Layout(torch.empty(w.E, **i32), torch.empty(w.E + 1, **i32), torch.empty(w.R + 1, **i32),
                   torch.empty((w.S, w.K), **i32), torch.empty(cap, **i32), cap)
    xd, xs = _sentinels(w, cap)
    status = torch.zeros(1, **i32)

    def call():
        return B.moe_route_dispatch(dl, dx, w.K, w.R, w.P, B.MOE_QUANT_FP8_E4M3_B128, cap, topk_idx=idx,
                                    topk_w=wt, layout=lay, xd=xd, xs=xs, workspace=ws, status=status)

    for _ in range(3):
        got = call()
    torch.cuda.synchronize()
    _assert_oracle(w, lg1, x1, got)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    dl.copy_(dev(lg2))
    dx.copy_(dev(x2))
    xd.fill_(0x5A)
    xs.fill_(-7.0)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    _assert_oracle(w2, lg2, x2, (idx, wt, lay, xd, xs))
    assert status.item() == 0
    assert int(ws[:8].sum().item()) == 0  # grid-barrier count back at zero


def test_one_workspace_shared_with_the_layout_entry_point():
    """moe_route_dispatch (fused) and moe_dispatch_layout take turns on one
    workspace, eagerly and inside a replayed graph; every call gives the
    separate kernels' results and leaves the workspace ready."""
    w = _wl(300, 1024, 256, 8, 8, 0, "bf16", "fp8", seed=31)
    assert B.moe_route_dispatch_kernels(w.S, w.H, w.E, w.K, torch.bfloat16, _qcode(w)) == 1
    lg, x = synth.logits(w), synth.activations(w)
    dl, dx = dev(lg), dev(x)
    cap = B.moe_capacity(w.S, w.E, w.K, w.P)
    ref = _separate(w, dl, dx)
    need = max(B.moe_route_dispatch_workspace(w.S, w.E, w.K), B.moe_dispatch_layout_workspace(w.S, w.E, w.K))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    idx = torch.empty((w.S, w.K), **i32)
    wt = torch.empty((w.S, w.K), dtype=torch.float32, device="cuda")
    lay = B.Layout(torch.empty(w.E, **i32), torch.empty(w.E + 1, **i32), torch.empty(w.R + 1, **i32),
                   torch.empty((w.S, w.K), **i32), torch.empty(cap, **i32), cap)
    xd, xs = _sentinels(w, cap)

    def reset():
        idx.fill_(-3)
        wt.fill_(-3.0)
        for k in LAYOUT_KEYS:
            getattr(lay, k).fill_(-3)

    def rd():
        B.moe_route_dispatch(dl, dx, w.K, w.R, w.P, _qcode(w), cap, topk_idx=idx, topk_w=wt, layout=lay, xd=xd,
                             xs=xs, workspace=ws, status=status)

    def lay_only():
        B.moe_dispatch_layout(ref[0], w.E, w.R, w.P, cap, out=lay, workspace=ws, status=status)

    def check(full):
        torch.cuda.synchronize()
        if full:
            assert torch.equal(idx, ref[0]) and torch.equal(wt, ref[1])
            assert torch.equal(xd.view(torch.uint8), ref[3].view(torch.uint8)) and torch.equal(xs, ref[4])
        for k in LAYOUT_KEYS:
            assert torch.equal(getattr(lay, k), getattr(ref[2], k)), k

    for f, full in [(rd, True), (lay_only, False), (lay_only, False), (rd, True), (rd, True), (lay_only, False),
                    (rd, True)]:
        reset()
        f()
        check(full)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lay_only()
        rd()
    for _ in range(3):
        reset()
        g.replay()
        check(True)
    assert status.item() == 0
