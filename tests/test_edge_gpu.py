"""GPU parity on ragged shapes and on the degenerate cases of each step.

Ragged shapes cross every tiling boundary of the kernels: token counts that
are not multiples of the warps per CTA, pair counts that leave a partial
layout tile, hidden sizes that leave a partial warp iteration (bf16, fp32 and
FP8), K above the 8-row gather chunk, E up to 1024 and K up to 32, and odd
paddings.  Degenerate cases: S = 0, K = E, ties, expert ids out of range, a
capacity that is too small, slots outside [0, cap), all-zero FP8 blocks and
signed zeros, in-place residual, workspace reuse.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import synth

from .helpers import assert_act_close, assert_f32_close

pytestmark = pytest.mark.gpu


def dev(a):
    return synth.to_torch(a, device="cuda")


def host(t):
    return synth.from_torch(t)


def _wl(S, H, E, K, R, P, dtype, quant, fused, seed):
    return synth.Workload(f"ragged_{S}_{H}_{E}_{K}", S, H, E, K, R, P, dtype, quant, fused, seed=seed)


RAGGED = [
    _wl(1, 8, 1, 1, 1, 0, "bf16", "none", True, 11),
    _wl(37, 136, 40, 3, 4, 5, "bf16", "none", True, 12),
    _wl(2049, 384, 96, 6, 3, 128, "bf16", "fp8", True, 13),
    _wl(300, 260, 17, 17, 17, 1, "f32", "none", True, 14),
    _wl(513, 1024, 1024, 32, 8, 16, "bf16", "fp8", False, 15),
    _wl(64, 512, 64, 8, 8, 0, "f32", "fp8", True, 16),
    _wl(5000, 64, 8, 2, 2, 0, "f32", "none", False, 17),
    _wl(77, 128, 32, 32, 4, 3, "bf16", "fp8", True, 18),
    _wl(4099, 264, 384, 8, 4, 128, "bf16", "none", False, 19),
    _wl(700, 1032, 64, 8, 8, 0, "bf16", "none", True, 22),    # 2064-byte rows: just past 2 KB (6 combine warps)
    _wl(333, 2048, 64, 6, 4, 16, "f32", "fp8", True, 23),     # 8 KB fp32 rows: three 3 KB chunks, FP8 dispatch
    _wl(257, 4104, 32, 4, 4, 0, "bf16", "none", False, 24),   # 8208-byte rows: 8 warps, a 16-byte last chunk
]


@pytest.mark.parametrize("w", RAGGED, ids=lambda w: w.name)
def test_ragged_pass(w):
    lg, x = synth.logits(w), synth.activations(w)
    y = synth.expert_outputs(w)
    sh = synth.shared_out(w) if w.fused else None
    rs = synth.residual(w) if w.fused else None
    idx, wt = oracle.route_topk(lg, w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    q = oracle.QUANT_FP8_E4M3_B128 if w.quant == "fp8" else oracle.QUANT_NONE
    xd, xs = oracle.dispatch(x, lay["slot_of"], lay["cap"], quant=q)
    out, rnr = oracle.combine(y, lay["slot_of"], wt, sh, rs)

    gidx, gw = B.moe_route_topk(dev(lg), w.K)
    np.testing.assert_array_equal(host(gidx), idx)
    assert_f32_close(host(gw), wt, 1e-5, "topk_w")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    glay = B.moe_dispatch_layout(dev(idx), w.E, w.R, w.P, status=status)
    for k in ("counts", "offsets", "rank_offsets", "slot_of", "row_src"):
        np.testing.assert_array_equal(host(getattr(glay, k)), lay[k], err_msg=k)
    valid = lay["row_src"] >= 0
    gxd, gxs = B.moe_dispatch(dev(x), dev(lay["slot_of"]), lay["cap"], q, status=status)
    np.testing.assert_array_equal(host(gxd)[valid], xd[valid])
    if q:
        np.testing.assert_array_equal(host(gxs)[valid], xs[valid])
    gout, grnr = B.moe_combine_dual_residual(dev(y), dev(lay["slot_of"]), dev(wt),
                                             dev(sh) if w.fused else None,
                                             dev(rs) if w.fused else None)
    assert_act_close(host(gout), out, "residual_out")
    if w.fused:
        assert_act_close(host(grnr), rnr, "residual_no_routed_out")
    assert status.item() == 0


def test_empty_batch():
    E, K, R, P, H = 16, 4, 4, 8, 256
    lg = torch.empty((0, E), dtype=torch.float32, device="cuda")
    idx, w = B.moe_route_topk(lg, K)
    assert idx.shape == (0, K)
    cap = 40  # rows exist, but no token maps to them
    lay = B.moe_dispatch_layout(idx, E, R, P, cap)
    assert host(lay.counts).tolist() == [0] * E
    assert host(lay.offsets).tolist() == [0] * (E + 1)
    assert host(lay.rank_offsets).tolist() == [0] * (R + 1)
    assert np.all(host(lay.row_src) == -1)
    x = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    xd, xs = B.moe_dispatch(x, lay.slot_of, cap, B.MOE_QUANT_FP8_E4M3_B128)
    y = torch.zeros((cap, H), dtype=torch.bfloat16, device="cuda")
    out, rnr = B.moe_combine_dual_residual(y, lay.slot_of, w, x, x)
    torch.cuda.synchronize()
    assert out.shape == (0, H) and rnr.shape == (0, H)


def test_route_ties_and_full_sort():
    rng = np.random.default_rng(5)
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 2.0], np.float32)
    for E, K in ((12, 3), (32, 32), (100, 8), (1024, 32)):
        lg = vals[rng.integers(0, len(vals), size=(333, E))]
        idx, wt = oracle.route_topk(lg, K)
        gidx, gw = B.moe_route_topk(dev(lg), K)
        np.testing.assert_array_equal(host(gidx), idx)
        assert_f32_close(host(gw), wt, 1e-5, "topk_w")


def test_bad_expert_ids_are_dropped_and_flagged():
    S, E, K, R = 300, 16, 4, 4
    rng = np.random.default_rng(1)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(S)]).astype(np.int32)
    idx[3, 1] = -1
    idx[100, 0] = E
    idx[299, 3] = 1 << 30
    good = (idx >= 0) & (idx < E)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lay = B.moe_dispatch_layout(dev(idx), E, R, 0, status=status)
    assert status.item() & B.MOE_STATUS_BAD_INDEX
    slot = host(lay.slot_of)
    assert np.all(slot[~good] == -1)
    counts = host(lay.counts)
    np.testing.assert_array_equal(counts, np.bincount(idx[good], minlength=E))
    # valid pairs: a stable counting sort of the valid ones, in ascending pair order
    offs = host(lay.offsets)
    flat, sl = idx.reshape(-1), slot.reshape(-1)
    for e in range(E):
        members = np.nonzero(flat == e)[0]
        np.testing.assert_array_equal(sl[members], offs[e] + np.arange(len(members)))
    rs = host(lay.row_src)
    assert np.count_nonzero(rs >= 0) == good.sum()


def test_capacity_overflow_is_flagged_not_written():
    S, E, K, R, P = 200, 8, 2, 2, 64
    rng = np.random.default_rng(2)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(S)]).astype(np.int32)
    full = oracle.layout(idx, E, R, P)
    cap = int(full["offsets"][E]) - 100
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    row_src = torch.full((cap + 8,), 12345, dtype=torch.int32, device="cuda")  # 8 guard entries
    out = B.Layout(torch.empty(E, dtype=torch.int32, device="cuda"),
                   torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                   torch.empty(R + 1, dtype=torch.int32, device="cuda"),
                   torch.empty((S, K), dtype=torch.int32, device="cuda"), row_src[:cap], cap)
    lay = B.moe_dispatch_layout(dev(idx), E, R, P, cap, status=status, out=out)
    assert status.item() & B.MOE_STATUS_OVERFLOW
    np.testing.assert_array_equal(host(lay.counts), full["counts"])
    np.testing.assert_array_equal(host(lay.offsets), full["offsets"])
    s_ref = full["slot_of"]
    s_got = host(lay.slot_of)
    np.testing.assert_array_equal(s_got[s_ref < cap], s_ref[s_ref < cap])
    assert np.all(s_got[s_ref >= cap] == -1)
    np.testing.assert_array_equal(host(row_src)[:cap], full["row_src"][:cap])
    assert np.all(host(row_src)[cap:] == 12345)  # nothing written past cap


def test_out_of_range_slots_skipped_in_dispatch_and_combine():
    S, H, K, cap = 64, 256, 2, 128
    rng = np.random.default_rng(3)
    slot = rng.permutation(cap)[:S * K].reshape(S, K).astype(np.int32)
    slot[5, 1] = cap + 3
    slot[9, 0] = -1
    x = synth.f32_to_bf16_bits(rng.standard_normal((S, H)).astype(np.float32))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xd = torch.zeros((cap, H), dtype=torch.bfloat16, device="cuda")
    B.moe_dispatch(dev(x), dev(slot), cap, B.MOE_QUANT_NONE, xd, status=status)
    assert status.item() == B.MOE_STATUS_BAD_SLOT
    ok = (slot >= 0) & (slot < cap)
    ref_xd, _ = oracle.dispatch(x, np.where(ok, slot, -1), cap)
    np.testing.assert_array_equal(host(xd), ref_xd)
    w = rng.uniform(0.1, 1, (S, K)).astype(np.float32)
    status.zero_()
    out, _ = B.moe_combine_dual_residual(xd, dev(slot), dev(w), status=status)
    assert status.item() == B.MOE_STATUS_BAD_SLOT
    ref_out, _ = oracle.combine(ref_xd, np.where(ok, slot, -1), w)
    assert_act_close(host(out), ref_out, "out")


def test_fp8_zero_blocks_and_signed_zeros():
    S, H, K = 9, 512, 2
    rng = np.random.default_rng(4)
    x = rng.standard_normal((S, H)).astype(np.float32)
    x[0, :128] = 0.0
    x[1, 128:256] = -0.0
    x[2, 256:384] = np.where(rng.random(128) < 0.5, 0.0, -0.0)
    x[3, 5] = -0.0
    x[4, :] *= 1e-38   # tiny blocks: subnormal-range scales
    x[5, 384:] = 448.0 * 3
    x[6, :128] = np.float32(2.0 ** -133) * rng.integers(-3, 4, 128)  # bf16 subnormals
    xb = synth.f32_to_bf16_bits(x)
    slot = np.arange(S * K, dtype=np.int32).reshape(S, K)
    cap = S * K
    for xin in (xb, x):
        ref_xd, ref_xs = oracle.dispatch(xin, slot, cap, quant=oracle.QUANT_FP8_E4M3_B128)
        gxd, gxs = B.moe_dispatch(dev(xin), dev(slot), cap, B.MOE_QUANT_FP8_E4M3_B128)
        np.testing.assert_array_equal(host(gxd), ref_xd)
        np.testing.assert_array_equal(host(gxs), ref_xs)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_in_place_residual_and_partial_epilogues(dtype):
    w = _wl(333, 264, 24, 4, 4, 0, dtype, "none", True, 21)
    y, sh, rs = synth.expert_outputs(w), synth.shared_out(w), synth.residual(w)
    idx, wt = oracle.route_topk(synth.logits(w), w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    out, rnr = oracle.combine(y, lay["slot_of"], wt, sh, rs)
    r_dev = dev(rs)
    gout, grnr = B.moe_combine_dual_residual(dev(y), dev(lay["slot_of"]), dev(wt), dev(sh), r_dev,
                                             residual_out=r_dev)
    assert gout.data_ptr() == r_dev.data_ptr()
    assert_act_close(host(gout), out, "in-place residual_out")
    assert_act_close(host(grnr), rnr, "residual_no_routed_out")
    for kw in (dict(shared=sh), dict(residual=rs)):
        o_ref, _ = oracle.combine(y, lay["slot_of"], wt, **kw)
        g, gn = B.moe_combine_dual_residual(dev(y), dev(lay["slot_of"]), dev(wt),
                                            shared_out=dev(kw["shared"]) if "shared" in kw else None,
                                            residual=dev(kw["residual"]) if "residual" in kw else None)
        assert gn is None
        assert_act_close(host(g), o_ref, f"partial epilogue {list(kw)}")


def test_workspace_reused_across_calls_and_shapes():
    ws = torch.zeros(B.moe_dispatch_layout_workspace(9000, 256, 8), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(6)
    for S, E, K, R, P in ((9000, 256, 8, 8, 0), (100, 64, 4, 8, 128), (9000, 256, 8, 8, 0),
                          (4096, 128, 8, 4, 32)):
        idx = np.stack([rng.permutation(E)[:K] for _ in range(S)]).astype(np.int32)
        ref = oracle.layout(idx, E, R, P)
        for _ in range(3):
            lay = B.moe_dispatch_layout(dev(idx), E, R, P, workspace=ws)
            np.testing.assert_array_equal(host(lay.slot_of), ref["slot_of"])
            np.testing.assert_array_equal(host(lay.row_src), ref["row_src"])
            np.testing.assert_array_equal(host(lay.offsets), ref["offsets"])
        assert int(ws[:8].sum().item()) == 0  # arrival ticket and barrier count back at zero


def test_invalid_args_raise_before_launch():
    x = torch.zeros((8, 100), dtype=torch.bfloat16, device="cuda")  # 200-byte rows
    slot = torch.zeros((8, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError):
        B.moe_dispatch(x, slot, 16)
    lg = torch.zeros((8, 4), dtype=torch.float32, device="cuda")
    with pytest.raises(B.MoeError):
        B.moe_route_topk(lg, 5)


def _midpoint_blocks(rng, S, H, in_bf16: bool):
    """Rows whose quotients x/s sit within a few fp32 ulps of e4m3 rounding midpoints."""
    codes = np.arange(0, 0x7E, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.empty((S, H), np.float32)
    for t in range(S):
        for b in range(H // 128):
            a = np.float32(rng.uniform(0.5, 4.0) * 2.0 ** int(rng.integers(-20, 21)))
            if in_bf16:
                a = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.array([a], np.float32)))[0]
            s = np.float32(a) / np.float32(448.0)
            m = rng.choice(mids, 127) * rng.choice([-1.0, 1.0], 127)
            v = (m * np.float64(s)).astype(np.float32)
            v = (v.view(np.int32) + rng.integers(-2, 3, 127).astype(np.int32)).view(np.float32)
            blk = np.concatenate([[a], v]).astype(np.float32)
            rng.shuffle(blk)
            x[t, 128 * b:128 * (b + 1)] = blk
    return synth.f32_to_bf16_bits(x) if in_bf16 else x


@pytest.mark.parametrize("S,H,K", [
    # few items: per-thread stores
    (300, 640, 8), (300, 1664, 3), (300, 4224, 8), (300, 7296, 8), (300, 7168, 5), (300, 512, 32),
    # enough items per SM for the bulk-store path
    (2400, 640, 8), (2400, 1664, 3), (1300, 7296, 8), (1200, 7168, 5), (2400, 512, 32),
])
def test_fp8_dispatch_row_shapes(S, H, K):
    """Rows whose block count is or is not a multiple of 4 (scale segments sent as one
    bulk store per copy, or stored per block), one or two items per row, small and large K,
    on both store paths; slots scattered over a larger capacity with unused rows left untouched."""
    rng = np.random.default_rng(H + K + S)
    cap = S * K + 77
    x = synth.f32_to_bf16_bits((rng.standard_normal((S, H)) * rng.uniform(0.01, 50, (S, 1))).astype(np.float32))
    slot = rng.permutation(cap)[:S * K].astype(np.int32).reshape(S, K)
    ref_xd, ref_xs = oracle.dispatch(x, slot, cap, quant=oracle.QUANT_FP8_E4M3_B128)
    xd = torch.full((cap, H), 0x5A, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
    xs = torch.full((cap, H // 128), -7.0, dtype=torch.float32, device="cuda")
    B.moe_dispatch(dev(x), dev(slot), cap, B.MOE_QUANT_FP8_E4M3_B128, xd=xd, xs=xs)
    used = np.zeros(cap, bool)
    used[slot.reshape(-1)] = True
    np.testing.assert_array_equal(host(xd)[used], ref_xd[used])
    np.testing.assert_array_equal(host(xs)[used], ref_xs[used])
    assert np.all(host(xd.view(torch.uint8))[~used] == 0x5A) and np.all(host(xs)[~used] == -7.0)


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_runs_out_and_reports(which):
    """A wait that nothing completes (an mbarrier phase with no arrival, or a flag nobody
    writes) gives up after its limit, reports MOE_STATUS_TIMEOUT, and the context stays
    usable: a routing pass right after it matches the oracle."""
    import time

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    B.moe_selftest_wait_timeout(which, 2_000_000, status, flag)  # 2 ms
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert status.item() == B.MOE_STATUS_TIMEOUT
    w = synth.WORKLOADS["1"]
    logits = synth.logits(w)
    idx, _ = B.moe_route_topk(dev(logits), w.K)
    lay = B.moe_dispatch_layout(idx, w.E, w.R, w.P)
    ref_idx, _ = oracle.route_topk(logits, w.K)
    np.testing.assert_array_equal(host(idx), ref_idx)
    np.testing.assert_array_equal(host(lay.slot_of), oracle.layout(ref_idx, w.E, w.R, w.P)["slot_of"])
    with pytest.raises(B.MoeError):
        B.moe_selftest_wait_timeout(2, 1000, status)


@pytest.mark.parametrize("S", [64, 2400])
def test_fp8_dispatch_scale_rows_not_16_byte_aligned(S):
    """A scale array whose base is only 4-byte aligned: scales are stored per block
    (on both store paths)."""
    rng = np.random.default_rng(5)
    H, K = 2048, 4
    cap = S * K
    x = synth.f32_to_bf16_bits(rng.standard_normal((S, H)).astype(np.float32))
    slot = rng.permutation(cap).astype(np.int32).reshape(S, K)
    ref_xd, ref_xs = oracle.dispatch(x, slot, cap, quant=oracle.QUANT_FP8_E4M3_B128)
    big = torch.zeros(cap * (H // 128) + 1, dtype=torch.float32, device="cuda")
    xs = big[1:].view(cap, H // 128)  # base + 4 bytes
    xd = torch.empty((cap, H), dtype=torch.float8_e4m3fn, device="cuda")
    B.moe_dispatch(dev(x), dev(slot), cap, B.MOE_QUANT_FP8_E4M3_B128, xd=xd, xs=xs)
    np.testing.assert_array_equal(host(xd), ref_xd)
    np.testing.assert_array_equal(host(xs), ref_xs)


@pytest.mark.parametrize("in_bf16", [False, True])
def test_fp8_quotients_near_rounding_midpoints(in_bf16):
    rng = np.random.default_rng(8 + in_bf16)
    S, H, K = 96, 1024, 3
    x = _midpoint_blocks(rng, S, H, in_bf16)
    slot = np.arange(S * K, dtype=np.int32).reshape(S, K)
    ref_xd, ref_xs = oracle.dispatch(x, slot, S * K, quant=oracle.QUANT_FP8_E4M3_B128)
    gxd, gxs = B.moe_dispatch(dev(x), dev(slot), S * K, B.MOE_QUANT_FP8_E4M3_B128)
    np.testing.assert_array_equal(host(gxs), ref_xs)
    np.testing.assert_array_equal(host(gxd), ref_xd)


@pytest.mark.parametrize("S,E,K,R,P", [
    (8192, 1024, 32, 8, 16),   # T*E above the fused layout's scan bound: the two-kernel layout
    (150000, 64, 8, 8, 128),   # more tiles than co-resident CTAs: several tiles per CTA (fused)
    (20000, 512, 8, 4, 0),     # mid-size fused
    (1024, 512, 32, 8, 16),    # cluster layout: 16 CTAs of 2048 pairs, the largest E it takes
    (1024, 1024, 32, 8, 16),   # the same pairs with E = 1024: cooperative single launch
    (4095, 256, 8, 8, 0),      # cluster layout, ragged last tile
    (1000, 300, 8, 3, 0),      # cluster of 4 CTAs, E not a multiple of 32
    (4097, 256, 8, 8, 128),    # one tile past the cluster layout's bound: fused
    (3, 7, 2, 1, 5),           # cluster of one CTA, E not a multiple of 32
])
def test_layout_paths_large(S, E, K, R, P):
    rng = np.random.default_rng(S + E)
    # distinct experts per token, skewed
    p = rng.dirichlet(np.full(E, 0.5))
    idx = np.argsort(rng.random((S, E)) / p[None, :], axis=1)[:, :K].astype(np.int32)
    ref = oracle.layout(idx, E, R, P)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        lay = B.moe_dispatch_layout(dev(idx), E, R, P, status=status)
        for k in ("counts", "offsets", "rank_offsets", "slot_of", "row_src"):
            np.testing.assert_array_equal(host(getattr(lay, k)), ref[k], err_msg=k)
    assert status.item() == 0


@pytest.mark.parametrize("S,E,K,n", [
    (4096, 256, 8, 1),       # cluster layout
    (1, 7, 2, 1),
    (1024, 1024, 32, 1),     # E above the cluster layout's bound: cooperative
    (150000, 64, 8, 1),      # cooperative single launch
    (8192, 1024, 32, 2),     # histogram + slots
])
def test_layout_kernel_count(S, E, K, n):
    assert B.moe_dispatch_layout_kernels(S, E, K) == n


def test_kernels_accept_any_size_order():
    """Launch shapes whose shared-memory needs go up, down and up again."""
    rng = np.random.default_rng(9)
    for H in (1024, 128, 7168, 512, 1024, 7168):
        S, K = 40, 3
        x = synth.f32_to_bf16_bits(rng.standard_normal((S, H)).astype(np.float32))
        slot = np.arange(S * K, dtype=np.int32).reshape(S, K)
        ref_xd, ref_xs = oracle.dispatch(x, slot, S * K, quant=oracle.QUANT_FP8_E4M3_B128)
        gxd, gxs = B.moe_dispatch(dev(x), dev(slot), S * K, B.MOE_QUANT_FP8_E4M3_B128)
        np.testing.assert_array_equal(host(gxd), ref_xd)
        np.testing.assert_array_equal(host(gxs), ref_xs)
    for K, H in ((8, 2048), (32, 7168), (2, 256), (8, 7168), (17, 1024), (8, 2048)):
        S = 24
        y = synth.f32_to_bf16_bits(rng.standard_normal((S * K, H)).astype(np.float32))
        slot = rng.permutation(S * K).astype(np.int32).reshape(S, K)
        w = rng.uniform(0.1, 1.0, (S, K)).astype(np.float32)
        ref, _ = oracle.combine(y, slot, w)
        got, _ = B.moe_combine_dual_residual(dev(y), dev(slot), dev(w))
        assert_act_close(host(got), ref, f"combine K={K} H={H}")
