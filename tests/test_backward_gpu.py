"""GPU parity of the backward entry points against the oracle.

Tolerances: grad_y, grad_skip and the dispatch backward use the same fp32
operations in the same order as the oracle (<= 1 bf16 ulp, or 1e-5 relative
for fp32).  grad_w is an fp32 sum of H products in a fixed order (a thread's
8 or 4 products, a 32-lane xor tree, the row's chunks, then the 4, 6 or 16
consumer warps in order): a leaf passes at most 8 + 5 + chunks + warps
roundings, 31 for the shapes here, so its error against the oracle's fp64 sum
is at most about 32 * 2^-24 * sum_h |y_h g_h|.
The router backward is fp32 against fp64: 1e-5 relative plus 1e-6 of the
row's sum_k |w_k gw_k|.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import synth

from .helpers import assert_act_close, bf16_f64

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def dev(a):
    return synth.to_torch(a, device="cuda")


def host(t):
    return synth.from_torch(t)


def _f64(a):
    return bf16_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


CASES = [
    synth.WORKLOADS["1"],
    synth.WORKLOADS["2b"],
    synth.WORKLOADS["4"],                                    # full size
    synth.WORKLOADS["5"].replace(S=3000),
    synth.WORKLOADS["4"].replace(S=500, H=4608),             # rows of 9 KB: 16 warps, a ragged second chunk
    synth.WORKLOADS["4"].replace(S=300, H=2304, dtype="f32"),  # fp32 rows of 9 KB
    synth.WORKLOADS["5"].replace(S=700, H=1536, dtype="f32"),  # fp32 rows of 6 KB: 6 warps, 3 KB chunks
    synth.Workload("bwd_ragged", 777, 264, 40, 5, 4, 3, "bf16", "none", True, seed=31),
    synth.Workload("bwd_2k", 300, 1032, 40, 5, 4, 3, "bf16", "none", True, seed=33),   # 2064-byte rows: 6 warps
    synth.Workload("bwd_8k", 200, 4104, 32, 4, 4, 0, "bf16", "none", True, seed=34),   # 8208-byte rows: 16 warps
    synth.Workload("bwd_k17_f32", 301, 260, 17, 17, 17, 1, "f32", "none", True, seed=32),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_combine_and_dispatch_backward(w):
    idx, wt = oracle.route_topk(synth.logits(w), w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    y = synth.expert_outputs(w)
    rng = np.random.default_rng(w.seed + 100)
    cast = (lambda a: a.astype(np.float32)) if w.dtype == "f32" else synth.f32_to_bf16_bits
    g = cast(rng.standard_normal((w.S, w.H), dtype=np.float32))
    gn = cast(rng.standard_normal((w.S, w.H), dtype=np.float32))
    ref_gy, ref_gw, ref_skip = oracle.combine_backward(g, y, lay["slot_of"], wt, gn=gn)

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gy, gw, skip = B.moe_combine_dual_residual_backward(dev(g), dev(y), dev(lay["slot_of"]), dev(wt),
                                                        grad_no_routed=dev(gn), status=status)
    valid = lay["row_src"] >= 0
    assert_act_close(host(gy)[valid], ref_gy[valid], "grad_y")
    assert np.all(host(gy)[~valid] == 0)  # padding rows untouched (the binding zero-fills)
    assert_act_close(host(skip), ref_skip, "grad_skip")
    # grad_w: fixed-order fp32 sum against fp64
    yg = _f64(y)[lay["slot_of"]]                      # [S,K,H]
    mag = np.einsum("skh,sh->sk", np.abs(yg), np.abs(_f64(g)))
    err = np.abs(host(gw).astype(np.float64) - ref_gw.astype(np.float64))
    assert np.all(err <= 32 * U * mag + 1e-30), float((err / (mag + 1e-30)).max())

    # dispatch backward of the expert-input gradients (here: the grad_y just computed)
    ref_gx = oracle.dispatch_backward(ref_gy, lay["slot_of"])
    gx = B.moe_dispatch_backward(dev(ref_gy), dev(lay["slot_of"]), status=status)
    assert_act_close(host(gx), ref_gx, "grad_x")
    assert status.item() == 0


def test_combine_backward_without_gn_and_skip():
    w = synth.WORKLOADS["2b"].replace(S=300)
    idx, wt = oracle.route_topk(synth.logits(w), w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    y = synth.expert_outputs(w)
    g = synth.f32_to_bf16_bits(np.random.default_rng(3).standard_normal((w.S, w.H), dtype=np.float32))
    ref_gy, ref_gw, ref_skip = oracle.combine_backward(g, y, lay["slot_of"], wt)
    gy, gw, skip = B.moe_combine_dual_residual_backward(dev(g), dev(y), dev(lay["slot_of"]), dev(wt))
    valid = lay["row_src"] >= 0
    assert_act_close(host(gy)[valid], ref_gy[valid], "grad_y")
    assert_act_close(host(skip), ref_skip, "grad_skip (= grad_out)")
    gy2, gw2, none = B.moe_combine_dual_residual_backward(dev(g), dev(y), dev(lay["slot_of"]), dev(wt),
                                                          want_skip=False)
    assert none is None
    assert torch.equal(gw2, gw) and torch.equal(gy2, gy)  # deterministic


def test_backward_skips_bad_slots():
    S, H, K, cap = 40, 256, 3, 150
    rng = np.random.default_rng(4)
    slot = rng.permutation(cap)[:S * K].reshape(S, K).astype(np.int32)
    slot[2, 1] = cap + 1
    slot[5, 0] = -1
    y = synth.f32_to_bf16_bits(rng.standard_normal((cap, H), dtype=np.float32))
    g = synth.f32_to_bf16_bits(rng.standard_normal((S, H), dtype=np.float32))
    w = rng.uniform(0.1, 1, (S, K)).astype(np.float32)
    ok = np.where((slot >= 0) & (slot < cap), slot, -1)
    ref_gy, ref_gw, _ = oracle.combine_backward(g, y, ok, w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gy, gw, _ = B.moe_combine_dual_residual_backward(dev(g), dev(y), dev(slot), dev(w), status=status)
    assert status.item() == B.MOE_STATUS_BAD_SLOT
    assert host(gw)[2, 1] == 0 and host(gw)[5, 0] == 0
    assert_act_close(host(gy), ref_gy, "grad_y")
    status.zero_()
    gx = B.moe_dispatch_backward(gy, dev(slot), status=status)
    assert status.item() == B.MOE_STATUS_BAD_SLOT
    assert_act_close(host(gx), oracle.dispatch_backward(ref_gy, ok), "grad_x")


@pytest.mark.parametrize("S,E,K", [(4096, 256, 8), (1000, 384, 8), (77, 8, 2), (300, 1024, 32), (5, 32, 32)])
def test_route_backward(S, E, K):
    rng = np.random.default_rng(S + E)
    logits = rng.standard_normal((S, E)).astype(np.float32)
    idx, wt = oracle.route_topk(logits, K)
    gw = rng.standard_normal((S, K)).astype(np.float32)
    ref = oracle.route_backward(idx, wt, gw, E)
    got = host(B.moe_route_topk_backward(dev(idx), dev(wt), dev(gw), E))
    scale = (np.abs(wt.astype(np.float64)) * np.abs(gw)).sum(axis=1, keepdims=True)
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= 1e-5 * np.abs(ref) + 1e-6 * scale)
    assert np.all(got[ref == 0] == 0)
