"""GPU parity: every step through the C ABI against the CPU oracle.

Each step is checked on its own with identical inputs (the oracle's upstream
results are fed to both sides), then the whole pass is run the way the
benchmark launches it (MoeBuffer.step on one stream) and its outputs compared
with the oracle's pass.  All five workloads run at full size: the oracle
finishes each in seconds.  Tolerances are stated in tests/helpers.py.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import synth
from combine_moe_route_09_b200.buffer import MoeBuffer

from .helpers import abs_weighted_sum, assert_act_close, assert_f32_close, workload_inputs

pytestmark = pytest.mark.gpu

WORKLOADS = ["1", "2", "2b", "3", "4", "5"]


def dev(a):
    return synth.to_torch(a, device="cuda")


def host(t):
    return synth.from_torch(t)


@pytest.fixture(scope="module", params=WORKLOADS)
def case(request):
    """Inputs and the oracle's pass for one workload (pytest groups the tests by it)."""
    w = synth.WORKLOADS[request.param]
    inp = workload_inputs(w)
    idx, wt = oracle.route_topk(inp["logits"], w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    q = oracle.QUANT_FP8_E4M3_B128 if w.quant == "fp8" else oracle.QUANT_NONE
    xd, xs = oracle.dispatch(inp["x"], lay["slot_of"], lay["cap"], quant=q)
    out, rnr = oracle.combine(inp["y"], lay["slot_of"], wt, inp.get("shared"), inp.get("residual"))
    return w, inp, dict(idx=idx, w=wt, lay=lay, xd=xd, xs=xs, out=out, rnr=rnr)


def test_route(case):
    w, inp, ref = case
    idx, wt = B.moe_route_topk(dev(inp["logits"]), w.K)
    np.testing.assert_array_equal(host(idx), ref["idx"])
    assert_f32_close(host(wt), ref["w"], 1e-5, "topk_w")


def _check_layout(lay_gpu, ref_lay):
    for k in ("counts", "offsets", "rank_offsets", "slot_of", "row_src"):
        np.testing.assert_array_equal(host(getattr(lay_gpu, k)), ref_lay[k], err_msg=k)


def test_layout(case):
    w, inp, ref = case
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lay = B.moe_dispatch_layout(dev(ref["idx"]), w.E, w.R, w.P, status=status)
    _check_layout(lay, ref["lay"])
    assert status.item() == 0


def _sentinel_buffers(w, cap):
    if w.quant == "fp8":
        xd = torch.full((cap, w.H), 0x5A, dtype=torch.uint8, device="cuda")
        xs = torch.full((cap, w.H // 128), -7.0, dtype=torch.float32, device="cuda")
        return xd, xs
    t = torch.float32 if w.dtype == "f32" else torch.bfloat16
    return torch.full((cap, w.H), -7.0, dtype=t, device="cuda"), None


def test_dispatch(case):
    w, inp, ref = case
    lay = ref["lay"]
    xd, xs = _sentinel_buffers(w, lay["cap"])
    q = B.MOE_QUANT_FP8_E4M3_B128 if w.quant == "fp8" else B.MOE_QUANT_NONE
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.moe_dispatch(dev(inp["x"]), dev(lay["slot_of"]), lay["cap"], q, xd, xs, status=status)
    valid = lay["row_src"] >= 0
    gxd = host(xd)
    if w.quant == "fp8":
        np.testing.assert_array_equal(gxd[valid], ref["xd"][valid])
        np.testing.assert_array_equal(host(xs)[valid], ref["xs"][valid])
        assert np.all(gxd[~valid] == 0x5A) and np.all(host(xs)[~valid] == -7.0)  # padding untouched
    else:
        np.testing.assert_array_equal(gxd[valid], ref["xd"][valid])
        sent = host(torch.full((1,), -7.0, dtype=xd.dtype))[0]
        assert np.all(gxd[~valid] == sent)
    assert status.item() == 0


def test_combine(case):
    w, inp, ref = case
    lay = ref["lay"]
    out, rnr = B.moe_combine_dual_residual(
        dev(inp["y"]), dev(lay["slot_of"]), dev(ref["w"]),
        dev(inp["shared"]) if w.fused else None, dev(inp["residual"]) if w.fused else None)
    assert_act_close(host(out), ref["out"], "residual_out")
    if w.fused:
        assert_act_close(host(rnr), ref["rnr"], "residual_no_routed_out")
    else:
        assert rnr is None


def test_full_pass_as_benchmarked(case):
    """MoeBuffer.step: the exact call sequence bench.py times, twice in a row."""
    w, inp, ref = case
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, dtype=dt, fp8=w.quant == "fp8")
    args = [dev(inp["logits"]), dev(inp["x"]), dev(inp["y"])]
    if w.fused:
        args += [dev(inp["shared"]), dev(inp["residual"])]
    weight_slack = 2e-5 * abs_weighted_sum(inp["y"], ref["lay"]["slot_of"], ref["w"])
    for _ in range(2):
        buf.step(*args)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(buf.topk_idx), ref["idx"])
        _check_layout(buf.layout, ref["lay"])
        valid = ref["lay"]["row_src"] >= 0
        np.testing.assert_array_equal(host(buf.xd)[valid], ref["xd"][valid])
        if w.quant == "fp8":
            np.testing.assert_array_equal(host(buf.xs)[valid], ref["xs"][valid])
        assert_f32_close(host(buf.topk_w), ref["w"], 1e-5, "topk_w")
        # The GPU combine used the GPU's weights, equal to the oracle's within 1e-5
        # relative, so its outputs may differ from the oracle's pass by that much
        # of sum_k |w_k y_k| on top of the combine tolerance.
        assert_act_close(host(buf.out), ref["out"], "residual_out", extra_abs=weight_slack)
        if w.fused:
            assert_act_close(host(buf.out_no_routed), ref["rnr"], "residual_no_routed_out")
        assert buf.read_status() == 0
    assert int(buf.workspace[:8].sum().item()) == 0  # arrival ticket and barrier count back at zero


def test_both_step_plans_give_the_pass(case):
    """MoeBuffer.step with route + layout + dispatch in the fused kernel (where it
    applies) and with the separate kernels: the same pass both times."""
    w, inp, ref = case
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q = B.MOE_QUANT_FP8_E4M3_B128 if w.quant == "fp8" else B.MOE_QUANT_NONE
    applies = B.moe_route_dispatch_kernels(w.S, w.H, w.E, w.K, dt, q) == 1
    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, dtype=dt, fp8=w.quant == "fp8", fused=applies)
    args = [dev(inp["logits"]), dev(inp["x"]), dev(inp["y"])]
    if w.fused:
        args += [dev(inp["shared"]), dev(inp["residual"])]
    weight_slack = 2e-5 * abs_weighted_sum(inp["y"], ref["lay"]["slot_of"], ref["w"])
    valid = ref["lay"]["row_src"] >= 0
    for fused in ([True, False] if applies else [False]):
        buf.fused = fused
        assert buf.kernels_per_step == (2 if fused else 3 + B.moe_dispatch_layout_kernels(w.S, w.E, w.K))
        buf.layout.slot_of.fill_(-7)
        buf.topk_idx.fill_(-7)
        buf.out.zero_()
        buf.step(*args)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(buf.topk_idx), ref["idx"])
        _check_layout(buf.layout, ref["lay"])
        np.testing.assert_array_equal(host(buf.xd)[valid], ref["xd"][valid])
        if w.quant == "fp8":
            np.testing.assert_array_equal(host(buf.xs)[valid], ref["xs"][valid])
        assert_act_close(host(buf.out), ref["out"], "residual_out", extra_abs=weight_slack)
        assert buf.read_status() == 0


def test_captured_step_replays_the_pass(case):
    """One step captured in a CUDA graph and replayed twice gives the oracle's pass."""
    w, inp, ref = case
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, dtype=dt, fp8=w.quant == "fp8")
    args = [dev(inp["logits"]), dev(inp["x"]), dev(inp["y"])]
    if w.fused:
        args += [dev(inp["shared"]), dev(inp["residual"])]
    buf.step(*args)
    torch.cuda.synchronize()
    graph = buf.capture(*args)
    weight_slack = 2e-5 * abs_weighted_sum(inp["y"], ref["lay"]["slot_of"], ref["w"])
    for _ in range(2):
        buf.out.zero_()
        buf.layout.slot_of.fill_(-7)
        graph.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(buf.topk_idx), ref["idx"])
        _check_layout(buf.layout, ref["lay"])
        valid = ref["lay"]["row_src"] >= 0
        np.testing.assert_array_equal(host(buf.xd)[valid], ref["xd"][valid])
        assert_act_close(host(buf.out), ref["out"], "residual_out", extra_abs=weight_slack)
        assert buf.read_status() == 0


@pytest.mark.parametrize("name", ["3", "4"])
def test_captured_step_with_new_inputs(name):
    """A captured step replayed after its inputs were refilled in place with another
    draw (different routing, different activations) gives that draw's pass."""
    w = synth.WORKLOADS[name]
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, dtype=dt, fp8=w.quant == "fp8")
    first = workload_inputs(w)
    args = {k: dev(v) for k, v in first.items()}
    order = ["logits", "x", "y"] + (["shared", "residual"] if w.fused else [])
    buf.step(*[args[k] for k in order])
    torch.cuda.synchronize()
    graph = buf.capture(*[args[k] for k in order])
    w2 = w.replace(seed=w.seed + 1000)
    second = workload_inputs(w2)
    for k in order:
        args[k].copy_(dev(second[k]))
    graph.replay()
    torch.cuda.synchronize()
    idx, wt = oracle.route_topk(second["logits"], w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    q = oracle.QUANT_FP8_E4M3_B128 if w.quant == "fp8" else oracle.QUANT_NONE
    xd, xs = oracle.dispatch(second["x"], lay["slot_of"], lay["cap"], quant=q)
    out, rnr = oracle.combine(second["y"], lay["slot_of"], wt, second.get("shared"), second.get("residual"))
    assert not np.array_equal(idx, oracle.route_topk(first["logits"], w.K)[0])  # the routing did change
    np.testing.assert_array_equal(host(buf.topk_idx), idx)
    _check_layout(buf.layout, lay)
    valid = lay["row_src"] >= 0
    np.testing.assert_array_equal(host(buf.xd)[valid], xd[valid])
    if q == oracle.QUANT_FP8_E4M3_B128:
        np.testing.assert_array_equal(host(buf.xs)[valid], xs[valid])
    slack = 2e-5 * abs_weighted_sum(second["y"], lay["slot_of"], wt)
    assert_act_close(host(buf.out), out, "residual_out", extra_abs=slack)
    if w.fused:
        assert_act_close(host(buf.out_no_routed), rnr, "residual_no_routed_out")
    assert buf.read_status() == 0
