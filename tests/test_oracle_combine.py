"""Pins for the oracle's combine and dual-residual epilogue (CPU only).

* Identity round trip: dispatch -> identity expert -> combine with the router
  weights (which sum to 1) returns the input.
* Closed form with per-expert gains: out[t] = x[t] * sum_k w_k g_{e_k}.
* The dual residual (FarSkip-Collective): residual_no_routed is the correctly
  rounded residual + shared_out, and the main stream equals the standard MoE
  block output residual + (shared_out + sum_k w_k y_k) evaluated in fp64 within
  the fp32 accumulation error bound.
* Pairs with a negative slot contribute nothing.
"""
import numpy as np
import pytest

from combine_moe_route_09_b200 import synth

U32 = 2.0 ** -24


def _f(a):
    return synth.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _route_layout(oracle_lib, w):
    idx, wt = oracle_lib.route_topk(synth.logits(w), w.K)
    lay = oracle_lib.layout(idx, w.E, w.R, w.P)
    return idx, wt, lay


@pytest.mark.parametrize("name,S", [("1", 128), ("2b", 256), ("5", 512)])
def test_identity_round_trip(oracle_lib, name, S):
    w = synth.WORKLOADS[name].replace(S=S)
    x = synth.activations(w)
    idx, wt, lay = _route_layout(oracle_lib, w)
    y, _ = oracle_lib.dispatch(x, lay["slot_of"], lay["cap"])
    out, rnr = oracle_lib.combine(y, lay["slot_of"], wt)
    assert rnr is None
    if w.dtype == "f32":
        np.testing.assert_allclose(out, x, rtol=(w.K + 2) * U32, atol=0)
    else:
        np.testing.assert_array_equal(out, x)  # the tiny fp32 deviation never crosses half a bf16 step


def test_closed_form_with_gains(oracle_lib):
    w = synth.WORKLOADS["1"]
    x = synth.activations(w)
    g = synth.expert_gains(w)
    idx, wt, lay = _route_layout(oracle_lib, w)
    xd, _ = oracle_lib.dispatch(x, lay["slot_of"], lay["cap"])
    # expert stand-in: y = g_e * x on every dispatched row (row -> expert from row_src)
    y = np.zeros_like(xd)
    for s in np.nonzero(lay["row_src"] >= 0)[0]:
        i = lay["row_src"][s]
        y[s] = xd[s] * g[idx.reshape(-1)[i]]
    out, _ = oracle_lib.combine(y, lay["slot_of"], wt)
    ref = x.astype(np.float64) * (wt.astype(np.float64) * g[idx].astype(np.float64)).sum(axis=1)[:, None]
    np.testing.assert_allclose(out, ref, rtol=4 * (w.K + 2) * U32, atol=1e-30)


@pytest.mark.parametrize("name,S", [("1", 128), ("4", 64), ("5", 256)])
def test_dual_residual(oracle_lib, name, S):
    w = synth.WORKLOADS[name].replace(S=S)
    y = synth.expert_outputs(w)
    sh, rs = synth.shared_out(w), synth.residual(w)
    idx, wt, lay = _route_layout(oracle_lib, w)
    out, rnr = oracle_lib.combine(y, lay["slot_of"], wt, shared=sh, residual=rs)
    # residual_no_routed: the correctly rounded fp32 sum, then (bf16) one more rounding
    exact = _f(rs) + _f(sh)
    r32 = exact.astype(np.float32)  # numpy rounds fp64 -> fp32 to nearest even
    if w.dtype == "bf16":
        np.testing.assert_array_equal(rnr, synth.f32_to_bf16_bits(r32))
    else:
        np.testing.assert_array_equal(rnr, r32)
    # main stream = residual + (shared + sum_k w_k y_k), fp64 via a library einsum
    yg = _f(y)[lay["slot_of"]]                                  # [S,K,H] gathered
    routed = np.einsum("sk,skh->sh", wt.astype(np.float64), yg)
    ref = _f(rs) + (_f(sh) + routed)
    mag = np.abs(_f(rs)) + np.abs(_f(sh)) + np.einsum("sk,skh->sh", np.abs(wt.astype(np.float64)), np.abs(yg))
    bound = (w.K + 2) * U32 * mag
    got = _f(out)
    if w.dtype == "bf16":
        bound = bound + np.abs(ref) * 2.0 ** -8 + 1e-38  # one final bf16 rounding
    assert np.all(np.abs(got - ref) <= bound)
    # without the routed term the two streams would coincide: check the routed part is really there
    assert np.mean(np.abs(got - _f(rnr))) > 0.1


def test_residual_only_and_shared_only(oracle_lib):
    w = synth.WORKLOADS["1"].replace(S=16)
    y = synth.expert_outputs(w)
    sh, rs = synth.shared_out(w), synth.residual(w)
    idx, wt, lay = _route_layout(oracle_lib, w)
    plain, _ = oracle_lib.combine(y, lay["slot_of"], wt)
    only_r, none1 = oracle_lib.combine(y, lay["slot_of"], wt, residual=rs)
    only_s, none2 = oracle_lib.combine(y, lay["slot_of"], wt, shared=sh)
    assert none1 is None and none2 is None
    np.testing.assert_array_equal(only_r, (rs + plain).astype(np.float32))
    np.testing.assert_array_equal(only_s, (sh + plain).astype(np.float32))


def test_negative_slots_contribute_nothing(oracle_lib):
    y = np.array([[1.0, 2.0], [10.0, 20.0]], np.float32)
    slot_of = np.array([[0, -1], [1, 0]], np.int32)
    w = np.array([[0.5, 0.5], [0.25, 0.75]], np.float32)
    out, _ = oracle_lib.combine(y, slot_of, w)
    np.testing.assert_array_equal(out, np.array([[0.5, 1.0], [3.25, 6.5]], np.float32))


def test_combine_k_order_is_fixed(oracle_lib):
    # fp32 accumulation in k order: (1e8 * 1 + 1) + (-1e8) = 0 in fp32, not 1
    y = np.array([[1e8], [1.0], [-1e8]], np.float32)
    out, _ = oracle_lib.combine(y, np.array([[0, 1, 2]], np.int32), np.ones((1, 3), np.float32))
    assert out[0, 0] == 0.0
    out2, _ = oracle_lib.combine(y, np.array([[0, 2, 1]], np.int32), np.ones((1, 3), np.float32))
    assert out2[0, 0] == 1.0


@pytest.mark.parametrize("name,S", [("4", 48), ("3", 32)])
def test_combine_fp8_equals_combine_of_dequantised_rows(oracle_lib, name, S):
    """The FP8-input combine equals the fp32 combine of rows dequantised independently:
    torch's e4m3 decode, times the block scale in numpy fp32."""
    import torch

    w = synth.WORKLOADS[name].replace(S=S)
    x = synth.activations(w)
    idx, wt, lay = _route_layout(oracle_lib, w)
    yq, ys = oracle_lib.dispatch(x, lay["slot_of"], lay["cap"], quant=oracle_lib.QUANT_FP8_E4M3_B128)
    deq = torch.from_numpy(yq).view(torch.float8_e4m3fn).float().numpy()
    deq = (deq * np.repeat(ys, 128, axis=1)).astype(np.float32)          # fp32 product
    rng = np.random.default_rng(5)
    sh = rng.standard_normal((S, w.H)).astype(np.float32)
    rs = rng.standard_normal((S, w.H)).astype(np.float32)
    for kw in (dict(), dict(shared=sh, residual=rs)):
        ref, ref_n = oracle_lib.combine(deq, lay["slot_of"], wt, **kw)
        got, got_n = oracle_lib.combine_fp8(yq, ys, lay["slot_of"], wt, dtype="f32", **kw)
        np.testing.assert_array_equal(got, ref)
        if kw:
            np.testing.assert_array_equal(got_n, ref_n)
    # identity round trip through the quantiser: within the e4m3 error bound
    out, _ = oracle_lib.combine_fp8(yq, ys, lay["slot_of"], wt, dtype="f32")
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    assert np.all(np.abs(out - xf) <= 2.0 ** -4 * np.abs(xf) + np.repeat(ys[lay["slot_of"][:, 0]], 128, 1) * 2.0 ** -9)
