"""Pins for the oracle's dispatch and its number formats (CPU only).

* e4m3 encode: every bf16 bit pattern with |x| <= 448, and random fp32 values
  including exact ties, against torch's float8_e4m3fn conversion (a library
  routine, round to nearest even); hand-worked codes in
  tests/golden/e4m3_codes.txt; decode of all 256 codes against torch.
* bf16 rounding against torch's fp32 -> bfloat16 conversion.
* the FP8 dispatch against the error bounds that the format fixes: the
  dequantised value is within half an e4m3 step of x; every block whose amax is
  non-zero reaches the code magnitude 448; an all-zero block gives scale 0.
* the plain dispatch is an exact row copy.
"""
import os

import numpy as np
import pytest
import torch

from combine_moe_route_09_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _torch_e4m3(v_f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v_f32, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def _encode_all(oracle_lib, vals):
    return np.array([oracle_lib.e4m3_encode(float(v)) for v in vals], np.uint8)


def test_e4m3_golden(oracle_lib):
    with open(os.path.join(GOLDEN, "e4m3_codes.txt")) as f:
        rows = [l for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 15
    for line in rows:
        v, code = (p.strip() for p in line.split("|"))
        assert oracle_lib.e4m3_encode(float(v)) == int(code, 16), line


def test_e4m3_decode_all_codes(oracle_lib):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle_lib.e4m3_decode(int(c)) for c in codes], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_e4m3_encode_every_bf16_in_range(oracle_lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = synth.bf16_bits_to_f32(bits)
    keep = np.isfinite(vals) & (np.abs(vals) <= 448.0)
    vals = vals[keep]
    np.testing.assert_array_equal(_encode_all(oracle_lib, vals), _torch_e4m3(vals))


def test_e4m3_encode_fp32_values_and_ties(oracle_lib):
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(20000) * np.exp2(rng.uniform(-14, 8, 20000))).astype(np.float32)
    v = v[np.abs(v) <= 448]
    # exact midpoints between adjacent codes (ties) and their fp32 neighbours
    codes = np.arange(0, 0x7E, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    allv = np.concatenate([v, near, -near])
    np.testing.assert_array_equal(_encode_all(oracle_lib, allv), _torch_e4m3(allv))


def test_e4m3_saturates(oracle_lib):
    for v in (448.0, 449.0, 470.0, 1e6, 3.4e38):
        assert oracle_lib.e4m3_encode(v) == 0x7E
        assert oracle_lib.e4m3_encode(-v) == 0xFE


def test_bf16_round_matches_torch(oracle_lib):
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(20000) * np.exp2(rng.uniform(-130, 120, 20000))).astype(np.float32)
    # exact bf16 midpoints (ties) and neighbours
    b = rng.integers(0, 0x7F7F, 3000).astype(np.uint32)
    mids = ((b << 16) | 0x8000).view(np.float32)
    allv = np.concatenate([v, mids, -mids, np.nextafter(mids, np.float32(0)),
                           np.array([0.0, -0.0, 3.3895314e38, 3.40282e38], np.float32)])
    ref = synth.f32_to_bf16_bits(allv)
    got = np.array([oracle_lib.bf16_round(float(x)) for x in allv], np.uint16)
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_plain_dispatch_is_row_copy(oracle_lib, dt):
    w = synth.WORKLOADS["2b"].replace(dtype=dt, S=300)
    x = synth.activations(w)
    idx, _ = oracle_lib.route_topk(synth.logits(w), w.K)
    lay = oracle_lib.layout(idx, w.E, w.R, w.P)
    sentinel = np.full((lay["cap"], w.H), 0x5A5A if dt == "bf16" else 7.0,
                       np.uint16 if dt == "bf16" else np.float32)
    xd, _ = oracle_lib.dispatch(x, lay["slot_of"], lay["cap"], xd=sentinel.copy())
    for t in range(w.S):
        for k in range(w.K):
            assert np.array_equal(xd[lay["slot_of"][t, k]], x[t])
    pad = lay["row_src"] < 0
    assert np.array_equal(xd[pad], sentinel[pad])  # padding rows untouched


def _fp8_case(oracle_lib, w):
    x = synth.activations(w)
    idx, _ = oracle_lib.route_topk(synth.logits(w), w.K)
    lay = oracle_lib.layout(idx, w.E, w.R, w.P)
    xd, xs = oracle_lib.dispatch(x, lay["slot_of"], lay["cap"], quant=oracle_lib.QUANT_FP8_E4M3_B128)
    return x, lay, xd, xs


def test_fp8_dispatch_error_bounds(oracle_lib):
    w = synth.WORKLOADS["3"].replace(S=48)
    x, lay, xd, xs = _fp8_case(oracle_lib, w)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    nb = w.H // 128
    for t in range(w.S):
        rows = lay["slot_of"][t]
        # identical bytes and scales in all K copies
        for k in range(1, w.K):
            assert np.array_equal(xd[rows[k]], xd[rows[0]])
            assert np.array_equal(xs[rows[k]], xs[rows[0]])
        q = torch.from_numpy(xd[rows[0]].copy()).view(torch.float8_e4m3fn).double().numpy()
        s = xs[rows[0]].astype(np.float64)
        blk = xf[t].reshape(nb, 128)
        amax = np.abs(blk).max(axis=1)
        np.testing.assert_array_equal(s.astype(np.float32), (amax / 448.0).astype(np.float32))
        qq = q.reshape(nb, 128)
        assert np.all(np.abs(qq).max(axis=1)[amax > 0] == 448.0)
        deq = qq * s[:, None]
        u = np.abs(blk) / s[:, None]
        # normal range: half a step of a 3-bit mantissa is 2^-4 relative; the fp32
        # quotient adds at most one fp32 rounding
        normal = u >= 2.0 ** -6
        err = np.abs(deq - blk)
        assert np.all(err[normal] <= (2.0 ** -4) * np.abs(blk[normal]) * (1 + 2.0 ** -20))
        # subnormal range: half the subnormal step 2^-9, times the scale
        sub = ~normal
        assert np.all(err[sub] <= (2.0 ** -10) * np.broadcast_to(s[:, None], blk.shape)[sub] * (1 + 2.0 ** -20))


def test_fp8_outlier_channels_dominate_amax(oracle_lib):
    w = synth.WORKLOADS["3"].replace(S=8)
    x, lay, xd, xs = _fp8_case(oracle_lib, w)
    # blocks holding an outlier channel (x20) get a clearly larger scale
    s = xs[lay["slot_of"][:, 0]]
    assert s.max() / np.median(s) > 5


def test_fp8_zero_block_and_signed_zero(oracle_lib):
    H = 256
    x = np.zeros((1, H), np.float32)
    x[0, 0] = -0.0
    x[0, 5] = -0.0
    x[0, 128:] = np.linspace(-3, 3, 128, dtype=np.float32)
    slot_of = np.array([[1]], np.int32)
    xd, xs = oracle_lib.dispatch(x, slot_of, 2, quant=oracle_lib.QUANT_FP8_E4M3_B128)
    assert xs[1, 0] == 0.0
    assert xd[1, 0] == 0x80 and xd[1, 5] == 0x80 and xd[1, 1] == 0x00
    assert xs[1, 1] == np.float32(3.0) / np.float32(448.0)
    assert xd[1, 128] == 0xFE and xd[1, 255] == 0x7E
    assert np.all(xd[0] == 0) and np.all(xs[0] == 0)  # row not mapped: untouched


def test_dispatch_negative_slot_skipped_and_overflow(oracle_lib):
    x = np.ones((2, 8), np.float32)
    xd, _ = oracle_lib.dispatch(x, np.array([[-1], [0]], np.int32), 1)
    assert np.all(xd[0] == 1)
    with pytest.raises(oracle_lib.OracleError) as e:
        oracle_lib.dispatch(x, np.array([[0], [1]], np.int32), 1)
    assert e.value.rc == oracle_lib.EOVERFLOW
