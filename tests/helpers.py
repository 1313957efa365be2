"""Shared test helpers: tolerances, and the oracle / GPU versions of one pass.

Tolerances (the accuracy bar of the four steps):
* top-K indices, counts, offsets, slots, row sources, dispatched bytes, FP8
  codes and scales: bit-exact;
* gating weights: |gpu - oracle| <= 1e-5 * |oracle| (the oracle evaluates
  the softmax in fp64; the kernel's fp32 expf / sum / divide stay well within);
* combine outputs: at most 1 bf16 ulp for bf16 outputs, and 1e-5 relative for
  fp32 outputs, after an fp32 accumulate.
"""
from __future__ import annotations

import numpy as np

from combine_moe_route_09_b200 import synth


def bf16_f64(a: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(a).astype(np.float64)


def bf16_ulp(r: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |r| (r in float64, a bf16 value)."""
    a = np.abs(r)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    u = np.exp2(e - 7)
    return np.where(a > 0, u, 2.0 ** -133)


def assert_bf16_close(got: np.ndarray, ref: np.ndarray, ulps: float = 1.0, what: str = "",
                      extra_abs=0.0):
    g, r = bf16_f64(got), bf16_f64(ref)
    err = np.abs(g - r)
    lim = ulps * bf16_ulp(r) + extra_abs
    bad = err > lim
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements beyond {ulps} bf16 ulp; "
                             f"first at {tuple(i)}: got {g[tuple(i)]!r} ref {r[tuple(i)]!r}")


def assert_f32_close(got: np.ndarray, ref: np.ndarray, rtol: float = 1e-5, what: str = "",
                     extra_abs=0.0):
    g, r = got.astype(np.float64), ref.astype(np.float64)
    bad = np.abs(g - r) > rtol * np.abs(r) + 1e-37 + extra_abs
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} beyond rtol {rtol}; "
                             f"first at {tuple(i)}: got {g[tuple(i)]!r} ref {r[tuple(i)]!r}")


def assert_act_close(got: np.ndarray, ref: np.ndarray, what: str = "", extra_abs=0.0):
    """Combine outputs: 1 bf16 ulp (bf16) or 1e-5 relative (fp32), plus an optional
    absolute slack that a caller derives from known input differences."""
    if ref.dtype == np.uint16:
        assert_bf16_close(got, ref, 1.0, what, extra_abs)
    else:
        assert_f32_close(got, ref, 1e-5, what, extra_abs)


def abs_weighted_sum(y: np.ndarray, slot_of: np.ndarray, w: np.ndarray, chunk: int = 256):
    """sum_k |w[t,k]| * |y[slot_of[t,k], :]| in fp64, [S,H] (a bound, not a result)."""
    S, K = slot_of.shape
    out = np.empty((S, y.shape[1]), np.float64)
    for t0 in range(0, S, chunk):
        sl = slot_of[t0:t0 + chunk]
        yy = y[np.maximum(sl, 0)]
        yy = yy.astype(np.float64) if y.dtype == np.float32 else bf16_f64(yy)
        ww = np.abs(w[t0:t0 + chunk]).astype(np.float64) * (sl >= 0)
        out[t0:t0 + chunk] = np.einsum("sk,skh->sh", ww, np.abs(yy))
    return out


def workload_inputs(w: synth.Workload) -> dict:
    d = dict(logits=synth.logits(w), x=synth.activations(w), y=synth.expert_outputs(w))
    if w.fused:
        d["shared"] = synth.shared_out(w)
        d["residual"] = synth.residual(w)
    return d
