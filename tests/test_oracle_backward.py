"""Pins for the oracle's backward functions (CPU only).

The combine and the dispatch are linear maps, so their backward functions are
pinned by the adjoint ("dot product") identity against the already-pinned
forward oracle: <F(dx), g> = <dx, F^T(g)>, evaluated in fp64 on fp32 data.
The combine is linear in y (and in shared/residual) for fixed weights and
linear in the weights for fixed y, which pins grad_y, grad_skip and grad_w.
The router backward is pinned by central finite differences of scipy's
softmax over the selected logits.
"""
import numpy as np
import pytest
from scipy.special import softmax

from combine_moe_route_09_b200 import synth


def _setup(oracle_lib, S, H, E, K, R, P, seed):
    w = synth.Workload("bwd", S, H, E, K, R, P, "f32", "none", True, seed=seed)
    idx, wt = oracle_lib.route_topk(synth.logits(w), K)
    lay = oracle_lib.layout(idx, E, R, P)
    return w, idx, wt, lay


def _dot(a, b):
    return float(np.dot(a.astype(np.float64).ravel(), b.astype(np.float64).ravel()))


@pytest.mark.parametrize("S,H,E,K,R,P,seed", [(64, 32, 8, 2, 2, 0, 1), (50, 24, 16, 4, 4, 4, 2),
                                              (33, 128, 64, 8, 8, 16, 3)])
def test_combine_backward_adjoint_in_y_shared_residual(oracle_lib, S, H, E, K, R, P, seed):
    w, idx, wt, lay = _setup(oracle_lib, S, H, E, K, R, P, seed)
    rng = np.random.default_rng(seed)
    cap = lay["cap"]
    dy = rng.standard_normal((cap, H)).astype(np.float32)
    dsh = rng.standard_normal((S, H)).astype(np.float32)
    dres = rng.standard_normal((S, H)).astype(np.float32)
    g = rng.standard_normal((S, H)).astype(np.float32)
    gn = rng.standard_normal((S, H)).astype(np.float32)
    out, rnr = oracle_lib.combine(dy, lay["slot_of"], wt, shared=dsh, residual=dres)
    grad_y, grad_w, skip = oracle_lib.combine_backward(g, dy, lay["slot_of"], wt, gn=gn)
    lhs = _dot(out, g) + _dot(rnr, gn)
    rhs = _dot(dy, grad_y) + _dot(dsh, skip) + _dot(dres, skip)
    mag = (np.abs(out) * np.abs(g)).sum() + (np.abs(rnr) * np.abs(gn)).sum()
    assert abs(lhs - rhs) <= 1e-5 * mag
    # padding rows of grad_y are untouched (zeros)
    assert np.all(grad_y[lay["row_src"] < 0] == 0)


@pytest.mark.parametrize("S,H,E,K,seed", [(40, 64, 8, 2, 4), (30, 96, 32, 8, 5)])
def test_combine_backward_adjoint_in_weights(oracle_lib, S, H, E, K, seed):
    w, idx, wt, lay = _setup(oracle_lib, S, H, E, K, 2, 0, seed)
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((lay["cap"], H)).astype(np.float32)
    g = rng.standard_normal((S, H)).astype(np.float32)
    dw = rng.standard_normal((S, K)).astype(np.float32)
    out, _ = oracle_lib.combine(y, lay["slot_of"], dw)             # linear in the weights
    _, grad_w, _ = oracle_lib.combine_backward(g, y, lay["slot_of"], wt, want_skip=False)
    lhs, rhs = _dot(out, g), _dot(dw, grad_w)
    mag = (np.abs(out) * np.abs(g)).sum()
    assert abs(lhs - rhs) <= 1e-5 * mag


def test_combine_backward_skipped_pairs(oracle_lib):
    y = np.arange(8, dtype=np.float32).reshape(4, 2)
    slot = np.array([[0, -1], [3, 1]], np.int32)
    w = np.array([[0.5, 0.5], [0.25, 0.75]], np.float32)
    g = np.array([[1.0, 2.0], [-1.0, 4.0]], np.float32)
    grad_y, grad_w, skip = oracle_lib.combine_backward(g, y, slot, w)
    assert grad_w[0, 1] == 0.0
    np.testing.assert_array_equal(grad_y[0], [0.5, 1.0])
    np.testing.assert_array_equal(grad_y[2], [0.0, 0.0])     # no pair maps to row 2
    np.testing.assert_array_equal(grad_y[3], [-0.25, 1.0])
    assert grad_w[1, 0] == 6 * -1.0 + 7 * 4.0
    np.testing.assert_array_equal(skip, g)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_dispatch_backward_adjoint(oracle_lib, dt):
    w, idx, wt, lay = _setup(oracle_lib, 70, 48, 16, 4, 4, 8, 6)
    rng = np.random.default_rng(7)
    dx = rng.standard_normal((70, 48)).astype(np.float32)
    G = rng.standard_normal((lay["cap"], 48)).astype(np.float32)
    if dt == "bf16":
        dx, G = synth.f32_to_bf16_bits(dx), synth.f32_to_bf16_bits(G)
    xd, _ = oracle_lib.dispatch(dx, lay["slot_of"], lay["cap"])
    gx = oracle_lib.dispatch_backward(G, lay["slot_of"])
    f = (lambda a: a.astype(np.float64)) if dt == "f32" else (lambda a: synth.bf16_bits_to_f32(a).astype(np.float64))
    lhs = float((f(xd) * f(G)).sum())
    rhs = float((f(dx) * f(gx)).sum())
    tol = 1e-5 if dt == "f32" else 2.0 ** -7  # bf16: the K-term sums are rounded once to bf16
    mag = float((np.abs(f(xd)) * np.abs(f(G))).sum())
    assert abs(lhs - rhs) <= tol * mag


def test_route_backward_finite_differences(oracle_lib):
    rng = np.random.default_rng(8)
    S, E, K = 20, 12, 4
    logits = rng.standard_normal((S, E)).astype(np.float32)
    idx, wt = oracle_lib.route_topk(logits, K)
    gw = rng.standard_normal((S, K)).astype(np.float32)
    got = oracle_lib.route_backward(idx, wt, gw, E)
    h = 1e-6
    for t in range(S):
        sel = logits[t, idx[t]].astype(np.float64)
        for e in range(E):
            if e not in idx[t]:
                assert got[t, e] == 0.0
                continue
            j = list(idx[t]).index(e)
            up, dn = sel.copy(), sel.copy()
            up[j] += h
            dn[j] -= h
            fd = (np.dot(softmax(up), gw[t]) - np.dot(softmax(dn), gw[t])) / (2 * h)
            assert abs(got[t, e] - fd) <= 1e-6 + 1e-5 * abs(fd)


def test_route_backward_rows_sum_to_zero(oracle_lib):
    # the softmax weights sum to 1, so the gradient over the selected logits sums to 0
    rng = np.random.default_rng(9)
    logits = rng.standard_normal((50, 64)).astype(np.float32)
    idx, wt = oracle_lib.route_topk(logits, 8)
    got = oracle_lib.route_backward(idx, wt, rng.standard_normal((50, 8)).astype(np.float32), 64)
    np.testing.assert_allclose(got.astype(np.float64).sum(axis=1), 0.0, atol=1e-6)
