"""Pins for the oracle's router variant: sigmoid scores, selection-only bias,
group-limited top-K (CPU only).

* The fp32 exp the variant uses is within 2 ulp of fp64 exp over its range,
  exact at 0, monotone, with the stated overflow / underflow thresholds; the
  sigmoid is within 3 ulp of fp64.
* Selection is checked against a reference built with numpy/scipy in fp64
  (expit, library sorts with group masking) on logits spaced far wider than
  fp32 rounding, so both precisions agree on every order.
* Weights: proportional to the unbiased scores, summing to `scale` when
  normalised; hand-made ties go to the lower expert / group.
"""
import numpy as np
import pytest
from scipy.special import expit


def test_exp_accuracy_and_shape(oracle_lib):
    x = np.concatenate([np.linspace(-103.9, 88.7, 150001), np.random.default_rng(0).uniform(-20, 20, 50000)])
    x = x.astype(np.float32)
    e = oracle_lib.route_exp(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    normal = ref >= 2.0 ** -126
    assert np.all(np.abs(e[normal] - ref[normal]) <= 2 * 2.0 ** -23 * ref[normal])
    sub = ~normal
    assert np.all(np.abs(e[sub] - ref[sub]) <= 2.0 ** -149 * 2)      # subnormal results: within 2 steps
    xs = np.sort(x)
    assert np.all(np.diff(oracle_lib.route_exp(xs).astype(np.float64)) >= 0)
    assert oracle_lib.route_exp(np.array([0.0], np.float32))[0] == 1.0
    assert np.isinf(oracle_lib.route_exp(np.array([89.0], np.float32))[0])
    assert oracle_lib.route_exp(np.array([-104.0], np.float32))[0] == 0.0


def test_sigmoid_accuracy(oracle_lib):
    x = np.linspace(-30, 30, 60001).astype(np.float32)
    s = oracle_lib.route_sigmoid(x).astype(np.float64)
    ref = expit(x.astype(np.float64))
    assert np.all(np.abs(s - ref) <= 3 * 2.0 ** -24 * ref)
    assert oracle_lib.route_sigmoid(np.array([0.0], np.float32))[0] == 0.5


def _reference(logits, K, bias, n_group, topk_group, normalize, scale):
    """fp64 numpy/scipy reference of the variant (for well-separated inputs)."""
    S, E = logits.shape
    s = expit(logits.astype(np.float64))
    c = s + (0.0 if bias is None else bias.astype(np.float64))
    idx = np.empty((S, K), np.int64)
    for t in range(S):
        allowed = np.ones(E, bool)
        if n_group > 1:
            g = c[t].reshape(n_group, -1)
            top2 = -np.sort(-g, axis=1)[:, :2].sum(axis=1)
            order = np.lexsort((np.arange(n_group), -top2))
            keep = np.zeros(n_group, bool)
            keep[order[:topk_group]] = True
            allowed = np.repeat(keep, E // n_group)
        cand = np.where(allowed, c[t], -np.inf)
        idx[t] = np.lexsort((np.arange(E), -cand))[:K]
    w = np.take_along_axis(s, idx, axis=1)
    if normalize:
        w = w / w.sum(axis=1, keepdims=True)
    return idx, w * scale


def _grid_logits(rng, S, E):
    # distinct values on a grid of 0.003 (scores differ by far more than fp32 rounding)
    base = (np.arange(E) - E / 2) * 0.003
    return np.stack([rng.permutation(base) for _ in range(S)]).astype(np.float32)


@pytest.mark.parametrize("E,K,n_group,topk_group,use_bias,normalize,scale", [
    (256, 8, 8, 4, True, True, 2.5),     # DeepSeek-V3-shaped
    (64, 6, 4, 2, True, False, 1.0),
    (96, 8, 1, 1, False, True, 1.0),
    (40, 4, 8, 3, True, True, 0.5),      # groups of 5
    (32, 32, 1, 1, True, True, 1.0),     # K = E
])
def test_variant_matches_fp64_reference(oracle_lib, E, K, n_group, topk_group, use_bias, normalize, scale):
    rng = np.random.default_rng(E + K)
    logits = _grid_logits(rng, 60, E)
    # bias on a coarser grid, so c keeps distinct, well separated values
    bias = (rng.permutation(E) * 0.0101).astype(np.float32) if use_bias else None
    idx, w = oracle_lib.route_sigmoid_grouped(logits, K, bias, n_group, topk_group, normalize, scale)
    ridx, rw = _reference(logits, K, bias, n_group, topk_group, normalize, scale)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=4 * 2.0 ** -24 * (K + 4), atol=0)
    if normalize:
        np.testing.assert_allclose(w.astype(np.float64).sum(axis=1), scale, rtol=(K + 2) * 2.0 ** -24)


def test_variant_ties_and_plain_case(oracle_lib):
    logits = np.array([[0.0, 1.0, 1.0, 0.0, 2.0, 2.0, -1.0, 1.0]], np.float32)
    # no bias, one group: experts 4, 5 (tie -> lower first), then 1, 2, 7 (tie)
    idx, _ = oracle_lib.route_sigmoid_grouped(logits, 4, None, 1, 1, True, 1.0)
    assert idx[0].tolist() == [4, 5, 1, 2]
    # two groups of 4 with equal group scores (1+1 vs 2+2 -> group 1 wins; then equal -> lower)
    idx, _ = oracle_lib.route_sigmoid_grouped(logits, 2, None, 2, 1, True, 1.0)
    assert idx[0].tolist() == [4, 5]
    eq = np.array([[1.0, 1.0, 0.0, 0.0, 1.0, 1.0, 0.0, 0.0]], np.float32)
    idx, _ = oracle_lib.route_sigmoid_grouped(eq, 2, None, 2, 1, True, 1.0)
    assert idx[0].tolist() == [0, 1]
    # with no bias and no groups the selected experts are those of the softmax router
    rng = np.random.default_rng(5)
    lg = _grid_logits(rng, 40, 64)
    a, _ = oracle_lib.route_sigmoid_grouped(lg, 8, None, 1, 1, True, 1.0)
    b, _ = oracle_lib.route_topk(lg, 8)
    np.testing.assert_array_equal(a, b)


def test_variant_rejects_bad_groups(oracle_lib):
    lg = np.zeros((2, 12), np.float32)
    for args in ((4, None, 5, 1), (8, None, 4, 2), (2, None, 12, 1)):  # E%g, too few kept, group of 1
        with pytest.raises(oracle_lib.OracleError):
            oracle_lib.route_sigmoid_grouped(lg, *args)
