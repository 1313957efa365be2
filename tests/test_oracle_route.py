"""Pins for the oracle's router top-K gating (CPU only).

Selection is checked against a library sort (numpy lexsort on (-logit, id))
and hand-worked tie cases; the weights against the full softmax over all E
experts renormalised over the chosen K (scipy, fp64), which is a different
formula for the same quantity, plus the closed-form facts sum(w) = 1 and w
non-increasing in k.
"""
import os

import numpy as np
import pytest
from scipy.special import softmax

from combine_moe_route_09_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sorted_topk(logits, K):
    # Library sort: primary key -logit (so larger first), secondary key expert id.
    S, E = logits.shape
    out = np.empty((S, K), np.int64)
    ids = np.arange(E)
    for t in range(S):
        row = logits[t].astype(np.float64) + 0.0  # -0.0 -> +0.0 so both compare equal
        order = np.lexsort((ids, -row))
        out[t] = order[:K]
    return out


@pytest.mark.parametrize("S,E,K,seed", [(1, 1, 1, 0), (7, 5, 3, 1), (16, 8, 8, 2), (64, 384, 8, 3),
                                        (33, 256, 8, 4), (20, 64, 32, 5), (5, 1024, 1, 6)])
def test_topk_matches_library_sort(oracle_lib, S, E, K, seed):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((S, E)).astype(np.float32)
    idx, w = oracle_lib.route_topk(logits, K)
    np.testing.assert_array_equal(idx, _sorted_topk(logits, K))


def test_topk_with_many_ties_matches_library_sort(oracle_lib):
    rng = np.random.default_rng(11)
    # Values drawn from a tiny set so that ties are everywhere, zeros of both signs included.
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 0.5, 2.0], np.float32)
    logits = vals[rng.integers(0, len(vals), size=(200, 12))]
    for K in (1, 3, 12):
        idx, _ = oracle_lib.route_topk(logits, K)
        np.testing.assert_array_equal(idx, _sorted_topk(logits, K))


def test_topk_golden_ties(oracle_lib):
    with open(os.path.join(GOLDEN, "topk_ties.txt")) as f:
        rows = [l for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 5
    for line in rows:
        k, lg, exp = (p.strip() for p in line.split("|"))
        logits = np.array([[float(v) for v in lg.split()]], np.float32)
        idx, w = oracle_lib.route_topk(logits, int(k))
        assert idx[0].tolist() == [int(v) for v in exp.split()], line


@pytest.mark.parametrize("name", ["1", "2", "3", "4", "5"])
def test_weights_equal_renormalised_full_softmax(oracle_lib, name):
    w = synth.WORKLOADS[name]
    logits = synth.logits(w)
    sub = slice(0, 512)
    idx, wt = oracle_lib.route_topk(logits[sub], w.K)
    p = softmax(logits[sub].astype(np.float64), axis=1)          # full softmax over E
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    ref = sel / sel.sum(axis=1, keepdims=True)                   # renormalised over the chosen K
    np.testing.assert_allclose(wt, ref, rtol=1e-6, atol=0)
    # closed-form facts
    np.testing.assert_allclose(wt.astype(np.float64).sum(axis=1), 1.0, rtol=0, atol=2e-6)
    assert np.all(np.diff(wt, axis=1) <= 0)
    assert np.all(wt > 0)


def test_k_equals_e_is_a_full_sort(oracle_lib):
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((10, 16)).astype(np.float32)
    idx, w = oracle_lib.route_topk(logits, 16)
    for t in range(10):
        assert sorted(idx[t].tolist()) == list(range(16))
        assert np.all(np.diff(logits[t][idx[t]]) <= 0)
    # K = E: the weights are the full softmax
    np.testing.assert_allclose(w, np.take_along_axis(softmax(logits.astype(np.float64), axis=1),
                                                     idx.astype(np.int64), axis=1), rtol=1e-6)


def test_k1_weight_is_one(oracle_lib):
    logits = np.random.default_rng(0).standard_normal((50, 9)).astype(np.float32)
    idx, w = oracle_lib.route_topk(logits, 1)
    assert np.all(w == 1.0)
    np.testing.assert_array_equal(idx[:, 0], np.argmax(logits, axis=1))


def test_route_rejects_bad_k(oracle_lib):
    logits = np.zeros((2, 4), np.float32)
    with pytest.raises(oracle_lib.OracleError):
        oracle_lib.route_topk(logits, 5)
    with pytest.raises(oracle_lib.OracleError):
        oracle_lib.route_topk(logits, 0)
