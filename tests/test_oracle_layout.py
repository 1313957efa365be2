"""Pins for the oracle's dispatch layout (CPU only).

Checked against: a hand-worked case (tests/golden/layout_worked.txt); a
construction by a different algorithm (numpy's stable argsort of the flat
expert ids, instead of the oracle's counting pass); and the invariants the
pages fix (counts sum to S*K, padding to multiples of token_padding, capacity
bound, expert blocks per rank, slot_of/row_src mutual inverses).
"""
import os

import numpy as np
import pytest

from combine_moe_route_09_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden():
    d = {}
    with open(os.path.join(GOLDEN, "layout_worked.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            d[k.strip()] = [int(x) for x in v.split()]
    return d


def test_layout_golden(oracle_lib):
    g = _read_golden()
    S, E, K, R, P, cap = g["S E K R P cap"]
    idx = np.array(g["topk_idx"], np.int32).reshape(S, K)
    lay = oracle_lib.layout(idx, E, R, P, cap)
    assert lay["counts"].tolist() == g["counts"]
    assert lay["offsets"].tolist() == g["offsets"]
    assert lay["rank_offsets"].tolist() == g["rank_offsets"]
    assert lay["slot_of"].reshape(-1).tolist() == g["slot_of"]
    assert lay["row_src"].tolist() == g["row_src"]


def _argsort_layout(idx, E, P):
    """The same layout built a different way: a stable sort of pairs by expert."""
    flat = idx.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    padded = counts if P == 0 else -(-counts // P) * P
    offsets = np.concatenate([[0], np.cumsum(padded)])
    starts = np.concatenate([[0], np.cumsum(counts)])
    slot = np.empty_like(flat)
    for e in range(E):
        members = order[starts[e]:starts[e + 1]]
        slot[members] = offsets[e] + np.arange(len(members))
    return counts, offsets, slot.reshape(idx.shape)


def _random_topk(rng, S, E, K):
    # distinct experts per token, like a real top-K
    return np.stack([rng.permutation(E)[:K] for _ in range(S)]).astype(np.int32) if S else \
        np.zeros((0, K), np.int32)


@pytest.mark.parametrize("S,E,K,R,P,seed", [
    (1, 1, 1, 1, 0, 0), (3, 4, 2, 2, 0, 1), (8, 8, 2, 2, 4, 2), (100, 16, 4, 4, 128, 3),
    (257, 64, 8, 8, 128, 4), (50, 384, 8, 4, 128, 5), (31, 12, 12, 3, 5, 6), (0, 8, 2, 2, 4, 7)])
def test_layout_matches_stable_sort(oracle_lib, S, E, K, R, P, seed):
    rng = np.random.default_rng(seed)
    idx = _random_topk(rng, S, E, K)
    lay = oracle_lib.layout(idx, E, R, P)
    counts, offsets, slot = _argsort_layout(idx, E, P)
    np.testing.assert_array_equal(lay["counts"], counts)
    np.testing.assert_array_equal(lay["offsets"], offsets)
    np.testing.assert_array_equal(lay["slot_of"], slot)


def check_layout_invariants(idx, E, R, P, lay):
    """Properties every correct layout has, at any size."""
    S, K = idx.shape
    counts, offsets, ro = lay["counts"], lay["offsets"], lay["rank_offsets"]
    slot_of, row_src, cap = lay["slot_of"], lay["row_src"], lay["cap"]
    assert counts.sum() == S * K
    assert offsets[0] == 0 and np.all(np.diff(offsets) >= 0)
    pc = np.diff(offsets)
    assert np.all(pc >= counts)
    if P > 0:
        assert np.all(pc % P == 0) and np.all(pc - counts < P)
    else:
        assert np.all(pc == counts)
    assert offsets[E] <= cap
    Eloc = E // R
    np.testing.assert_array_equal(ro, offsets[np.arange(R + 1) * Eloc])
    flat = slot_of.reshape(-1)
    e_of = idx.reshape(-1)
    # each slot inside its expert's segment, distinct, and the inverse of row_src
    assert np.all(flat >= offsets[e_of]) and np.all(flat < offsets[e_of] + counts[e_of])
    assert len(np.unique(flat)) == flat.size
    np.testing.assert_array_equal(row_src[flat], np.arange(flat.size))
    assert np.count_nonzero(row_src >= 0) == flat.size
    # inside each expert segment the source pairs ascend
    for e in range(E):
        seg = row_src[offsets[e]:offsets[e] + counts[e]]
        assert np.all(np.diff(seg) > 0)


@pytest.mark.parametrize("name", ["1", "2", "2b", "3", "4", "5"])
def test_layout_invariants_on_workloads(oracle_lib, name):
    w = synth.WORKLOADS[name]
    idx, _ = oracle_lib.route_topk(synth.logits(w), w.K)
    lay = oracle_lib.layout(idx, w.E, w.R, w.P)
    assert lay["cap"] == w.cap
    check_layout_invariants(idx, w.E, w.R, w.P, lay)


def test_imbalanced_workload_load_ratio(oracle_lib):
    w = synth.WORKLOADS["5"]
    idx, _ = oracle_lib.route_topk(synth.logits(w), w.K)
    c = oracle_lib.layout(idx, w.E, w.R, w.P)["counts"]
    assert 3.9 <= c.max() / c.mean() <= 4.1


def test_layout_errors(oracle_lib):
    idx = np.array([[0, 1], [1, 2]], np.int32)
    with pytest.raises(oracle_lib.OracleError) as e:
        oracle_lib.layout(idx, 4, 2, 4, cap=7)  # needs 3 experts x 4 rows = 12
    assert e.value.rc == oracle_lib.EOVERFLOW
    with pytest.raises(oracle_lib.OracleError) as e:
        oracle_lib.layout(np.array([[0, 4]], np.int32), 4, 2, 0)
    assert e.value.rc == oracle_lib.EINDEX
    with pytest.raises(oracle_lib.OracleError) as e:
        oracle_lib.layout(idx, 4, 3, 0)  # E % R != 0
    assert e.value.rc == oracle_lib.EINVAL


@pytest.mark.parametrize("name,S", [("1", 128), ("2", 512), ("5", 700)])
def test_route_weights_dispatched(oracle_lib, name, S):
    """Row r of the dispatched order carries the weight of the pair row_src[r] names (read
    through row_src, the other direction of the layout); rows no pair fills carry 0; per
    expert, the rows' weights add up to the weights of the tokens routed there (bincount)."""
    w = synth.WORKLOADS[name].replace(S=S)
    idx, wt = oracle_lib.route_topk(synth.logits(w), w.K)
    lay = oracle_lib.layout(idx, w.E, w.R, w.P)
    rw = oracle_lib.route_weights_dispatched(wt, lay["slot_of"], lay["cap"])
    src = lay["row_src"]
    valid = src >= 0
    np.testing.assert_array_equal(rw[valid], wt.reshape(-1)[src[valid]])
    assert np.all(rw[~valid] == 0)
    seg = np.repeat(np.arange(w.E), np.diff(lay["offsets"]))
    per_expert = np.bincount(seg, weights=rw[:lay["offsets"][-1]].astype(np.float64), minlength=w.E)
    ref = np.bincount(idx.reshape(-1), weights=wt.reshape(-1).astype(np.float64), minlength=w.E)
    np.testing.assert_allclose(per_expert, ref, rtol=1e-12, atol=0)


def test_route_weights_dispatched_worked_example(oracle_lib):
    # 3 tokens, K = 2, hand-placed slots in a capacity of 8 (slot -1: pair dropped)
    slot_of = np.array([[4, 0], [1, -1], [7, 2]], np.int32)
    wt = np.array([[0.6, 0.4], [0.9, 0.1], [0.5, 0.5]], np.float32)
    rw = oracle_lib.route_weights_dispatched(wt, slot_of, 8)
    assert rw.tolist() == [np.float32(0.4), np.float32(0.9), 0.5, 0.0, np.float32(0.6), 0.0, 0.0, 0.5]
