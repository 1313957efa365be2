"""GPU parity of the router variant (sigmoid scores, selection-only bias,
group-limited top-K) against the oracle.

Both sides compute every score with the same fp32 IEEE operations in the same
order (the exp routine is built from basic operations, not a library call), so
selected experts AND weights are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import synth

pytestmark = pytest.mark.gpu


def _run(logits, K, bias, n_group, topk_group, normalize, scale):
    lg = torch.from_numpy(logits).cuda()
    b = None if bias is None else torch.from_numpy(bias).cuda()
    idx, w = B.moe_route_sigmoid_grouped(lg, K, bias=b, n_group=n_group, topk_group=topk_group,
                                         normalize=normalize, scale=scale)
    return idx.cpu().numpy(), w.cpu().numpy()


def _check(logits, K, bias, n_group, topk_group, normalize, scale):
    ridx, rw = oracle.route_sigmoid_grouped(logits, K, bias, n_group, topk_group, normalize, scale)
    idx, w = _run(logits, K, bias, n_group, topk_group, normalize, scale)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_array_equal(w.view(np.uint32), rw.view(np.uint32))
    return idx, w


CASES = [
    # S, E, K, n_group, topk_group, bias, normalize, scale
    (4096, 256, 8, 8, 4, True, True, 2.5),       # DeepSeek-V3-shaped, prefill batch
    (777, 40, 4, 8, 3, True, True, 0.5),         # groups of 5, ragged lanes and token count
    (300, 1024, 32, 32, 8, True, True, 1.0),     # largest E and K
    (513, 96, 8, 1, 1, False, False, 1.0),       # one group, no bias, unnormalised
    (129, 33, 5, 1, 1, True, True, 1.0),         # E not a multiple of 32
    (64, 64, 6, 4, 2, True, False, 1.5),
    (3, 32, 32, 1, 1, True, True, 1.0),          # K = E
    (100, 256, 8, 32, 4, True, True, 1.0),       # groups of 8, 32 groups
]


@pytest.mark.parametrize("S,E,K,n_group,topk_group,use_bias,normalize,scale", CASES)
def test_variant_bit_exact(S, E, K, n_group, topk_group, use_bias, normalize, scale):
    rng = np.random.default_rng(S * 7 + E)
    logits = (rng.standard_normal((S, E)) * 2.0).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.05).astype(np.float32) if use_bias else None
    _check(logits, K, bias, n_group, topk_group, normalize, scale)


def test_variant_ties():
    # integer logits and a zero bias: heavy ties in the scores and in the group scores
    rng = np.random.default_rng(11)
    logits = rng.integers(-2, 3, (500, 256)).astype(np.float32)
    bias = np.zeros(256, np.float32)
    _check(logits, 8, bias, 8, 4, True, 1.0)
    _check(logits, 8, None, 1, 1, True, 1.0)
    const = np.zeros((5, 64), np.float32)
    idx, w = _check(const, 4, None, 4, 2, True, 1.0)
    assert idx.tolist() == [[0, 1, 2, 3]] * 5
    assert np.all(w == 0.25)


def test_variant_extreme_logits():
    # scores that saturate at 0 and 1, and exp overflow / underflow paths
    logits = np.array([[-200.0, -104.5, -90.0, -87.5, 0.0, 87.5, 89.0, 200.0] * 4], np.float32)
    _check(logits, 8, None, 4, 2, True, 1.0)
    _check(logits, 8, None, 1, 1, False, 3.0)


def test_variant_selection_matches_softmax_router():
    w = synth.WORKLOADS["4"]
    logits = synth.logits(w)
    idx, _ = _run(logits, w.K, None, 1, 1, True, 1.0)
    lg = torch.from_numpy(logits).cuda()
    idx2, _ = B.moe_route_topk(lg, w.K)
    # the sigmoid is monotone, so without bias and groups the same experts win -- except where
    # two distinct logits round to the same fp32 sigmoid, and there the lower id wins on both
    # sides only if it also had the larger logit: compare the multisets of scores instead
    sg = torch.sigmoid(lg.double())
    a = torch.gather(sg, 1, torch.from_numpy(idx).long().cuda())
    b = torch.gather(sg, 1, idx2.long())
    assert torch.allclose(a.sort(1).values, b.sort(1).values, rtol=1e-6, atol=0)


def test_variant_empty_and_bad_args():
    lg = torch.zeros((0, 64), dtype=torch.float32, device="cuda")
    idx, w = B.moe_route_sigmoid_grouped(lg, 4, n_group=4, topk_group=2)
    assert idx.shape == (0, 4)
    lg = torch.zeros((4, 12), dtype=torch.float32, device="cuda")
    for kw in (dict(n_group=5), dict(n_group=4, topk_group=2, K=8), dict(n_group=12),
               dict(n_group=4, topk_group=5), dict(n_group=64)):
        K = kw.pop("K", 4)
        with pytest.raises(B.MoeError):
            B.moe_route_sigmoid_grouped(lg, K, **kw)


@pytest.mark.parametrize("E,K,n_group,topk_group,use_bias,normalize,scale", [
    (256, 8, 8, 4, True, True, 2.5),     # DeepSeek-V3-shaped
    (64, 6, 4, 2, True, False, 1.0),
    (96, 8, 1, 1, False, True, 1.0),
    (40, 4, 8, 3, True, True, 0.5),      # groups of 5
    (1024, 32, 32, 8, True, True, 1.0),  # largest E and K
])
def test_kernel_matches_fp64_reference(E, K, n_group, topk_group, use_bias, normalize, scale):
    """The kernel against a reference that shares nothing with the oracle's exp:
    scipy's fp64 sigmoid and library sorts with group masking, on logits spaced
    far wider than fp32 rounding (so both precisions agree on every order).
    Experts must be identical; weights within 4 fp32 ulp per term of the
    normalising sum, (K + 4) * 4 * 2^-24 relative."""
    from .test_oracle_route_variant import _grid_logits, _reference

    rng = np.random.default_rng(E + K + 1)
    logits = _grid_logits(rng, 200, E)
    bias = (rng.permutation(E) * 0.0101).astype(np.float32) if use_bias else None
    idx, w = _run(logits, K, bias, n_group, topk_group, normalize, scale)
    ridx, rw = _reference(logits, K, bias, n_group, topk_group, normalize, scale)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=4 * 2.0 ** -24 * (K + 4), atol=0)
