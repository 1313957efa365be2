"""The allocation-free layout entry point, moe_dispatch_layout_static.

It exists for callers that may not allocate device memory where they call the
layout (a framework or plugin that owns all device memory up front, or a
latency-critical loop that cannot afford cudaMalloc's device synchronisation):
its scratch is a fixed array inside the library instead of a caller-supplied
workspace.  These tests call it through the C ABI and require outputs identical
to the CPU oracle's layout and to moe_dispatch_layout's (the layout is integer
work: bit-exact), on two calls in a row, so that leftovers of one call in the
shared array cannot change the next.  The cases cover every layout kernel:
the single-cluster one (no scratch), the cooperative one (the grid-barrier
header) and the histogram + slots pair (the arrival ticket and the per-tile
histograms, all in the shared array).  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B

pytestmark = pytest.mark.gpu

CASES = [  # S, E, K, R, token_padding, kernels moe_dispatch_layout launches
    (4096, 256, 8, 8, 0, 1),      # DeepSeek-V3-shaped prefill: one cluster, no scratch
    (16384, 64, 8, 8, 128, 1),    # imbalanced 16B-A3B-style, padded: cooperative grid
    (4099, 384, 8, 4, 128, 1),    # ragged tail, E = 384
    (3, 8, 2, 2, 4, 1),           # a few tokens
    (8192, 1024, 32, 8, 16, 2),   # 128 tiles x 1024 experts: histogram + slots kernels
    (32768, 1024, 8, 8, 0, 2),    # the same path with K = 8
]


def _routing(S, E, K, seed):
    rng = np.random.default_rng(seed)
    # skewed choice of distinct experts per token, like a biased router
    p = rng.dirichlet(np.full(E, 0.3))
    idx = np.stack([rng.choice(E, K, replace=False, p=p) for _ in range(S)]).astype(np.int32)
    return torch.from_numpy(idx).cuda()


def _assert_same(a: B.Layout, b: B.Layout):
    for k in ("counts", "offsets", "rank_offsets", "slot_of", "row_src"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k


@pytest.mark.parametrize("S,E,K,R,P,kernels", CASES)
def test_static_layout_matches_oracle_and_workspace_layout_twice(S, E, K, R, P, kernels):
    assert B.moe_dispatch_layout_workspace(S, E, K) <= B.MOE_STATIC_LAYOUT_SCRATCH_BYTES
    assert B.moe_dispatch_layout_kernels(S, E, K) == kernels
    idx = _routing(S, E, K, seed=S + E)
    ref_o = oracle.layout(idx.cpu().numpy(), E, R, P)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = B.moe_dispatch_layout(idx, E, R, P, status=status)
    for _ in range(2):
        got = B.moe_dispatch_layout_static(idx, E, R, P, status=status)
        torch.cuda.synchronize()
        _assert_same(got, ref)
        for k in ("counts", "offsets", "rank_offsets", "slot_of", "row_src"):
            np.testing.assert_array_equal(getattr(got, k).cpu().numpy(), ref_o[k], err_msg=k)
    assert status.item() == 0


def test_static_layout_second_call_with_other_routing():
    # Two calls in a row with different inputs: the second must not see the first's scratch.
    S, E, K, R, P = 2048, 128, 8, 4, 16
    a, b = _routing(S, E, K, 1), _routing(S, E, K, 2)
    for idx in (a, b, a):
        got = B.moe_dispatch_layout_static(idx, E, R, P)
        ref = B.moe_dispatch_layout(idx, E, R, P)
        torch.cuda.synchronize()
        _assert_same(got, ref)


def test_static_layout_refuses_sizes_beyond_its_scratch():
    S, E, K = 20000, 1024, 32  # needs ~1.3 MB of scratch, more than the 1 MiB built in
    assert B.moe_dispatch_layout_workspace(S, E, K) > B.MOE_STATIC_LAYOUT_SCRATCH_BYTES
    idx = torch.zeros((S, K), dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_dispatch_layout_static(idx, E, 8, 0)
    assert e.value.rc == B.MOE_ERR_SCRATCH_TOO_SMALL
    assert "scratch" in str(e.value)
