"""GPU parity of the routing weights in dispatched order against the oracle
(bit-exact: the kernel only moves fp32 values)."""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["1", "2", "4", "5"])
def test_route_weights_match_oracle(name):
    w = synth.WORKLOADS[name]
    idx, wt = oracle.route_topk(synth.logits(w), w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    ref = oracle.route_weights_dispatched(wt, lay["slot_of"], lay["cap"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((lay["cap"],), float("nan"), dtype=torch.float32, device="cuda")
    B.moe_dispatch_route_weights(torch.from_numpy(wt).cuda(), torch.from_numpy(lay["row_src"]).cuda(), out=out,
                                 status=status)
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert status.item() == 0


def test_route_weights_bad_rows_and_empty():
    wt = np.arange(1, 7, dtype=np.float32).reshape(3, 2)
    row_src = np.array([5, -1, 0, 6, 100, 3, -1], np.int32)       # 6 and 100 >= S*K = 6
    slot_of = np.full((3, 2), -1, np.int32)
    for r, s in enumerate(row_src):
        if 0 <= s < 6:
            slot_of.reshape(-1)[s] = r
    ref = oracle.route_weights_dispatched(wt, slot_of, len(row_src))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = B.moe_dispatch_route_weights(torch.from_numpy(wt).cuda(), torch.from_numpy(row_src).cuda(),
                                       status=status)
    np.testing.assert_array_equal(out.cpu().numpy(), ref)
    assert status.item() == B.MOE_STATUS_BAD_SLOT
    empty = B.moe_dispatch_route_weights(torch.from_numpy(wt).cuda(), torch.zeros(0, dtype=torch.int32,
                                                                                  device="cuda"))
    assert empty.shape == (0,)
