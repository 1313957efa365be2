"""GPU parity of the combine over FP8 expert outputs (e4m3 codes + block scales).

The kernel dequantises (exact e4m3 decode, fp32 product with the scale) and
accumulates in the oracle's order, so outputs match within the combine
tolerance (in fact bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import synth

from .helpers import assert_act_close

pytestmark = pytest.mark.gpu


def dev(a):
    return synth.to_torch(a, device="cuda")


def host(t):
    return synth.from_torch(t)


CASES = [
    (synth.WORKLOADS["4"], True),                                       # full size, dual residual
    (synth.WORKLOADS["3"], False),                                      # decode, plain
    (synth.Workload("c8_f32", 333, 1536, 24, 5, 4, 3, "f32", "fp8", True, seed=41), True),
    (synth.Workload("c8_k32", 97, 512, 64, 32, 8, 0, "bf16", "fp8", False, seed=42), False),
    (synth.Workload("c8_k20_h2560", 150, 2560, 40, 20, 4, 7, "bf16", "fp8", True, seed=43), True),
]


@pytest.mark.parametrize("w,fused", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_combine_fp8(w, fused):
    idx, wt = oracle.route_topk(synth.logits(w), w.K)
    lay = oracle.layout(idx, w.E, w.R, w.P)
    # expert outputs in FP8: quantise a seeded N(0,1) buffer with the oracle's dispatch rule
    y = synth.expert_outputs(w)
    ident = np.arange(lay["cap"], dtype=np.int32).reshape(-1, 1)
    yq, ys = oracle.dispatch(y, ident, lay["cap"], quant=oracle.QUANT_FP8_E4M3_B128)
    sh = synth.shared_out(w) if fused else None
    rs = synth.residual(w) if fused else None
    ref, ref_n = oracle.combine_fp8(yq, ys, lay["slot_of"], wt, shared=sh, residual=rs, dtype=w.dtype)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, rnr = B.moe_combine_fp8_dual_residual(dev(yq), dev(ys), dev(lay["slot_of"]), dev(wt),
                                               shared_out=dev(sh) if fused else None,
                                               residual=dev(rs) if fused else None, dtype=dt, status=status)
    assert_act_close(host(out), ref, "residual_out")
    if fused:
        assert_act_close(host(rnr), ref_n, "residual_no_routed_out")
    assert status.item() == 0


def test_combine_fp8_rejects_h_not_multiple_of_512():
    yq = torch.zeros((16, 384), dtype=torch.uint8, device="cuda")
    ys = torch.zeros((16, 3), dtype=torch.float32, device="cuda")
    slot = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    w = torch.ones((4, 2), dtype=torch.float32, device="cuda")
    with pytest.raises(B.MoeError):
        B.moe_combine_fp8_dual_residual(yq, ys, slot, w)
