"""Expert parallelism with the CUDA kernels: W ranks emulated on one GPU.

Each emulated rank routes, lays out and dispatches only its own tokens with
the library's kernels (ep.EpRank.local_dispatch); the rows then move between
the ranks' buffers along the plan's segments (ep.exchange_local: device
copies where separate GPUs would use NCCL), and each rank combines its own
tokens.  Against the CPU oracle run over the whole batch on one GPU's layout:
every rank's receive buffer is its part of the single-GPU dispatched buffer
(bytes and FP8 scales bit-exact), every pair's whole-batch slot is the
oracle's, and each rank's combine gives the oracle's outputs for its tokens
(within 1 bf16 ulp plus the gating-weight slack, as the single-GPU tests).
No kernel waits on another rank's kernel: the exchange happens between steps.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_09_b200 import ep, synth

from .helpers import abs_weighted_sum, assert_act_close, assert_f32_close

pytestmark = pytest.mark.gpu


def dev(a):
    return synth.to_torch(a, device="cuda")


def host(t):
    return synth.from_torch(t)


CASES = [  # S, H, E, K, W, P, quant
    (4096, 7168, 256, 8, 8, 0, "fp8"),      # DeepSeek-V3-shaped prefill over 8 ranks
    (4096, 2048, 64, 8, 8, 128, "none"),    # padded bf16 rows over 8 ranks
    (1000, 512, 48, 6, 3, 16, "fp8"),       # 3 ranks, ragged token split
]


@pytest.mark.parametrize("S,H,E,K,W,P,q", CASES)
def test_emulated_ranks_reproduce_the_single_gpu_pass(S, H, E, K, W, P, q):
    w = synth.Workload(f"epg_{S}_{E}_{W}", S, H, E, K, W, P, "bf16", q, True, bias="normal", seed=S + W)
    lg, x, y = synth.logits(w), synth.activations(w), synth.expert_outputs(w)
    sh, rs = synth.shared_out(w), synth.residual(w)
    idx, wt = oracle.route_topk(lg, K)
    glob = oracle.layout(idx, E, W, P)
    oq = oracle.QUANT_FP8_E4M3_B128 if q == "fp8" else oracle.QUANT_NONE
    xd, xs = oracle.dispatch(x, glob["slot_of"], glob["cap"], quant=oq)
    out, rnr = oracle.combine(y, glob["slot_of"], wt, sh, rs)

    bounds = [S * r // W for r in range(W + 1)]
    ranks = []
    for r in range(W):
        a, b = bounds[r], bounds[r + 1]
        er = ep.EpRank(b - a, H, K, E, W, r, P, fp8=q == "fp8")
        er.local_dispatch(dev(lg[a:b]), dev(x[a:b]))
        ranks.append(er)
    torch.cuda.synchronize()
    counts = np.stack([host(er.layout.counts) for er in ranks])
    plan = ep.ep_plan(counts, P)
    for er in ranks:
        er.plan = plan
    recv = [ranks[0].new_recv(int(plan.recv_rows[d])) for d in range(W)]
    ep.exchange_local(plan, [er.send for er in ranks], recv)
    torch.cuda.synchronize()

    np.testing.assert_array_equal(plan.expert_offsets, glob["offsets"])
    rows = int(plan.expert_offsets[-1])
    valid = glob["row_src"][:rows] >= 0
    np.testing.assert_array_equal(torch.cat([b[0] for b in recv]).view(torch.uint8).cpu().numpy()[valid],
                                  xd[:rows].view(np.uint8)[valid])
    if q == "fp8":
        np.testing.assert_array_equal(host(torch.cat([b[1] for b in recv]))[valid], xs[:rows][valid])
    for r, er in enumerate(ranks):
        a, b = bounds[r], bounds[r + 1]
        np.testing.assert_array_equal(host(er.topk_idx), idx[a:b])
        assert_f32_close(host(er.topk_w), wt[a:b], 1e-5, "topk_w")
        np.testing.assert_array_equal(ep.global_slots(plan, r, host(er.layout.slot_of)), glob["slot_of"][a:b])

    # experts: y rows of the whole-batch layout, each rank holding its part; back and combined
    y_recv = [dev(y[plan.rank_base(d):plan.rank_base(d) + int(plan.recv_rows[d])]) for d in range(W)]
    y_send = [torch.empty((er.cap, H), dtype=torch.bfloat16, device="cuda") for er in ranks]
    ep.exchange_local(plan, [[t] for t in y_recv], [[t] for t in y_send], reverse=True)
    slack = 2e-5 * abs_weighted_sum(y, glob["slot_of"], wt)
    for r, er in enumerate(ranks):
        a, b = bounds[r], bounds[r + 1]
        o, n = er.local_combine(y_send[r], dev(sh[a:b]), dev(rs[a:b]))
        torch.cuda.synchronize()
        assert_act_close(host(o), out[a:b], f"rank {r} residual_out", extra_abs=slack[a:b])
        assert_act_close(host(n), rnr[a:b], f"rank {r} residual_no_routed_out")
        assert er.status.item() == 0
