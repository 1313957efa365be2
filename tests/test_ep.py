"""Expert parallelism over W ranks, host side (CPU, no GPU).

The receive plan (moe_ep_plan, C) and the segment exchange (ep.exchange over
torch.distributed, ep.exchange_local in one process) are checked against the
oracle's single-GPU layout, dispatch and combine over the whole batch: each
rank routes and lays out only its own tokens, yet after the exchange every
rank must hold exactly its part of the single-GPU dispatched buffer, every
pair's place must be its single-GPU slot, and the combine on each rank must
give the single-GPU outputs of its tokens, bit for bit.  The multi-process
case runs W = 2 and W = 4 gloo ranks on CPU tensors.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from combine_moe_route_09_b200 import binding as B
from combine_moe_route_09_b200 import ep, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _splits(S, W, uneven):
    if not uneven:
        return [S * r // W for r in range(W + 1)]
    rng = np.random.default_rng(S + W)
    cuts = np.sort(rng.choice(np.arange(1, S), W - 1, replace=False))
    return [0, *cuts.tolist(), S]


def _case(S, H, E, K, W, P, quant, seed, uneven=False):
    w = synth.Workload(f"ep_{S}_{E}_{W}", S, H, E, K, W, P, "bf16", quant, True, bias="normal", seed=seed)
    inp = dict(logits=synth.logits(w), x=synth.activations(w), y=synth.expert_outputs(w),
               shared=synth.shared_out(w), residual=synth.residual(w))
    q = oracle.QUANT_FP8_E4M3_B128 if quant == "fp8" else oracle.QUANT_NONE
    idx, wt = oracle.route_topk(inp["logits"], K)
    glob = oracle.layout(idx, E, W, P)
    xd, xs = oracle.dispatch(inp["x"], glob["slot_of"], glob["cap"], quant=q)
    out, rnr = oracle.combine(inp["y"], glob["slot_of"], wt, inp["shared"], inp["residual"])
    bounds = _splits(S, W, uneven)
    ranks = []
    for r in range(W):
        a, b = bounds[r], bounds[r + 1]
        li, lw = oracle.route_topk(inp["logits"][a:b], K)
        lay = oracle.layout(li, E, W, 0)
        sxd, sxs = oracle.dispatch(inp["x"][a:b], lay["slot_of"], lay["cap"], quant=q)
        ranks.append(dict(a=a, b=b, idx=li, w=lw, lay=lay, send_xd=sxd, send_xs=sxs))
    return w, inp, dict(idx=idx, w=wt, lay=glob, xd=xd, xs=xs, out=out, rnr=rnr), ranks


CASES = [  # S, H, E, K, W, P, quant, uneven
    (96, 256, 16, 4, 2, 0, "fp8", False),
    (130, 128, 24, 3, 4, 8, "none", True),
    (200, 256, 64, 8, 8, 16, "fp8", False),
    (64, 128, 8, 2, 1, 4, "none", False),
    (257, 128, 12, 3, 3, 5, "none", True),
]


@pytest.mark.parametrize("S,H,E,K,W,P,q,uneven", CASES)
def test_plan_and_local_exchange_reproduce_the_single_gpu_pass(S, H, E, K, W, P, q, uneven):
    w, inp, ref, ranks = _case(S, H, E, K, W, P, q, seed=S + 7 * W, uneven=uneven)
    counts = np.stack([r["lay"]["counts"] for r in ranks])
    plan = ep.ep_plan(counts, P)
    # the plan is the single-GPU layout's bookkeeping
    np.testing.assert_array_equal(plan.expert_offsets, ref["lay"]["offsets"])
    for d in range(W):
        lo, hi = d * plan.Eloc, (d + 1) * plan.Eloc
        assert plan.recv_rows[d] == ref["lay"]["offsets"][hi] - ref["lay"]["offsets"][lo]
    for s, r in enumerate(ranks):
        np.testing.assert_array_equal(ep.global_slots(plan, s, r["lay"]["slot_of"]),
                                      ref["lay"]["slot_of"][r["a"]:r["b"]])
    # rows moved segment by segment land exactly where the single-GPU dispatch puts them
    fp8 = q == "fp8"
    send = [[torch.from_numpy(r["send_xd"])] + ([torch.from_numpy(r["send_xs"])] if fp8 else []) for r in ranks]
    recv = []
    for d in range(W):
        n = int(plan.recv_rows[d])
        bufs = [torch.full((n, H), 0x5A if fp8 else 0x7FFF, dtype=torch.uint8 if fp8 else torch.int16)]
        if fp8:
            bufs.append(torch.full((n, H // 128), -7.0))
        recv.append(bufs)
    if not fp8:
        send = [[t[0].view(torch.int16)] for t in send]
    ep.exchange_local(plan, send, recv)
    xd_cat = torch.cat([b[0] for b in recv]).numpy()
    rows = int(plan.expert_offsets[-1])  # the receive buffers cover the layout, not the spare capacity past it
    assert xd_cat.shape[0] == rows
    valid = ref["lay"]["row_src"][:rows] >= 0
    ref_xd = (ref["xd"] if fp8 else ref["xd"].view(np.int16))[:rows]
    np.testing.assert_array_equal(xd_cat[valid], ref_xd[valid])
    if fp8:
        np.testing.assert_array_equal(torch.cat([b[1] for b in recv]).numpy()[valid], ref["xs"][:rows][valid])
    # the combine direction: expert outputs back to each source rank, combined there
    y = inp["y"]
    y_recv = [[torch.from_numpy(y[plan.rank_base(d):plan.rank_base(d) + int(plan.recv_rows[d])].copy())]
              for d in range(W)]
    y_send = [[torch.empty((r["lay"]["cap"], H), dtype=torch.int16)] for r in ranks]
    ep.exchange_local(plan, [[t[0].view(torch.int16)] for t in y_recv], y_send, reverse=True)
    for r, ys in zip(ranks, y_send):
        o, n = oracle.combine(ys[0].numpy().view(np.uint16), r["lay"]["slot_of"], r["w"],
                              inp["shared"][r["a"]:r["b"]], inp["residual"][r["a"]:r["b"]])
        np.testing.assert_array_equal(o, ref["out"][r["a"]:r["b"]])
        np.testing.assert_array_equal(n, ref["rnr"][r["a"]:r["b"]])


def test_plan_rejects_bad_arguments():
    ok = np.zeros((2, 8), np.int32)
    with pytest.raises(B.MoeError):
        ep.ep_plan(np.zeros((3, 8), np.int32))  # E % W != 0
    with pytest.raises(B.MoeError):
        ep.ep_plan(ok, -1)
    bad = ok.copy()
    bad[1, 3] = -2
    with pytest.raises(B.MoeError):
        ep.ep_plan(bad)
    plan = ep.ep_plan(ok, 128)  # all empty: zero rows everywhere
    assert plan.expert_offsets.tolist() == [0] * 9 and plan.recv_rows.tolist() == [0, 0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, q):
    import datetime
    import sys

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle as orc
        from combine_moe_route_09_b200 import ep as E_

        S, H, E, K, W, P, quant, uneven = case
        w, inp, ref, ranks = _case(S, H, E, K, W, P, quant, seed=S + 11 * W, uneven=uneven)
        me = ranks[rank]
        fp8 = quant == "fp8"
        # exchange the counts as the GPU path does (an all-gather), then plan
        mine = torch.from_numpy(me["lay"]["counts"].copy())
        got = [torch.empty_like(mine) for _ in range(W)]
        dist.all_gather(got, mine)
        plan = E_.ep_plan(torch.stack(got).numpy(), P)
        send = [torch.from_numpy(me["send_xd"]) if fp8 else torch.from_numpy(me["send_xd"]).view(torch.int16)]
        if fp8:
            send.append(torch.from_numpy(me["send_xs"]))
        n = int(plan.recv_rows[rank])
        recv = [torch.zeros((n, H), dtype=send[0].dtype)] + ([torch.zeros((n, H // 128))] if fp8 else [])
        E_.exchange(plan, rank, send, recv)
        base = plan.rank_base(rank)
        valid = ref["lay"]["row_src"][base:base + n] >= 0
        ref_xd = ref["xd"][base:base + n]
        ok_xd = np.array_equal(recv[0].numpy()[valid], (ref_xd if fp8 else ref_xd.view(np.int16))[valid])
        ok_xs = (not fp8) or np.array_equal(recv[1].numpy()[valid], ref["xs"][base:base + n][valid])
        y_recv = torch.from_numpy(inp["y"][base:base + n].copy()).view(torch.int16)
        y_send = torch.empty((me["lay"]["cap"], H), dtype=torch.int16)
        E_.exchange(plan, rank, [y_recv], [y_send], reverse=True)
        o, r2 = orc.combine(y_send.numpy().view(np.uint16), me["lay"]["slot_of"], me["w"],
                            inp["shared"][me["a"]:me["b"]], inp["residual"][me["a"]:me["b"]])
        ok_c = np.array_equal(o, ref["out"][me["a"]:me["b"]]) and np.array_equal(r2, ref["rnr"][me["a"]:me["b"]])
        q.put((rank, bool(ok_xd), bool(ok_xs), bool(ok_c)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [(160, 256, 16, 4, 2, 8, "fp8", False), (150, 128, 16, 3, 4, 4, "none", True)])
def test_gloo_ranks_reproduce_the_single_gpu_pass(case):
    W = case[4]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, W, port, case, q)) for r in range(W)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(W))
    assert res == [(r, True, True, True) for r in range(W)], res
