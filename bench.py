#!/usr/bin/env python
"""Benchmark of one MoE routing pass per step on B200.

A step is the whole hot path over one batch: router top-K gating, the padded
expert layout (histogram + scan), the dispatch scatter (FP8 e4m3 with
128-channel scales for the default workload) and the combine with the FarSkip
dual-residual epilogue, all through the C ABI on one stream.  The expert GEMMs
are not part of the path: their outputs y are a resident synthetic buffer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 4] [--impl ours|reference]

Prints ONE JSON line on rank 0.  Default workload: the DeepSeek-V3-shaped
prefill (S=4096 tokens, H=7168, E=256, K=8, R=8, FP8 dispatch, dual-residual
combine).  Its per-step working set (~1.5 GB) is far larger than L2, so no
L2 flush is needed between steps.  With N > 1 (torchrun) each rank runs an
independent replica on its own GPU (no data-path collective); timing is the
max over ranks.

--impl reference times the CPU oracle (test infrastructure, plain C,
single-threaded) on this machine's host cores over a bounded sample of the
same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dispatch+combine tokens/s and effective HBM GB/s (% of B200 peak), 1 GPU"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------------------------
# workload accounting
# ----------------------------------------------------------------------------------------------

def algorithmic_bytes(w) -> dict:
    """Bytes each step must move at least (padding rows and dense E-wide work excluded)."""
    b = w.esize
    bout = 1 if w.quant == "fp8" else b
    S, H, E, K = w.S, w.H, w.E, w.K
    route = S * E * 4 + S * K * 8
    layout = S * K * 4 * 3 + E * 8
    dispatch = S * H * b + S * K * H * bout + S * K * 4
    if w.quant == "fp8":
        dispatch += S * K * (H // 128) * 4
    combine = S * K * H * b + S * K * 8 + (4 * S * H * b if w.fused else S * H * b)
    return dict(route=route, layout=layout, dispatch=dispatch, combine=combine,
                route_dispatch=route + layout + dispatch)


def workload_config(w, world: int) -> dict:
    return {
        "workload": w.name, "tokens_per_gpu": w.S, "S": w.S, "H": w.H, "E": w.E, "K": w.K,
        "R_logical_ranks": w.R, "token_padding": w.P,
        "activations": w.dtype, "dispatch": "fp8_e4m3_block128" if w.quant == "fp8" else w.dtype,
        "combine": "dual_residual" if w.fused else "plain", "accumulate": "fp32",
        "global_batch": w.S * world, "parallelism": f"replicas x{world}",
        "l2": "no flush: per-step working set >> 126 MB L2",
    }


def read_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged.

    A summary under profiles/ carries lines 'kernel_source_sha256: <hex>',
    'workload: <name>' and 'dram_bytes_per_launch: <int>'."""
    src = os.path.join(ROOT, "combine_moe_route_09_b200", "csrc", kernel_file)
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith((".md", ".txt")):
            continue
        kv = {}
        for line in open(os.path.join(pdir, fn)):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip().strip("-* `")] = v.strip().strip("`")
        if kv.get("kernel_source_sha256") == sha and kv.get("workload") == workload \
                and "dram_bytes_per_launch" in kv:
            try:
                return int(kv["dram_bytes_per_launch"])
            except ValueError:
                return None
    return None


# ----------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ----------------------------------------------------------------------------------------------

_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.005):
        self.idx, self.period = device_index, period_s
        self.samples, self.reasons, self.max_mhz, self.err = [], 0, None, None
        self._stop = threading.Event()
        self._t = None

    def _poll(self, nv, h):
        self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)

    def _run(self):
        try:
            import pynvml as nv

            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.idx)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._poll(nv, h)
            while not self._stop.wait(self.period):
                self._poll(nv, h)
            self._poll(nv, h)
            nv.nvmlShutdown()
        except Exception as e:  # clocks are reported as unavailable, the run goes on
            self.err = repr(e)

    def start(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        time.sleep(0.02)

    def stop(self) -> dict:
        self._stop.set()
        self._t.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "error": self.err}
        names = [n for bit, n in _REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------------------------------------
# CPU oracle baseline (test infrastructure; this leg alone may run it)
# ----------------------------------------------------------------------------------------------

def oracle_pass(w, inp: dict, S: int, threads: int = 1):
    """One routing pass of the first S tokens through the oracle.

    With threads > 1 the per-token steps (route, dispatch, combine) are split
    over contiguous token ranges, one range per thread (the oracle's C calls
    release the GIL); the layout, a global counting sort, runs once."""
    import numpy as np

    import oracle

    lg = inp["logits"][:S]
    bounds = [S * i // threads for i in range(threads + 1)]
    ranges = [(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
    q = oracle.QUANT_FP8_E4M3_B128 if w.quant == "fp8" else oracle.QUANT_NONE

    def par(fn):
        if len(ranges) == 1:
            return [fn(*ranges[0])]
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=len(ranges)) as ex:
            return list(ex.map(lambda r: fn(*r), ranges))

    parts = par(lambda a, b: oracle.route_topk(lg[a:b], w.K))
    idx = np.concatenate([p[0] for p in parts])
    wt = np.concatenate([p[1] for p in parts])
    lay = oracle.layout(idx, w.E, w.R, w.P)
    cap, H = lay["cap"], w.H
    x = inp["x"][:S]
    if q == oracle.QUANT_FP8_E4M3_B128:
        xd, xs = np.zeros((cap, H), np.uint8), np.zeros((cap, H // 128), np.float32)
    else:
        xd, xs = np.zeros((cap, H), x.dtype), None
    par(lambda a, b: oracle.dispatch(x[a:b], lay["slot_of"][a:b], cap, quant=q, xd=xd, xs=xs))
    y = inp["y"][:cap]
    sh = inp["shared"][:S] if w.fused else None
    rs = inp["residual"][:S] if w.fused else None
    outs = par(lambda a, b: oracle.combine(y, lay["slot_of"][a:b], wt[a:b], None if sh is None else sh[a:b],
                                           None if rs is None else rs[a:b]))
    out = np.concatenate([o[0] for o in outs])
    rnr = np.concatenate([o[1] for o in outs]) if outs[0][1] is not None else None
    return dict(topk_idx=idx, topk_w=wt, layout=lay, xd=xd, xs=xs, out=out, out_no_routed=rnr)


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _time_passes(w, inp, S, threads, min_passes, min_seconds):
    times = []
    t_all = time.perf_counter()
    while len(times) < min_passes or time.perf_counter() - t_all < min_seconds:
        t0 = time.perf_counter()
        oracle_pass(w, inp, S, threads)
        times.append(time.perf_counter() - t0)
    return times


def cpu_baseline(w, inp: dict) -> dict:
    """The oracle on this machine's host cores over full passes of the workload:
    single-threaded, and split over token ranges on every core this process may
    use; each the median of at least 3 passes."""
    n = host_threads()
    single = _time_passes(w, inp, w.S, 1, 3, 0.0)
    multi = _time_passes(w, inp, w.S, n, 3, 5.0)
    med1, medn = statistics.median(single), statistics.median(multi)
    return {"value": w.S / medn, "unit": "tokens/s", "cores": n, "kind": "oracle",
            "sample": f"median of {len(multi)} full passes of {w.name} (S={w.S}) through the C oracle, "
                      f"per-token steps split over {n} threads by token range",
            "host_cpu_count": os.cpu_count(), "threads": n,
            "single_thread": {"value": w.S / med1, "unit": "tokens/s", "cores": 1,
                              "sample": f"median of {len(single)} full passes, one thread"}}


# ----------------------------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------------------------

def host_inputs(w) -> dict:
    from combine_moe_route_09_b200 import synth

    d = dict(logits=synth.logits(w), x=synth.activations(w), y=synth.expert_outputs(w))
    if w.fused:
        d["shared"], d["residual"] = synth.shared_out(w), synth.residual(w)
    return d


def run_reference(args, w, world):
    """CPU oracle as the reference arm: rank 0 only, every host core, a bounded
    token sample per step."""
    inp = host_inputs(w)
    n = host_threads()
    n_cal = min(w.S, max(256, 64 * n))
    t0 = time.perf_counter()
    oracle_pass(w, inp, n_cal, n)
    per_tok = (time.perf_counter() - t0) / n_cal
    budget = 60.0  # seconds for warm-up + timed steps together
    S_sample = int(max(1, min(w.S, budget / max(1, args.steps + args.warmup) / per_tok)))
    for _ in range(args.warmup):
        oracle_pass(w, inp, S_sample, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(w, inp, S_sample, n)
    el = time.perf_counter() - t0
    value = S_sample * args.steps / el
    sample = (f"first {S_sample} of {w.S} tokens of {w.name} per step (same H, E, K, R, padding, "
              f"quantisation and epilogue), C oracle split over {n} threads by token range")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded)", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle", "cores": n,
                         "host_cpu_count": os.cpu_count(), "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def _pct(v, q):
    v = sorted(v)
    if not v:
        return None
    i = (len(v) - 1) * q
    lo, hi = int(i), min(int(i) + 1, len(v) - 1)
    return v[lo] + (v[hi] - v[lo]) * (i - lo)


def _stats(v):
    return {"median": statistics.median(v), "p10": _pct(v, 0.1), "p90": _pct(v, 0.9), "n": len(v)}


def _graph_of(calls, n):
    """CUDA graph of n repetitions of the calls, captured on a side stream."""
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            for c in calls:
                c()
    return g


def time_windows(step, K, windows, world, device):
    """`windows` windows of exactly K steps each, every window bracketed by a
    barrier and a device synchronisation on both sides; ms per window (max over ranks)."""
    import torch

    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    for _ in range(windows):
        barrier(world)
        torch.cuda.synchronize()
        a.record()
        for _ in range(K):
            step()
        b.record()
        torch.cuda.synchronize()
        barrier(world)
        out.append(max_over_ranks(a.elapsed_time(b), world, device))
    return out


def phases_in_graph(phases, steps, windows):
    """Per-phase device time inside a CUDA graph of `steps` steps: an event node
    (cudaEventRecordExternal) before the first phase and after each phase of
    every step.  The event nodes sit between the kernels, so no phase overlaps
    its neighbour here; returns µs samples per phase."""
    import torch

    n = len(phases)
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)] for _ in range(steps)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            evs[i][0].record()
            for j, (_, call) in enumerate(phases):
                call()
                evs[i][j + 1].record()
    g.replay()
    torch.cuda.synchronize()
    samples = {name: [] for name, _ in phases}
    for _ in range(windows):
        g.replay()
        torch.cuda.synchronize()
        for i in range(steps):
            for j, (name, _) in enumerate(phases):
                samples[name].append(evs[i][j].elapsed_time(evs[i][j + 1]) * 1e3)
    del g
    return samples


def phases_marginal(phases, steps, windows):
    """Marginal cost of each phase in the graph-replayed step: the time per step
    of a graph of the first j+1 phases minus that of the first j phases (every
    graph `steps` steps long, consecutive kernels overlapping through
    programmatic dependent launch as in the product step).  The marginal costs
    add up to the step time; returns µs per phase."""
    import torch

    per_prefix = []
    for j in range(len(phases)):
        g = _graph_of([c for _, c in phases[:j + 1]], steps)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(windows):
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3 / steps)
        del g
        per_prefix.append(statistics.median(ts))
    out, prev = {}, 0.0
    for (name, _), t in zip(phases, per_prefix):
        out[name] = t - prev
        prev = t
    return out


def phases_eager(phases, steps):
    """Eager calls with an event between consecutive kernels (NVTX range per phase)."""
    import torch

    n = len(phases)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        ev[i][0].record()
        for j, (name, call) in enumerate(phases):
            with torch.cuda.nvtx.range(name):
                call()
            ev[i][j + 1].record()
    torch.cuda.synchronize()
    return {name: [ev[i][j].elapsed_time(ev[i][j + 1]) * 1e3 for i in range(steps)]
            for j, (name, _) in enumerate(phases)}


def _phase_table(us: dict, ab: dict, peak: float) -> dict:
    out = {}
    for name, t in us.items():
        gbs = ab[name] / (t * 1e-6) / 1e9
        out[name] = {"us": t, "algorithmic_bytes": ab[name], "gb_s": gbs, "frac_of_peak": gbs / peak,
                     "frac_of_nominal_8tbs": gbs / 8000.0}
    return out


def measure_workload(w, args, world, local_rank, device, windows, e2e: bool):
    """Times one workload: the graph-replayed step over `windows` windows of K
    steps, then its phases (event nodes in the graph, marginal costs, eager)."""
    import torch

    from combine_moe_route_09_b200 import synth
    from combine_moe_route_09_b200.buffer import MoeBuffer

    inp = host_inputs(w)
    pinned = {k: synth.to_torch(v).pin_memory() for k, v in inp.items()}
    d = {k: v.to(device, non_blocking=True) for k, v in pinned.items()}
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, dtype=dt, fp8=w.quant == "fp8", device=device,
                    fused=args.fused)
    sh, rs = (d["shared"], d["residual"]) if w.fused else (None, None)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        buf.step(d["logits"], d["x"], d["y"], sh, rs)
    torch.cuda.synchronize()
    if buf.read_status() != 0:
        raise RuntimeError("device status flagged a problem during warm-up")
    K = args.steps
    graph, gsteps = None, 1
    if args.graph:
        # consecutive steps captured in one graph, as a model's layers would be;
        # each kernel still waits for the one before it
        gsteps = max(1, min(args.graph_steps, K))
        while K % gsteps:
            gsteps -= 1
        graph = buf.capture(d["logits"], d["x"], d["y"], sh, rs, steps=gsteps)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        if buf.read_status() != 0:
            raise RuntimeError("device status flagged a problem in the captured steps")
    step = graph.replay if graph is not None else (lambda: buf.step(d["logits"], d["x"], d["y"], sh, rs))

    h0 = time.perf_counter()
    win_ms = time_windows(step, K // gsteps, windows, world, device)
    host_us = (time.perf_counter() - h0) / (K * windows) * 1e6
    phases = buf.step_phases(d["logits"], d["x"], d["y"], sh, rs)
    Kp = max(1, min(K, 50))
    ev_nodes = phases_in_graph(phases, Kp, max(3, windows // 2))
    marginal = phases_marginal(phases, Kp, max(3, windows // 2))
    eager = phases_eager(phases, Kp)
    torch.cuda.synchronize()
    status = buf.read_status()
    counts_ok = int(buf.layout.counts.sum().item()) == w.S * w.K
    if status != 0 or not counts_ok:
        raise RuntimeError(f"bench sanity check failed: status={status} counts_ok={counts_ok}")

    e2e_res = None
    if e2e:
        Ke = min(K, args.e2e_steps)
        out_h = torch.empty(buf.out.shape, dtype=buf.out.dtype).pin_memory()
        rnr_h = torch.empty(buf.out.shape, dtype=buf.out.dtype).pin_memory() if w.fused else None
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())
        d2h = out_h.numel() * out_h.element_size() * (2 if w.fused else 1)
        # Inputs go in on the compute stream; each step's outputs come back on a copy
        # stream, so that read overlaps the next step's input copies (PCIe is full
        # duplex).  A step's kernels wait for the previous read of the outputs.
        main = torch.cuda.current_stream(device)
        cstream = torch.cuda.Stream(device)
        step_done = torch.cuda.Event()
        read_done = torch.cuda.Event()
        read_done.record(cstream)

        def e2e_step():
            for k, v in pinned.items():
                d[k].copy_(v, non_blocking=True)
            main.wait_event(read_done)
            buf.step(d["logits"], d["x"], d["y"], sh, rs)
            step_done.record(main)
            cstream.wait_event(step_done)
            with torch.cuda.stream(cstream):
                out_h.copy_(buf.out, non_blocking=True)
                if rnr_h is not None:
                    rnr_h.copy_(buf.out_no_routed, non_blocking=True)
                read_done.record(cstream)

        e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        a.record()
        for _ in range(Ke):
            e2e_step()
        main.wait_event(read_done)  # the last step's outputs are on the host
        b.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, device)
        e2e_res = {"value": w.S * world * Ke / (e2e_ms / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": Ke,
                   "ms_per_step": e2e_ms / Ke,
                   "path": "MoeBuffer.step via the C ABI; pinned host inputs copied in and both residual "
                           "streams copied out each step (the copy out overlapping the next step's copy in), "
                           "inside the timed region"}

    ab = algorithmic_bytes(w)
    peak, peak_kind = read_peak_hbm()
    per_step = [t / K for t in win_ms]
    med = statistics.median(per_step)
    ph_in = {k: statistics.median(v) for k, v in ev_nodes.items()}
    res = {
        "ms_per_step": med, "ms_per_step_stats": _stats(per_step), "windows": windows, "steps_per_window": K,
        "tokens_per_s": w.S * world / (med * 1e-3),
        "phases": _phase_table(ph_in, ab, peak),
        "phases_p10_p90_us": {k: [_pct(v, 0.1), _pct(v, 0.9)] for k, v in ev_nodes.items()},
        "phases_marginal": _phase_table(marginal, ab, peak),
        "phases_eager": _phase_table({k: statistics.median(v) for k, v in eager.items()}, ab, peak),
        "gpu_launches_per_step": buf.kernels_per_step,
        "host_enqueue_us_per_step": host_us * gsteps,
        "graph": graph is not None, "graph_steps": gsteps,
        "plan": "fused route+layout+dispatch kernel" if buf.fused else "separate route, layout, dispatch kernels",
        "plan_timings_us": buf.plan_timings_us,
    }
    res["_buf"], res["_inp"], res["_e2e"], res["_peak"] = buf, inp, e2e_res, (peak, peak_kind)
    return res


def run_ours(args, w, rank, world, local_rank):
    import torch

    from combine_moe_route_09_b200 import synth

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    windows = max(10, args.windows)
    sampler = ClockSampler(local_rank)
    sampler.start()
    head = measure_workload(w, args, world, local_rank, device, windows, e2e=not args.no_e2e)
    others = {}
    if not args.headline_only:
        for key, ow in synth.WORKLOADS.items():
            if ow.name == w.name:
                continue
            r = measure_workload(ow, args, world, local_rank, device, windows, e2e=False)
            for k in ("_buf", "_inp", "_e2e", "_peak"):
                r.pop(k)
            r["config"] = {kk: vv for kk, vv in workload_config(ow, world).items() if kk != "l2"}
            others[key] = r
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
    clocks = sampler.stop()
    buf, inp, e2e, (peak, peak_kind) = head.pop("_buf"), head.pop("_inp"), head.pop("_e2e"), head.pop("_peak")
    if rank != 0:
        return
    ab = algorithmic_bytes(w)
    ph = head["phases"]
    dname = "route_dispatch" if "route_dispatch" in ph else "dispatch"
    dc_us = ph[dname]["us"] + ph["combine"]["us"]
    dc_gbs = (ab[dname] + ab["combine"]) / (dc_us * 1e-6) / 1e9
    comb = ph["combine"]
    roofline = {"kernel": "combine_kernel (gather + weighted sum + dual residual)", "bound": "hbm",
                "achieved": comb["gb_s"], "peak": peak, "unit": "GB/s", "frac": comb["gb_s"] / peak,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6650 GB/s",
                "algorithmic_bytes_per_launch": ab["combine"],
                "duration_us": comb["us"],
                "timing": "CUDA event nodes around the kernel inside the graph-replayed step",
                "traffic": recorded_traffic("combine.cu", w.name)}
    K = args.steps
    line = {
        "metric": METRIC, "value": head["tokens_per_s"], "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "ms_per_step_stats": head["ms_per_step_stats"], "windows": head["windows"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; no dataset or weights)", "config": workload_config(w, world),
        "dispatch_combine": {"tokens_per_s": w.S * world / (dc_us * 1e-6), "effective_gb_s": dc_gbs,
                             "frac_of_peak": dc_gbs / peak, "frac_of_nominal_8tbs": dc_gbs / 8000.0},
        "phases": ph, "phases_p10_p90_us": head["phases_p10_p90_us"],
        "phases_marginal": head["phases_marginal"], "phases_eager": head["phases_eager"],
        "roofline": roofline, "e2e": e2e,
        "gpu_launches": K * head["gpu_launches_per_step"], "clocks": clocks,
        "timing": ("value: median over windows of exactly K steps (barrier + synchronize around each window), "
                   + (f"{head['graph_steps']} consecutive steps per CUDA-graph replay" if head["graph"]
                      else "eager calls")
                   + "; phases: CUDA event nodes between the kernels inside a graph of min(K, 50) steps; "
                     "phases_marginal: leave-one-out graphs (a graph of the first j+1 phases minus one of the "
                     "first j), consecutive kernels overlapping as in the step; phases_eager: eager calls with "
                     "an event between kernels"),
        "host_enqueue_us_per_step": head["host_enqueue_us_per_step"],
        "plan": head["plan"], "plan_timings_us": head["plan_timings_us"],
        "workloads": others,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp)
    print(json.dumps(line), flush=True)


def backward_bytes(w) -> dict:
    """Bytes the backward calls must move at least (padding rows excluded)."""
    b = w.esize
    S, H, E, K = w.S, w.H, w.E, w.K
    gn = S * H * b if w.fused else 0
    combine_bwd = S * H * b + gn + 2 * S * K * H * b + S * K * 12 + (S * H * b if w.fused else 0)
    dispatch_bwd = S * K * H * b + S * H * b + S * K * 4
    route_bwd = S * K * 12 + S * E * 4
    return dict(combine_backward=combine_bwd, dispatch_backward=dispatch_bwd, route_backward=route_bwd)


def run_backward(args, w, rank, world, local_rank):
    """Times the training backward of the pass: combine backward (grad_y, grad_w and,
    with the dual residual, the skip gradient), dispatch backward of a synthetic
    expert-input gradient, and the router backward; forward state from one forward pass."""
    import numpy as np
    import torch

    from combine_moe_route_09_b200 import binding as B
    from combine_moe_route_09_b200 import synth
    from combine_moe_route_09_b200.buffer import MoeBuffer

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    inp = host_inputs(w)
    d = {k: synth.to_torch(v, device=device) for k, v in inp.items()}
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, dtype=dt, fp8=w.quant == "fp8", device=device)
    sh, rs = (d["shared"], d["residual"]) if w.fused else (None, None)
    buf.step(d["logits"], d["x"], d["y"], sh, rs)
    torch.cuda.synchronize()
    gen = torch.Generator(device=device).manual_seed(w.seed + 1000)
    g = torch.randn((w.S, w.H), generator=gen, device=device).to(dt)
    gn = torch.randn((w.S, w.H), generator=gen, device=device).to(dt) if w.fused else None
    gxd = torch.randn((buf.cap, w.H), generator=gen, device=device).to(dt)
    grad_y = torch.zeros((buf.cap, w.H), dtype=dt, device=device)
    grad_w = torch.empty((w.S, w.K), dtype=torch.float32, device=device)
    skip = torch.empty((w.S, w.H), dtype=dt, device=device) if w.fused else None
    grad_x = torch.empty((w.S, w.H), dtype=dt, device=device)
    grad_logits = torch.empty((w.S, w.E), dtype=torch.float32, device=device)
    status = buf.status
    slot = buf.layout.slot_of

    calls = [
        ("combine_backward", lambda: B.moe_combine_dual_residual_backward(
            g, d["y"], slot, buf.topk_w, grad_no_routed=gn, grad_y=grad_y, grad_w=grad_w, grad_skip=skip,
            want_skip=w.fused, status=status)),
        ("dispatch_backward", lambda: B.moe_dispatch_backward(gxd, slot, grad_x=grad_x, status=status)),
        ("route_backward", lambda: B.moe_route_topk_backward(buf.topk_idx, buf.topk_w, grad_w, w.E,
                                                             grad_logits=grad_logits)),
    ]

    def eager():
        for _, f in calls:
            f()

    for _ in range(args.warmup):
        eager()
    torch.cuda.synchronize()
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            eager()
        graph.replay()
        torch.cuda.synchronize()
    if buf.read_status() != 0:
        raise RuntimeError("device status flagged a problem")
    K = args.steps
    sampler = ClockSampler(local_rank)
    sampler.start()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(K):
        graph.replay() if graph is not None else eager()
    b.record()
    torch.cuda.synchronize()
    total_ms = max_over_ranks(a.elapsed_time(b), world, device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(K)]
    for i in range(K):
        ev[i][0].record()
        for j, (_, f) in enumerate(calls):
            f()
            ev[i][j + 1].record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if buf.read_status() != 0:
        raise RuntimeError("device status flagged a problem")
    if rank != 0:
        return
    ab = backward_bytes(w)
    peak, peak_kind = read_peak_hbm()
    phases = {}
    for j, (name, _) in enumerate(calls):
        ms = statistics.fmean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K))
        gbs = ab[name] / (ms * 1e-3) / 1e9
        phases[name] = {"us": ms * 1e3, "algorithmic_bytes": ab[name], "gb_s": gbs, "frac_of_peak": gbs / peak}
    cb = phases["combine_backward"]
    line = {
        "mode": "backward", "metric": "backward pass tokens/s (combine, dispatch and router backward), 1 GPU",
        "value": w.S * world * K / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded)",
        "config": workload_config(w, world), "phases": phases,
        "roofline": {"kernel": "combine_bwd_kernel", "bound": "hbm", "achieved": cb["gb_s"], "peak": peak,
                     "unit": "GB/s", "frac": cb["gb_s"] / peak, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": ab["combine_backward"],
                     "traffic": recorded_traffic("combine_bwd.cu", w.name)},
        "gpu_launches": K * 3, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_fp8_combine(args, w, rank, world, local_rank):
    """Times the combine over FP8 expert outputs (e4m3 + 128-channel scales) on the
    workload's shapes; the expert outputs are a seeded N(0,1) buffer quantised
    once by the FP8 dispatch kernel (identity slots)."""
    import torch

    from combine_moe_route_09_b200 import binding as B
    from combine_moe_route_09_b200 import synth
    from combine_moe_route_09_b200.buffer import MoeBuffer

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    inp = host_inputs(w)
    d = {k: synth.to_torch(v, device=device) for k, v in inp.items()}
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, dtype=dt, fp8=w.quant == "fp8", device=device)
    sh, rs = (d["shared"], d["residual"]) if w.fused else (None, None)
    buf.step(d["logits"], d["x"], d["y"], sh, rs)
    ident = torch.arange(buf.cap, dtype=torch.int32, device=device).reshape(-1, 1)
    yq, ys = B.moe_dispatch(d["y"], ident, buf.cap, B.MOE_QUANT_FP8_E4M3_B128)
    out = torch.empty((w.S, w.H), dtype=dt, device=device)
    rnr = torch.empty((w.S, w.H), dtype=dt, device=device) if w.fused else None

    def call():
        B.moe_combine_fp8_dual_residual(yq, ys, buf.layout.slot_of, buf.topk_w, shared_out=sh, residual=rs,
                                        residual_out=out, residual_no_routed_out=rnr, want_no_routed=w.fused,
                                        dtype=dt, status=buf.status)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    sampler = ClockSampler(local_rank)
    sampler.start()
    ev[0].record()
    for i in range(K):
        call()
        ev[i + 1].record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if buf.read_status() != 0:
        raise RuntimeError("device status flagged a problem")
    if rank != 0:
        return
    ms = statistics.fmean(ev[i].elapsed_time(ev[i + 1]) for i in range(K))
    S, H, Kk, b = w.S, w.H, w.K, w.esize
    nbytes = S * Kk * H + S * Kk * (H // 128) * 4 + S * Kk * 8 + (4 * S * H * b if w.fused else S * H * b)
    peak, peak_kind = read_peak_hbm()
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({"mode": "fp8_combine", "metric": "combine over FP8 expert outputs, tokens/s, 1 GPU",
                      "value": S / (ms * 1e-3), "unit": "tokens/s", "us_per_call": ms * 1e3,
                      "algorithmic_bytes": nbytes, "gb_s": gbs, "frac_of_peak": gbs / peak,
                      "peak_source": peak_kind, "traffic": recorded_traffic("combine_fp8.cu", w.name),
                      "config": workload_config(w, world), "clocks": clocks,
                      "steps": K, "warmup": args.warmup}), flush=True)


def run_router(args, w, rank, world, local_rank):
    """Times the two routers on the workload's logits: the softmax top-K of the
    routing pass and the variant (sigmoid scores, selection-only bias, n_group=8
    groups of which topk_group=4 are kept, normalised, scale 2.5)."""
    import numpy as np
    import torch

    from combine_moe_route_09_b200 import binding as B
    from combine_moe_route_09_b200 import synth

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    logits = synth.to_torch(synth.logits(w), device=device)
    bias = torch.from_numpy((np.random.default_rng(w.seed).standard_normal(w.E) * 0.05).astype(np.float32)).to(device)
    idx = torch.empty((w.S, w.K), dtype=torch.int32, device=device)
    wt = torch.empty((w.S, w.K), dtype=torch.float32, device=device)
    n_group = 8 if w.E % 8 == 0 and w.E // 8 >= 2 and 4 * (w.E // 8) >= w.K else 1
    # the layout of the softmax router's choice, for the routing weights in dispatched order
    from combine_moe_route_09_b200.buffer import MoeBuffer

    buf = MoeBuffer(w.S, w.H, w.K, w.E, w.R, w.P, device=device)
    buf.route(logits)
    lay = buf.plan()
    rw = torch.empty(buf.cap, dtype=torch.float32, device=device)
    calls = {
        "route_topk_softmax": lambda: B.moe_route_topk(logits, w.K, topk_idx=idx, topk_w=wt),
        "route_weights_dispatched": lambda: B.moe_dispatch_route_weights(buf.topk_w, lay.row_src, out=rw),
        "route_sigmoid_grouped": lambda: B.moe_route_sigmoid_grouped(
            logits, w.K, bias=bias, n_group=n_group, topk_group=4 if n_group > 1 else 1, normalize=True,
            scale=2.5, topk_idx=idx, topk_w=wt),
    }
    nbytes = w.S * w.E * 4 + w.S * w.K * 8 + (w.E * 4)
    rw_bytes = buf.cap * 8 + w.S * w.K * 4  # row_src read, weights written, topk_w gathered
    peak, peak_kind = read_peak_hbm()
    res = {}
    sampler = ClockSampler(local_rank)
    sampler.start()
    # Each call is a few microseconds of GPU work, less than a Python-side launch, so
    # the timed loop replays a CUDA graph of `per_graph` back-to-back calls.
    per_graph = 20
    for name, call in calls.items():
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for _ in range(per_graph):
                    call()
        torch.cuda.current_stream(device).wait_stream(side)
        g.replay()
        torch.cuda.synchronize()
        reps = max(1, args.steps // per_graph)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for _ in range(reps):
            g.replay()
        ev1.record()
        torch.cuda.synchronize()
        del g
        us = ev0.elapsed_time(ev1) * 1e3 / (reps * per_graph)
        gbs = (rw_bytes if name == "route_weights_dispatched" else nbytes) / (us * 1e-6) / 1e9
        res[name] = {"us_per_call": us, "tokens_per_s": w.S / (us * 1e-6), "gb_s": gbs, "frac_of_peak": gbs / peak}
    clocks = sampler.stop()
    if rank != 0:
        return
    print(json.dumps({"mode": "router", "metric": "router tokens/s, 1 GPU (CUDA-graph replays of back-to-back calls)",
                      "value": res["route_sigmoid_grouped"]["tokens_per_s"], "unit": "tokens/s",
                      "routers": res, "algorithmic_bytes": nbytes, "peak_source": peak_kind,
                      "n_group": n_group, "config": workload_config(w, world), "clocks": clocks,
                      "steps": args.steps, "warmup": args.warmup}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="4", help="1, 2, 2b, 3, 4 or 5 (default 4)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--windows", type=int, default=10,
                    help="timed windows of K steps each (at least 10); the value is their median")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other workloads (the JSON line's `workloads` object)")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=True,
                    help="time the value pass as CUDA-graph replays of one step (default; "
                         "--no-graph times eager calls)")
    ap.add_argument("--graph-steps", type=int, default=10,
                    help="consecutive steps captured in one CUDA graph (a divisor of --steps is used)")
    ap.add_argument("--fused", action=argparse.BooleanOptionalAction, default=None,
                    help="route + layout + dispatch as one kernel where it applies (--fused), never "
                         "(--no-fused), or (default) whichever of the two plans MoeBuffer times faster")
    ap.add_argument("--mode", default="forward", choices=["forward", "backward", "fp8_combine", "router"],
                    help="forward: the routing pass (default); backward: its training backward; "
                         "fp8_combine: the combine over FP8 expert outputs; router: both routers")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override S (a smaller case of the same workload, for profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from combine_moe_route_09_b200 import synth

    w = synth.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = w.replace(S=args.tokens, name=f"{w.name}_S{args.tokens}")
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.mode == "backward":
            run_backward(args, w, rank, world, local_rank)
        elif args.mode == "fp8_combine":
            run_fp8_combine(args, w, rank, world, local_rank)
        elif args.mode == "router":
            run_router(args, w, rank, world, local_rank)
        else:
            run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
