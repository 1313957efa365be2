"""bench.py host logic on CPU: the max-over-ranks timing with world size 2
(gloo), the reference arm's rank handling, and the JSON line's contract.
No GPU is used: the reference arm runs the CPU oracle."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(10.0 * (rank + 1), world, device="cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 20.0, 1: 20.0}


def test_single_rank_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5


def _run_bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, env=env, timeout=600, cwd=ROOT)


def bench_threads() -> int:
    sys.path.insert(0, ROOT)
    import bench

    return bench.host_threads()


def test_threaded_oracle_pass_equals_single_threaded():
    """The CPU baseline splits the per-token steps over threads by token range;
    the result must be the single-threaded pass, bit for bit."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import bench
    from combine_moe_route_09_b200 import synth

    for key in ("1", "2b"):
        w = synth.WORKLOADS[key]
        inp = bench.host_inputs(w)
        a = bench.oracle_pass(w, inp, w.S, 1)
        b = bench.oracle_pass(w, inp, w.S, 3)
        for k in ("topk_idx", "topk_w", "xd", "out"):
            assert np.array_equal(a[k], b[k]), (key, k)
        for k in ("slot_of", "row_src", "counts", "offsets"):
            assert np.array_equal(a["layout"][k], b["layout"][k]), (key, k)
        if a["out_no_routed"] is not None:
            assert np.array_equal(a["out_no_routed"], b["out_no_routed"])


def test_reference_arm_line_contract():
    r = _run_bench({}, "--impl", "reference", "--workload", "1", "--steps", "3", "--warmup", "3")
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 3 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == bench_threads()
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny_fp32"


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--impl", "reference",
                   "--workload", "1", "--steps", "3", "--warmup", "3")
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = _run_bench({}, "--impl", "reference", "--workload", "1", "--steps", "3", "--warmup", "2")
    assert r.returncode != 0


def test_algorithmic_bytes_formula():
    sys.path.insert(0, ROOT)
    import bench
    from combine_moe_route_09_b200 import synth

    b = bench.algorithmic_bytes(synth.WORKLOADS["4"])
    S, H, E, K = 4096, 7168, 256, 8
    assert b["dispatch"] == S * H * 2 + S * K * H + S * K * (H // 128) * 4 + S * K * 4
    assert b["combine"] == S * K * H * 2 + S * K * 8 + 4 * S * H * 2
    assert round(b["dispatch"] / 1e6, 1) == 301.1 and round(b["combine"] / 1e6, 1) == 704.9


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    """The roofline's DRAM traffic is read from a profile summary only while the kernel
    source it was captured from is unchanged (same SHA-256) and the workload matches."""
    import hashlib

    sys.path.insert(0, ROOT)
    import bench

    src = tmp_path / "combine_moe_route_09_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("// kernel v1\n")
    sha = hashlib.sha256(b"// kernel v1\n").hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k_w.md").write_text(f"# k\n\nkernel_source_sha256: {sha}\nworkload: w\ndram_bytes_per_launch: 12345\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k.cu", "w") == 12345
    assert bench.recorded_traffic("k.cu", "other") is None
    (src / "k.cu").write_text("// kernel v2\n")
    assert bench.recorded_traffic("k.cu", "w") is None
    assert bench.recorded_traffic("missing.cu", "w") is None
