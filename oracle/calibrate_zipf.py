"""Find the Zipf bias scale alpha of the imbalanced workload (test infrastructure).

The imbalanced 16B-A3B-style workload (S=16384, E=64, K=8) adds
alpha * (-1.1 * ln r_e) to every token's logits, r_e a seeded permutation of
1..E, and wants the busiest expert to receive about 4x the mean load.  This
script routes the seeded logits with the oracle for each trial alpha, bisects
on max/mean of the oracle's per-expert counts, and writes the result to
combine_moe_route_09_b200/zipf_alpha.json, which the input generator reads.

Run:  python -m oracle.calibrate_zipf
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
from combine_moe_route_09_b200 import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "combine_moe_route_09_b200", "zipf_alpha.json")


def load_ratio(w: synth.Workload, alpha: float) -> float:
    idx, _ = oracle.route_topk(synth.logits(w, alpha), w.K)
    counts = oracle.layout(idx, w.E, w.R, 0)["counts"]
    return float(counts.max() / counts.mean())


def main() -> None:
    w = synth.WORKLOADS["5"]
    lo, hi = 0.0, 4.0
    assert load_ratio(w, lo) < 4.0 < load_ratio(w, hi)
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if load_ratio(w, mid) < 4.0:
            lo = mid
        else:
            hi = mid
    alpha = round(hi, 6)
    ratio = load_ratio(w, alpha)
    assert 3.9 <= ratio <= 4.1, ratio
    rec = {"alpha": alpha, "max_over_mean": round(ratio, 4), "workload": w.name, "seed": w.seed,
           "written_by": "oracle/calibrate_zipf.py (oracle routing, bisection on max/mean load)"}
    with open(OUT, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))


if __name__ == "__main__":
    main()
