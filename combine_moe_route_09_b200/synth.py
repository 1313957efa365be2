"""Seeded synthetic inputs for the MoE dispatch/combine workloads.

This module only draws random numbers and fixes shapes; it holds none of the
routing, layout, quantisation or combine arithmetic.  Tests, the oracle and
the benchmark all take their inputs from here.

Every tensor gets its own stream family (numpy ``SeedSequence(seed).spawn``),
so a tensor's values do not depend on which other tensors were drawn.  Large
tensors are drawn in fixed chunks of rows, each chunk from its own SFC64
stream (spawned from the tensor's seed sequence), in parallel threads; the
values depend only on (seed, tensor, shape), never on the thread count.  bf16
tensors are drawn in fp32 and rounded to bf16 (nearest-even) by torch; they
are returned as numpy ``uint16`` bit patterns.

Workloads (S tokens in total over R logical ranks, hidden H, E experts, top-K,
P = token_padding, 0 = none):

====  ==============================  =====  ====  ===  ==  ==  ===  =====  =====  =====
name  what                            S      H     E    K   R   P    dtype  quant  fused
====  ==============================  =====  ====  ===  ==  ==  ===  =====  =====  =====
1     tiny, CPU-checkable             128    256   8    2   2   0    f32    none   yes
2     MoonEP API example, 4 x 1024    4096   768   384  8   4   128  bf16   none   no
2b    same, 1024 tokens in total      1024   768   384  8   4   128  bf16   none   no
3     DeepSeek-V3-shaped decode       128    7168  256  8   8   0    bf16   fp8    no
4     DeepSeek-V3-shaped prefill      4096   7168  256  8   8   0    bf16   fp8    yes
5     imbalanced 16B-A3B-style        16384  2048  64   8   8   128  bf16   none   yes
====  ==============================  =====  ====  ===  ==  ==  ===  =====  =====  =====

Distributions: logits ~N(0,1) fp32; workload 4 adds a per-expert bias
~N(0, 0.5); workload 5 adds a Zipf(s=1.1) bias alpha * (-1.1 * ln r_e) with r_e
a seeded permutation of 1..E and alpha chosen (once, offline, with the oracle)
so that the largest expert load is about 4x the mean.  Activations x, shared_out
and residual ~N(0,1); workload 3 multiplies 1% of the channels (a seeded choice)
by 20.  Expert gains ~U(0.5, 1.5).  Expert outputs for timing ~N(0,1).
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_ZIPF_FILE = os.path.join(_HERE, "zipf_alpha.json")


@dataclass(frozen=True)
class Workload:
    name: str
    S: int
    H: int
    E: int
    K: int
    R: int
    P: int
    dtype: str          # "f32" or "bf16"
    quant: str          # "none" or "fp8"
    fused: bool         # combine with the dual-residual epilogue
    bias: str = "none"  # "none", "normal" (sigma 0.5) or "zipf"
    outlier_frac: float = 0.0
    outlier_gain: float = 1.0
    seed: int = 0

    @property
    def cap(self) -> int:
        """Rows of the dispatched buffer: S*K + E*max(P-1, 0) always fits."""
        return self.S * self.K + self.E * max(self.P - 1, 0)

    @property
    def esize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "1": Workload("tiny_fp32", 128, 256, 8, 2, 2, 0, "f32", "none", True, seed=1),
    "2": Workload("moonep_api_4x1024", 4096, 768, 384, 8, 4, 128, "bf16", "none", False, seed=2),
    "2b": Workload("moonep_api_1024", 1024, 768, 384, 8, 4, 128, "bf16", "none", False, seed=2),
    "3": Workload("dsv3_decode_fp8", 128, 7168, 256, 8, 8, 0, "bf16", "fp8", False,
                  outlier_frac=0.01, outlier_gain=20.0, seed=3),
    "4": Workload("dsv3_prefill_fp8_dualres", 4096, 7168, 256, 8, 8, 0, "bf16", "fp8", True,
                  bias="normal", seed=4),
    "5": Workload("a3b_imbalanced_bf16_dualres", 16384, 2048, 64, 8, 8, 128, "bf16", "none", True,
                  bias="zipf", seed=5),
}

# Index of each tensor's stream family.
_STREAMS = dict(logits=0, bias=1, x=2, outliers=3, gains=4, shared=5, residual=6, y=7, perm=8)


_CHUNK_ELEMS = 1 << 22


def _seq(seed: int, name: str) -> np.random.SeedSequence:
    return np.random.SeedSequence(seed).spawn(len(_STREAMS))[_STREAMS[name]]


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.SFC64(_seq(seed, name)))


def _normal(seed: int, name: str, rows: int, cols: int) -> np.ndarray:
    """N(0,1) fp32 [rows, cols], drawn in fixed row chunks, one SFC64 stream per chunk."""
    out = np.empty((rows, cols), np.float32)
    if rows == 0:
        return out
    step = max(1, _CHUNK_ELEMS // max(cols, 1))
    starts = list(range(0, rows, step))
    seqs = _seq(seed, name).spawn(len(starts))

    def fill(i):
        r0 = starts[i]
        g = np.random.Generator(np.random.SFC64(seqs[i]))
        g.standard_normal(out=out[r0:r0 + step], dtype=np.float32)

    if len(starts) == 1:
        fill(0)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(len(starts))))
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (nearest-even, by torch) as uint16 bit patterns."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _cast(a: np.ndarray, dtype: str) -> np.ndarray:
    return a.astype(np.float32) if dtype == "f32" else f32_to_bf16_bits(a)


def zipf_alpha() -> float:
    """Bias scale for the imbalanced workload (written by oracle/calibrate_zipf.py)."""
    with open(_ZIPF_FILE) as f:
        return float(json.load(f)["alpha"])


def expert_bias(w: Workload, alpha: float | None = None) -> np.ndarray:
    if w.bias == "none":
        return np.zeros(w.E, np.float32)
    if w.bias == "normal":
        return (_rng(w.seed, "bias").standard_normal(w.E) * 0.5).astype(np.float32)
    if w.bias == "zipf":
        a = zipf_alpha() if alpha is None else alpha
        r = _rng(w.seed, "perm").permutation(w.E) + 1
        return (a * (-1.1 * np.log(r.astype(np.float64)))).astype(np.float32)
    raise ValueError(w.bias)


def logits(w: Workload, alpha: float | None = None) -> np.ndarray:
    """Router logits [S,E] fp32: N(0,1) plus the per-expert bias (added in fp32)."""
    z = _normal(w.seed, "logits", w.S, w.E)
    return (z + expert_bias(w, alpha)[None, :]).astype(np.float32)


def activations(w: Workload) -> np.ndarray:
    """Token activations x [S,H] in the workload dtype."""
    x = _normal(w.seed, "x", w.S, w.H)
    if w.outlier_frac > 0:
        n = int(round(w.outlier_frac * w.H))
        ch = _rng(w.seed, "outliers").permutation(w.H)[:n]
        x[:, ch] *= np.float32(w.outlier_gain)
    return _cast(x, w.dtype)


def shared_out(w: Workload) -> np.ndarray:
    return _cast(_normal(w.seed, "shared", w.S, w.H), w.dtype)


def residual(w: Workload) -> np.ndarray:
    return _cast(_normal(w.seed, "residual", w.S, w.H), w.dtype)


def expert_gains(w: Workload) -> np.ndarray:
    """Per-expert scalar gain ~U(0.5, 1.5) for the identity-times-gain expert stand-in."""
    return _rng(w.seed, "gains").uniform(0.5, 1.5, w.E).astype(np.float32)


def expert_outputs(w: Workload) -> np.ndarray:
    """Expert outputs y [cap,H] ~N(0,1) in the workload dtype (a timing stand-in)."""
    return _cast(_normal(w.seed, "y", w.cap, w.H), w.dtype)


def to_torch(a: np.ndarray, dtype: str | None = None, device="cpu"):
    """numpy -> torch; uint16 arrays become bfloat16 (bit reinterpretation)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(device)


def from_torch(t) -> np.ndarray:
    """torch -> numpy; bfloat16 becomes uint16 bit patterns, float8 becomes uint8."""
    import torch

    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()
