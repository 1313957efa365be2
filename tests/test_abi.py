"""The C-ABI library on a machine without a GPU: it builds, loads, exports
every entry point include/moe_route.h declares with the arity the binding
uses, and its host-side argument checks reject bad calls before any device
work.  No call here launches a kernel."""
import ctypes
import os
import re

import pytest

from combine_moe_route_09_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_route.h")


def _declared():
    """(name, number of parameters) of every function the header declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"\b([A-Za-z_][A-Za-z0-9_ \*]*?)\b(moe_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
        params = [p for p in m.group(3).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(2)] = len(params)
    return out


@pytest.fixture(scope="module")
def lib():
    from combine_moe_route_09_b200 import build

    build.build()
    return binding.lib()


def test_header_declares_the_four_steps():
    d = _declared()
    for name in ("moe_route_topk", "moe_dispatch_layout", "moe_dispatch_layout_workspace",
                 "moe_dispatch", "moe_combine_dual_residual"):
        assert name in d


def test_every_declared_symbol_is_exported(lib):
    for name, nparams in _declared().items():
        assert hasattr(lib, name), name
        assert name in binding.SIGNATURES, f"binding lacks {name}"
        assert len(binding.SIGNATURES[name][1]) == nparams, name


def test_library_path_is_in_tree(lib):
    assert os.path.dirname(binding.LIB_PATH) == os.path.join(ROOT, "combine_moe_route_09_b200")


def test_host_only_queries(lib):
    assert lib.moe_capacity(4096, 256, 8, 0) == 4096 * 8
    assert lib.moe_capacity(16384, 64, 8, 128) == 16384 * 8 + 64 * 127
    assert lib.moe_dispatch_layout_workspace(4096, 256, 8) >= 256 + 16 * 256 * 4
    assert lib.moe_dispatch_layout_workspace(4096, 2000, 8) == 0  # E > MOE_MAX_EXPERTS
    assert lib.moe_error_string(1) == b"invalid argument"
    # the wait self-test refuses bad arguments before launching anything
    assert lib.moe_selftest_wait_timeout(2, 1000, FAKE, FAKE, None) == 1
    assert lib.moe_selftest_wait_timeout(0, 0, FAKE, None, None) == 1
    assert lib.moe_selftest_wait_timeout(1, 1000, FAKE, None, None) == 1
    # invalid sizes answer 0 before any CUDA call
    assert lib.moe_dispatch_layout_kernels(0, 8, 2) == 0
    assert lib.moe_dispatch_layout_kernels(16, 2000, 2) == 0
    assert lib.moe_dispatch_layout_kernels(16, 64, 33) == 0


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails its host checks


@pytest.mark.parametrize("args", [
    (FAKE, 10, 8, 9, FAKE, FAKE, None),      # K > E
    (FAKE, 10, 2000, 8, FAKE, FAKE, None),   # E > MOE_MAX_EXPERTS
    (FAKE, 10, 64, 33, FAKE, FAKE, None),    # K > MOE_MAX_TOPK
    (FAKE, -1, 8, 2, FAKE, FAKE, None),      # S < 0
    (None, 10, 8, 2, FAKE, FAKE, None),      # NULL logits
])
def test_route_rejects(lib, args):
    assert lib.moe_route_topk(*args) == binding.MOE_ERR_INVALID_ARG


def test_route_empty_is_noop(lib):
    assert lib.moe_route_topk(None, 0, 8, 2, None, None, None) == binding.MOE_OK


def _layout(lib, S=16, E=8, K=2, R=2, P=0, cap=None, ws=FAKE, ws_bytes=1 << 20, **kw):
    cap = S * K if cap is None else cap
    a = dict(topk_idx=FAKE, counts=FAKE, offsets=FAKE, rank_offsets=FAKE, slot_of=FAKE, row_src=FAKE)
    a.update(kw)
    return lib.moe_dispatch_layout(a["topk_idx"], S, E, K, R, P, a["counts"], a["offsets"],
                                   a["rank_offsets"], a["slot_of"], a["row_src"], cap, ws, ws_bytes,
                                   None, None)


def test_layout_rejects(lib):
    bad = binding.MOE_ERR_INVALID_ARG
    assert _layout(lib, E=8, R=3) == bad                      # E % R != 0
    assert _layout(lib, P=-1) == bad
    assert _layout(lib, cap=-1) == bad
    assert _layout(lib, cap=1 << 31) == bad
    assert _layout(lib, ws=ctypes.c_void_p((1 << 20) + 4)) == bad   # misaligned workspace
    assert _layout(lib, ws_bytes=16) == bad                   # workspace too small
    assert _layout(lib, counts=None) == bad
    assert _layout(lib, S=1 << 28, K=16) == bad               # S*K >= 2^31
    assert _layout(lib, P=1 << 22, E=1024, R=1) == bad        # padded layout overflows int32


def test_dispatch_rejects(lib):
    bad = binding.MOE_ERR_INVALID_ARG
    D = lib.moe_dispatch
    assert D(FAKE, 1, 8, 100, 2, FAKE, 0, FAKE, None, 16, None, None) == bad   # bf16 row 200 B
    assert D(FAKE, 1, 8, 192, 2, FAKE, 1, FAKE, FAKE, 16, None, None) == bad   # FP8 needs H%128
    assert D(FAKE, 1, 8, 256, 2, FAKE, 1, FAKE, None, 16, None, None) == bad   # FP8 needs xs
    assert D(FAKE, 1, 8, 256, 2, FAKE, 0, FAKE, FAKE, 16, None, None) == bad   # xs only with FP8
    assert D(FAKE, 7, 8, 256, 2, FAKE, 0, FAKE, None, 16, None, None) == bad   # unknown dtype
    assert D(FAKE, 1, 8, 256, 2, FAKE, 5, FAKE, None, 16, None, None) == bad   # unknown quant
    assert D(ctypes.c_void_p((1 << 20) + 8), 1, 8, 256, 2, FAKE, 0, FAKE, None, 16, None, None) == bad
    assert D(None, 1, 0, 256, 2, None, 0, None, None, 0, None, None) == binding.MOE_OK  # S == 0


def test_combine_rejects(lib):
    bad = binding.MOE_ERR_INVALID_ARG
    C = lib.moe_combine_dual_residual
    # residual_no_routed_out without shared_out
    assert C(FAKE, 1, 8, 256, 2, 16, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None) == bad
    # f32 row of 5 elements (20 B)
    assert C(FAKE, 0, 8, 5, 2, 16, FAKE, FAKE, None, None, FAKE, None, None, None) == bad
    # K > MOE_MAX_TOPK
    assert C(FAKE, 1, 8, 256, 40, 16, FAKE, FAKE, None, None, FAKE, None, None, None) == bad
    # NULL output
    assert C(FAKE, 1, 8, 256, 2, 16, FAKE, FAKE, None, None, None, None, None, None) == bad


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="CUDA library missing"):
        binding.lib()
