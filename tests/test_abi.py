"""The C-ABI library without a GPU: it builds for sm_100a, loads, exports
every entry point include/*.h declares, and its host-side validation answers
with status codes before any CUDA call."""
import ctypes
import glob
import os
import re

import pytest

import token_dispatch_moe_b200 as moe
from token_dispatch_moe_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    path = build_mod.build()
    return moe.load_library(path)


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        with open(h) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("moe_gate_gemm", "moe_route", "moe_hash_route", "moe_dispatch",
              "moe_dispatch_workspace_size", "moe_permute", "moe_combine", "moe_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings(lib):
    assert moe.moe_status_string(0) == "ok"
    assert "timed out" in moe.moe_status_string(moe.MOE_ERR_TIMEOUT)


def _expected_workspace(T, k, E):
    """One int32 per (segment, expert), the expert row padded to whole 16-byte
    quads; a segment is 8 warps x 32 lanes x `items` slots, items the smallest
    of 4, 8, 16 for which 148 segments cover every slot; above 296 segments a
    segment takes as many such rounds as keep the segments at most 296;
    rounded up to 256 B."""
    n = T * k
    items = 4
    while items * 32 * 8 * 148 < n and items < 16:
        items *= 2
    seg = items * 32 * 8
    s1 = -(-n // seg)
    rounds = 1 if s1 <= 296 else -(-s1 // 296)
    segs = -(-n // (seg * rounds))
    b = segs * (-(-E // 4) * 4) * 4
    return -(-b // 256) * 256


def test_workspace_size(lib):
    assert moe.moe_dispatch_workspace_size(0, 8, 256) == 0
    for T, k, E in [(16384, 16, 128), (4000, 5, 130), (65536, 32, 512), (1, 1, 1),
                    (70000, 8, 256), (25000, 8, 7)]:
        assert moe.moe_dispatch_workspace_size(T, k, E) == _expected_workspace(T, k, E)
    assert moe.moe_dispatch_workspace_size(16384, 16, 128) == 128 * 128 * 4  # 128 segments of 8 items
    assert moe.moe_dispatch_workspace_size(1, 1, 1) == 256
    # rounds keep the segments at most 296, whatever the size
    assert moe.moe_dispatch_workspace_size(37888, 32, 512) == 296 * 512 * 4  # exactly 296
    assert moe.moe_dispatch_workspace_size(65536, 32, 512) == 256 * 512 * 4  # 512 -> 2 rounds
    for T in (37889, 262144, 1 << 22, (2 ** 31 - 1) // 32):
        assert moe.moe_dispatch_workspace_size(T, 32, 512) <= 296 * 512 * 4
    with pytest.raises(moe.MoeError):
        moe.moe_dispatch_workspace_size(10, 33, 8)   # k_max > 32
    with pytest.raises(moe.MoeError):
        moe.moe_dispatch_workspace_size(10, 4, 513)  # E > 512


def test_host_validation_needs_no_gpu(lib):
    P = moe.RouteParams
    bad = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    # route: NULL params, E % n_groups, k > kept experts, bad score, k_max > 32
    assert lib.moe_route(bad, None, None, None, 4, bad, bad, None, None) == moe.MOE_ERR_INVALID_ARG
    for p in (P.make(12, 4, "softmax", n_groups=5), P.make(12, 4, "softmax", n_groups=4),
              P.make(12, 4, 7), P.make(64, 33, "softmax"), P.make(600, 4, "softmax"),
              P.make(16, 2, "sigmoid", n_groups=4, topk_groups=2, group_topn=3)):
        assert lib.moe_route(bad, None, None, ctypes.byref(p), 4, bad, bad, None, None) != 0
    # T = 0 is a no-op that returns OK without touching the device
    p = P.make(12, 4, "softmax")
    assert lib.moe_route(None, None, None, ctypes.byref(p), 0, None, None, None, None) == 0
    assert lib.moe_gate_gemm(bad, bad, bad, 4, 12, 8, None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_gate_gemm(bad, bad, bad, 4, 64, 513, None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_gate_gemm(None, None, None, 0, 64, 8, None, None) == 0
    assert lib.moe_hash_route(bad, bad, 10, 0, None, ctypes.byref(p), 4, bad, bad, None,
                              None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(bad, bad, 4, 2, 12, bad, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(bad, bad, bad, None, 4, 2, 10, bad, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(ctypes.c_void_p(18), bad, 4, 2, 16, bad, None) == \
        moe.MOE_ERR_INVALID_ARG  # x not 16-byte aligned
    ws = ctypes.c_void_p(256 * 3 + 8)  # not 256-byte aligned
    assert lib.moe_dispatch(bad, 4, 2, 8, bad, bad, bad, bad, ws, 1 << 20, None, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lib.moe_dispatch(bad, 4, 2, 8, bad, bad, bad, bad, ctypes.c_void_p(256), 0, None,
                            None) == moe.MOE_ERR_INVALID_ARG  # workspace too small


def test_static_dispatch_refuses_without_launch(lib):
    """The only sizes moe_dispatch_static refuses are those moe_dispatch refuses
    (T*k_max >= 2^31): answered before any device call (pointers never read)."""
    bad = ctypes.c_void_p(16)
    assert lib.moe_dispatch_static(bad, 1 << 26, 32, 512, bad, bad, bad, bad, None,
                                   None) == moe.MOE_ERR_UNSUPPORTED


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        moe.load_library(str(tmp_path / "libmoe_dispatch.so"))


def test_limited_rows_bound(lib):
    # min(T*k, E*capacity) + E*(pad-1)
    assert moe.moe_dispatch_limited_rows(100, 2, 8) == 200
    assert moe.moe_dispatch_limited_rows(100, 2, 8, capacity=10) == 80
    assert moe.moe_dispatch_limited_rows(100, 2, 8, capacity=30, pad=128) == 200 + 8 * 127
    assert moe.moe_dispatch_limited_rows(0, 4, 16, capacity=5, pad=4) == 16 * 3
    for bad in (dict(capacity=-1), dict(pad=0), dict(pad=4097)):
        with pytest.raises(moe.MoeError):
            moe.moe_dispatch_limited_rows(10, 2, 8, **bad)
    with pytest.raises(moe.MoeError):
        moe.moe_dispatch_limited_rows(1 << 27, 16, 8)  # T*k_max reaches 2^31
    assert moe.switch_capacity(262144, 1, 128, 1.0) == 2048
    assert moe.switch_capacity(256, 2, 8, 1.25) == 80
