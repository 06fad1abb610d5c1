"""CPU oracle for the MoE router-and-dispatch path -- TEST INFRASTRUCTURE ONLY.

The arithmetic lives in ``oracle.c`` (plain C, fp64, single-threaded); this
module only compiles it with gcc and marshals numpy arrays.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm may
import it.  It shares nothing with the CUDA library and the library never
calls it.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SOFTMAX, SIGMOID, SQRT_SOFTPLUS, TOPK_SOFTMAX = 0, 1, 2, 3
OK, ERR_ARG, ERR_INDEX, ERR_NAN = 0, 1, 4, 6

_lib = None


def compile_c(src: str, out: str) -> str:
    """gcc an oracle source file into a shared library (ISO C, no FMA contraction)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
         "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_c(_SRC, _LIB)
    return _LIB


@contextlib.contextmanager
def using_library(path: str):
    """Route every wrapper below through another build of the oracle (tests
    use this to check that a planted mistake makes the pins fail)."""
    global _lib
    old = _lib
    _lib = _bind(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = old


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    lib.oracle_gate_rows.argtypes = [P, P, i32, i32, P, i64, P]
    lib.oracle_gate_rows.restype = None
    lib.oracle_scores.argtypes = [P, i64, i32, i32, P]
    lib.oracle_scores.restype = None
    lib.oracle_route.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, i32, i32, f64,
                                 P, P, P, P]
    lib.oracle_route.restype = ctypes.c_int
    lib.oracle_weights_for_ids.argtypes = [P, P, i64, i32, i32, i32, i32, f64, P]
    lib.oracle_weights_for_ids.restype = ctypes.c_int
    lib.oracle_hash_route.argtypes = [P, P, i32, i32, P, i64, i32, i32, i32, f64, P, P]
    lib.oracle_hash_route.restype = ctypes.c_int
    lib.oracle_dispatch.argtypes = [P, i64, i32, i32, P, P, P, P]
    lib.oracle_dispatch.restype = ctypes.c_int
    lib.oracle_dispatch_limited.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P, P]
    lib.oracle_dispatch_limited.restype = ctypes.c_int
    lib.oracle_route_grouped.argtypes = [P, i64, i32, i32, i32, i32, i32, i32, f64, P, P, P]
    lib.oracle_route_grouped.restype = ctypes.c_int
    lib.oracle_expert_gate_up.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, P, i64, P, P, P]
    lib.oracle_expert_gate_up.restype = ctypes.c_int
    lib.oracle_expert_down.argtypes = [P, P, P, P, i32, i32, i32, P, i64, P]
    lib.oracle_expert_down.restype = ctypes.c_int
    lib.oracle_ep_layout.argtypes = [P, i32, i64, i32, i32, P, P, P]
    lib.oracle_ep_layout.restype = ctypes.c_int
    lib.oracle_permute.argtypes = [P, P, i64, i32, i32, P]
    lib.oracle_permute.restype = None
    lib.oracle_combine.argtypes = [P, P, P, P, i64, i32, i32, P, P]
    lib.oracle_combine.restype = None
    return lib


def _c(a, dtype):
    """Contiguous array of the given dtype (no copy when already so)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data


def bf16_bits(a) -> np.ndarray:
    """uint16 view of bf16 data given as a uint16 array or a torch bf16 tensor."""
    if hasattr(a, "view") and hasattr(a, "dtype") and "bfloat16" in str(a.dtype):
        import torch
        return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return _c(a, np.uint16)


def gate_rows(x_bits, w_bits, rows=None) -> np.ndarray:
    """fp64 logits of the listed rows: sum_i x[t,i]*W[e,i] in ascending i."""
    x = _c(x_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    T, d = x.shape
    E = w.shape[0]
    assert w.shape[1] == d
    rows = np.arange(T, dtype=np.int64) if rows is None else _c(rows, np.int64)
    out = np.empty((rows.size, E), np.float64)
    _load().oracle_gate_rows(_p(x), _p(w), d, E, _p(rows), rows.size, _p(out))
    return out


def scores(logits, score: int) -> np.ndarray:
    lg = _c(logits, np.float32)
    T, E = lg.shape
    out = np.empty((T, E), np.float64)
    _load().oracle_scores(_p(lg), T, E, score, _p(out))
    return out


def route(logits, *, k_max, score, bias=None, k_per_token=None, n_groups=1, topk_groups=1,
          group_topn=1, renormalize=True, route_scale=1.0, want_keys=False):
    """Returns dict(ids, w, status[, keys, group_gap])."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    b = None if bias is None else _c(bias, np.float32)
    kp = None if k_per_token is None else _c(k_per_token, np.int32)
    ids = np.empty((T, k_max), np.int32)
    w = np.empty((T, k_max), np.float64)
    keys = np.empty((T, E), np.float64) if want_keys else None
    gap = np.empty((T,), np.float64) if want_keys else None
    st = _load().oracle_route(_p(lg), _p(b), _p(kp), T, E, k_max, score, n_groups, topk_groups,
                              group_topn, int(bool(renormalize)), float(route_scale), _p(ids),
                              _p(w), _p(keys), _p(gap))
    out = {"ids": ids, "w": w, "status": st}
    if want_keys:
        out["keys"] = keys
        out["group_gap"] = gap
    return out


def weights_for_ids(logits, ids, *, score, renormalize=True, route_scale=1.0) -> np.ndarray:
    lg = _c(logits, np.float32)
    ids = _c(ids, np.int32)
    T, E = lg.shape
    k_max = ids.shape[1]
    w = np.empty((T, k_max), np.float64)
    st = _load().oracle_weights_for_ids(_p(lg), _p(ids), T, E, k_max, score,
                                        int(bool(renormalize)), float(route_scale), _p(w))
    assert st == OK, st
    return w


def route_grouped(logits, *, k_max, score, n_groups, k_per_group, renormalize=True,
                  route_scale=1.0, want_keys=False):
    """Grouped top-k (per-group k, then the global top k_max of the candidates)."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k_max), np.int32)
    w = np.empty((T, k_max), np.float64)
    keys = np.empty((T, E), np.float64) if want_keys else None
    st = _load().oracle_route_grouped(_p(lg), T, E, k_max, score, n_groups, k_per_group,
                                      int(renormalize), float(route_scale), _p(ids), _p(w),
                                      _p(keys) if keys is not None else None)
    if st == ERR_ARG:
        raise ValueError("oracle_route_grouped: bad arguments")
    out = {"ids": ids, "w": w, "status": st}
    if want_keys:
        out["keys"] = keys
    return out


def hash_route(tok, table, *, num_experts, logits=None, score=SOFTMAX, renormalize=True,
               route_scale=1.0):
    tok = _c(tok, np.int32)
    table = _c(table, np.int32)
    vocab, k = table.shape
    T = tok.shape[0]
    lg = None if logits is None else _c(logits, np.float32)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    st = _load().oracle_hash_route(_p(tok), _p(table), vocab, k, _p(lg), T, num_experts, score,
                                   int(bool(renormalize)), float(route_scale), _p(ids), _p(w))
    return {"ids": ids, "w": w, "status": st}


def dispatch(ids, num_experts):
    ids = _c(ids, np.int32)
    T, k_max = ids.shape
    counts = np.empty((num_experts,), np.int32)
    offsets = np.empty((num_experts + 1,), np.int32)
    sorted_token = np.full((max(T * k_max, 1),), -7, np.int32)
    dest_pos = np.empty((T, k_max), np.int32)
    st = _load().oracle_dispatch(_p(ids), T, k_max, num_experts, _p(counts), _p(offsets),
                                 _p(sorted_token), _p(dest_pos))
    n = int(offsets[-1])
    return {"counts": counts, "offsets": offsets, "sorted_token": sorted_token[:n],
            "dest_pos": dest_pos, "status": st}


def dispatch_limited(ids, num_experts, capacity: int = 0, pad: int = 1):
    """Dispatch with a per-expert capacity (0 = none) and expert blocks padded
    to a multiple of ``pad`` rows; returns counts (demand), padded offsets,
    sorted_token (padding rows -1), dest_pos (-1 for dropped slots), dropped."""
    ids = _c(ids, np.int32)
    T, k_max = ids.shape
    counts = np.empty((num_experts,), np.int32)
    offsets = np.empty((num_experts + 1,), np.int32)
    rows = T * k_max if capacity <= 0 else min(T * k_max, num_experts * capacity)
    rows += num_experts * (pad - 1)
    sorted_token = np.full((max(rows, 1),), -7, np.int32)
    dest_pos = np.empty((T, k_max), np.int32)
    dropped = ctypes.c_int64(0)
    st = _load().oracle_dispatch_limited(_p(ids), T, k_max, num_experts, capacity, pad,
                                         _p(counts), _p(offsets), _p(sorted_token),
                                         _p(dest_pos), ctypes.byref(dropped))
    n = int(offsets[-1])
    return {"counts": counts, "offsets": offsets, "sorted_token": sorted_token[:n],
            "dest_pos": dest_pos, "dropped": int(dropped.value), "status": st}


def ep_layout(ids_all, num_experts):
    """Expert-parallel receive layout for G ranks' ids [G][T][k_max]: the owner
    rank and row of every slot, and each rank's received row count."""
    ids = _c(ids_all, np.int32)
    G, T, k_max = ids.shape
    dest_rank = np.empty((G, T, k_max), np.int32)
    dest_row = np.empty((G, T, k_max), np.int32)
    recv_rows = np.zeros((G,), np.int64)
    st = _load().oracle_ep_layout(_p(ids), G, T, k_max, num_experts, _p(dest_rank), _p(dest_row),
                                  _p(recv_rows))
    return {"dest_rank": dest_rank, "dest_row": dest_row, "recv_rows": recv_rows, "status": st}


def ep_permute(x_all_bits, dest_rank, dest_row, recv_rows):
    """Each rank's receive buffer: recv[d][dest_row] = x[r][t] for every slot
    (r, t, j) whose owner is d.  Rows are copied bit for bit."""
    x = np.asarray(x_all_bits, np.uint16)
    G, T, d = x.shape
    recv = [np.zeros((int(recv_rows[g]), d), np.uint16) for g in range(G)]
    for r in range(G):
        for t in range(T):
            for j in range(dest_rank.shape[2]):
                g = dest_rank[r, t, j]
                if g >= 0:
                    recv[g][dest_row[r, t, j]] = x[r, t]
    return recv


def ep_combine(y_bits_per_rank, w_all, dest_rank, dest_row, shared_all_bits=None, want_mag=True):
    """out[r][t] = sum_j w[r][t][j] * y[owner][row] (+ shared[r][t]): the
    combine of one source rank reads each slot's row from its owner.  Built
    from ``combine`` on the owners' rows laid end to end."""
    G = dest_rank.shape[0]
    starts = np.concatenate([[0], np.cumsum([y.shape[0] for y in y_bits_per_rank])])
    y_cat = np.concatenate([np.asarray(y, np.uint16) for y in y_bits_per_rank], axis=0)
    if y_cat.shape[0] == 0:
        y_cat = np.zeros((1, y_bits_per_rank[0].shape[1]), np.uint16)
    outs = []
    for r in range(G):
        gpos = np.where(dest_rank[r] >= 0, starts[np.maximum(dest_rank[r], 0)] + dest_row[r], -1)
        outs.append(combine(y_cat, w_all[r], gpos.astype(np.int32),
                            None if shared_all_bits is None else shared_all_bits[r],
                            want_mag=want_mag))
    return outs


SWIGLU, SWIGLU_OAI = 0, 1


def expert_gate_up(xs_bits, offsets, w1_bits, w3_bits, rows, *, act=SWIGLU, b1=None, b3=None,
                   want_pre=False):
    """h rows (fp64, unrounded) of the experts' gate/up step for the listed rows."""
    xs = _c(xs_bits, np.uint16)
    off = _c(offsets, np.int32)
    w1 = _c(w1_bits, np.uint16)
    w3 = _c(w3_bits, np.uint16)
    E, F, d = w1.shape
    r = _c(rows, np.int64)
    h = np.empty((r.size, F), np.float64)
    g = np.empty((r.size, F), np.float64) if want_pre else None
    u = np.empty((r.size, F), np.float64) if want_pre else None
    bb1 = None if b1 is None else _c(b1, np.float32)
    bb3 = None if b3 is None else _c(b3, np.float32)
    st = _load().oracle_expert_gate_up(_p(xs), _p(off), _p(w1), _p(w3), _p(bb1), _p(bb3), E, d, F,
                                       act, _p(r), r.size, _p(h), _p(g), _p(u))
    if st != OK:
        raise ValueError("oracle_expert_gate_up: a row lies in no expert block")
    return (h, g, u) if want_pre else h


def expert_down(h_bits, offsets, w2_bits, rows, *, b2=None):
    """y rows (fp64) of the experts' down projection for the listed rows of h."""
    hb = _c(h_bits, np.uint16)
    off = _c(offsets, np.int32)
    w2 = _c(w2_bits, np.uint16)
    E, d, F = w2.shape
    r = _c(rows, np.int64)
    y = np.empty((r.size, d), np.float64)
    bb2 = None if b2 is None else _c(b2, np.float32)
    st = _load().oracle_expert_down(_p(hb), _p(off), _p(w2), _p(bb2), E, d, F, _p(r), r.size,
                                    _p(y))
    if st != OK:
        raise ValueError("oracle_expert_down: a row lies in no expert block")
    return y


def permute(x_bits, dest_pos, n_rows: int) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    dp = _c(dest_pos, np.int32)
    T, d = x.shape
    xs = np.zeros((n_rows, d), np.uint16)
    _load().oracle_permute(_p(x), _p(dp), T, dp.shape[1], d, _p(xs))
    return xs


def combine(y_bits, w, dest_pos, shared_bits=None, want_mag=True):
    y = _c(y_bits, np.uint16)
    wf = _c(w, np.float32)
    dp = _c(dest_pos, np.int32)
    T, k_max = dp.shape
    d = y.shape[1]
    sh = None if shared_bits is None else _c(shared_bits, np.uint16)
    out = np.empty((T, d), np.float64)
    mag = np.empty((T, d), np.float64) if want_mag else None
    _load().oracle_combine(_p(y), _p(wf), _p(dp), _p(sh), T, k_max, d, _p(out), _p(mag))
    return (out, mag) if want_mag else out
