"""B200 (sm_100a) MoE router-and-dispatch path: Python binding of libmoe_dispatch.so.

The binding only marshals arguments: every step runs in the library's CUDA
kernels.  Each ``moe_*`` function below has the name, argument order and
meaning of the C entry point in ``include/moe_dispatch.h``; tensors are torch
CUDA tensors the caller allocated, and the launch goes to the current torch
stream unless ``stream`` is given.  A non-OK status raises :class:`MoeError`.

There is no fallback: if the library is missing, importing works but the first
call raises, telling how to build it.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "MoeError", "RouteParams", "library_path", "load_library",
    "SCORE_SOFTMAX", "SCORE_SIGMOID", "SCORE_SQRT_SOFTPLUS", "SCORE_TOPK_SOFTMAX",
    "MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_CUDA",
    "MOE_ERR_DEVICE_INDEX", "MOE_ERR_TIMEOUT", "MOE_ERR_NAN_LOGIT",
    "moe_status_string", "moe_gate_gemm", "moe_gate_route", "moe_route", "moe_hash_route",
    "moe_dispatch_workspace_size", "moe_dispatch", "moe_dispatch_static", "moe_permute",
    "moe_combine", "moe_permute_bounded", "moe_combine_bounded",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libmoe_dispatch.so"

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 0, 1, 2, 3
MOE_ERR_DEVICE_INDEX, MOE_ERR_TIMEOUT, MOE_ERR_NAN_LOGIT = 4, 5, 6
SCORE_SOFTMAX, SCORE_SIGMOID, SCORE_SQRT_SOFTPLUS, SCORE_TOPK_SOFTMAX = 0, 1, 2, 3

SCORE_BY_NAME = {"softmax": SCORE_SOFTMAX, "sigmoid": SCORE_SIGMOID,
                 "sqrt_softplus": SCORE_SQRT_SOFTPLUS, "topk_softmax": SCORE_TOPK_SOFTMAX}


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)} (status {status})")


class RouteParams(ctypes.Structure):
    """Mirror of moe_route_params."""
    _fields_ = [("num_experts", ctypes.c_int32), ("k_max", ctypes.c_int32),
                ("score", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("group_topn", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("route_scale", ctypes.c_float)]

    @classmethod
    def make(cls, num_experts, k_max, score, n_groups=1, topk_groups=1, group_topn=1,
             renormalize=True, route_scale=1.0):
        if isinstance(score, str):
            score = SCORE_BY_NAME[score]
        return cls(num_experts, k_max, score, n_groups, topk_groups, group_topn,
                   1 if renormalize else 0, route_scale)


_lib = None


def library_path() -> str:
    return os.path.join(_PKG, _LIB_NAME)


def load_library(path: str | None = None, strict: bool = True):
    """Load (once) and return the ctypes handle of libmoe_dispatch.so.  With a
    path, load that build instead (not cached); strict=False there tolerates
    an older build that lacks some entry points."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or library_path()
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m token_dispatch_moe_b200.build`")
    lib = ctypes.CDLL(p)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    st = ctypes.c_int
    sig = {
        "moe_status_string": ([st], ctypes.c_char_p),
        "moe_gate_gemm": ([P, P, P, i64, i32, i32, P, P], st),
        "moe_gate_route": ([P, P, P, P, ctypes.POINTER(RouteParams), i64, i32, P, P, P, P, P], st),
        "moe_route": ([P, P, P, ctypes.POINTER(RouteParams), i64, P, P, P, P], st),
        "moe_hash_route": ([P, P, i32, i32, P, ctypes.POINTER(RouteParams), i64, P, P, P, P], st),
        "moe_dispatch_workspace_size": ([i64, i32, i32, ctypes.POINTER(ctypes.c_size_t)], st),
        "moe_dispatch": ([P, i64, i32, i32, P, P, P, P, P, ctypes.c_size_t, P, P], st),
        "moe_dispatch_static": ([P, i64, i32, i32, P, P, P, P, P, P], st),
        "moe_expert_gate_up": ([P, P, P, P, P, P, i32, i32, i32, i64, i32, P, P, P], st),
        "moe_expert_down": ([P, P, P, P, i32, i32, i32, i64, P, P, P], st),
        "moe_wait_probe": ([ctypes.c_uint64, P, P, P], st),
        "moe_route_grouped": ([P, ctypes.POINTER(RouteParams), i32, i64, P, P, P, P], st),
        "moe_ep_layout": ([P, P, P, P, i32, i32, i64, i32, i32, P, P, P, P, P], st),
        "moe_ep_permute": ([P, P, P, P, i32, i64, i64, i32, i32, P, P], st),
        "moe_ep_combine": ([P, P, P, P, P, i32, i64, i64, i32, i32, P, P, P], st),
        "moe_dispatch_limited_rows": ([i64, i32, i32, i32, i32, ctypes.POINTER(i64)], st),
        "moe_dispatch_limited": ([P, i64, i32, i32, i32, i32, P, P, P, i64, P, P, P,
                                  ctypes.c_size_t, P, P], st),
        "moe_permute": ([P, P, i64, i32, i32, P, P], st),
        "moe_combine": ([P, P, P, P, i64, i32, i32, P, P], st),
        "moe_permute_bounded": ([P, P, i64, i32, i32, P, i64, P, P], st),
        "moe_combine_bounded": ([P, P, P, P, i64, i32, i32, i64, P, P, P], st),
    }
    for name, (args, res) in sig.items():
        if not strict and not hasattr(lib, name):
            continue
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path is None:
        _lib = lib
    return lib


def moe_status_string(status: int) -> str:
    try:
        return load_library().moe_status_string(status).decode()
    except RuntimeError:
        return f"status {status}"


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    """Raw handle of the stream to launch on (torch's current stream if None).
    A torch stream of another device than the current one is refused: the
    library launches on the current device, with its kernels reading the
    tensors' addresses there."""
    s = torch.cuda.current_stream() if stream is None else stream
    if hasattr(s, "device") and s.device.index != torch.cuda.current_device():
        raise ValueError(f"stream is on {s.device}, the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    return s.cuda_stream if hasattr(s, "cuda_stream") else s


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _need(t, dtype, name, ndim=None):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def moe_gate_gemm(x, w, logits, d_status=None, stream=None):
    """logits[T,E] (fp32) = x[T,d] (bf16) . w[E,d]^T (bf16), tcgen05 tensor cores."""
    _need(x, torch.bfloat16, "x", 2)
    _need(w, torch.bfloat16, "w", 2)
    _need(logits, torch.float32, "logits", 2)
    _need(d_status, torch.int32, "d_status")
    T, d = x.shape
    E = w.shape[0]
    if w.shape[1] != d or tuple(logits.shape) != (T, E):
        raise ValueError("shape mismatch")
    _check(load_library().moe_gate_gemm(_ptr(x), _ptr(w), _ptr(logits), T, d, E,
                                        _ptr(d_status), _stream(stream)), "moe_gate_gemm")


def moe_gate_route(x, w, bias, k_per_token, params: RouteParams, topk_ids, topk_w, logits=None,
                   d_status=None, stream=None):
    """moe_gate_gemm + moe_route in one kernel: each token's logits row is routed
    from the tensor-core accumulator; logits are written only if given."""
    _need(x, torch.bfloat16, "x", 2)
    _need(w, torch.bfloat16, "w", 2)
    _need(bias, torch.float32, "bias", 1)
    _need(k_per_token, torch.int32, "k_per_token", 1)
    _need(topk_ids, torch.int32, "topk_ids", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(logits, torch.float32, "logits", 2)
    _need(d_status, torch.int32, "d_status")
    T, d = x.shape
    E = w.shape[0]
    if w.shape[1] != d or E != params.num_experts or \
            tuple(topk_ids.shape) != (T, params.k_max) or tuple(topk_w.shape) != (T, params.k_max) \
            or (logits is not None and tuple(logits.shape) != (T, E)):
        raise ValueError("shape mismatch")
    _check(load_library().moe_gate_route(_ptr(x), _ptr(w), _ptr(bias), _ptr(k_per_token),
                                         ctypes.byref(params), T, d, _ptr(topk_ids), _ptr(topk_w),
                                         _ptr(logits), _ptr(d_status), _stream(stream)),
           "moe_gate_route")


def moe_route(logits, bias, k_per_token, params: RouteParams, topk_ids, topk_w, d_status=None,
              stream=None):
    """Scoring, bias, group limit, per-token top-k and weights (see the C header)."""
    _need(logits, torch.float32, "logits", 2)
    _need(bias, torch.float32, "bias", 1)
    _need(k_per_token, torch.int32, "k_per_token", 1)
    _need(topk_ids, torch.int32, "topk_ids", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(d_status, torch.int32, "d_status")
    T, E = logits.shape
    if E != params.num_experts or tuple(topk_ids.shape) != (T, params.k_max) or \
            tuple(topk_w.shape) != (T, params.k_max):
        raise ValueError("shape mismatch")
    _check(load_library().moe_route(_ptr(logits), _ptr(bias), _ptr(k_per_token),
                                    ctypes.byref(params), T, _ptr(topk_ids), _ptr(topk_w),
                                    _ptr(d_status), _stream(stream)), "moe_route")


def moe_route_grouped(logits, params: RouteParams, k_per_group: int, topk_ids, topk_w,
                      d_status=None, stream=None):
    """Per-group candidates (k_per_group best of each contiguous group), then
    the params.k_max best of them."""
    _need(logits, torch.float32, "logits", 2)
    _need(topk_ids, torch.int32, "topk_ids", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(d_status, torch.int32, "d_status")
    T, E = logits.shape
    if E != params.num_experts or tuple(topk_ids.shape) != (T, params.k_max) or \
            tuple(topk_w.shape) != (T, params.k_max):
        raise ValueError("shape mismatch")
    _check(load_library().moe_route_grouped(_ptr(logits), ctypes.byref(params), k_per_group, T,
                                            _ptr(topk_ids), _ptr(topk_w), _ptr(d_status),
                                            _stream(stream)), "moe_route_grouped")


def moe_hash_route(token_ids, tid2eid, logits, params: RouteParams, topk_ids, topk_w,
                   d_status=None, stream=None):
    """Expert ids = tid2eid[token_ids] (row-major [vocab][k]); weights per the C header."""
    _need(token_ids, torch.int32, "token_ids", 1)
    _need(tid2eid, torch.int32, "tid2eid", 2)
    _need(logits, torch.float32, "logits", 2)
    _need(topk_ids, torch.int32, "topk_ids", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(d_status, torch.int32, "d_status")
    vocab, k = tid2eid.shape
    T = token_ids.shape[0]
    if tuple(topk_ids.shape) != (T, k) or tuple(topk_w.shape) != (T, k):
        raise ValueError("shape mismatch")
    _check(load_library().moe_hash_route(_ptr(token_ids), _ptr(tid2eid), vocab, k, _ptr(logits),
                                         ctypes.byref(params), T, _ptr(topk_ids), _ptr(topk_w),
                                         _ptr(d_status), _stream(stream)), "moe_hash_route")


def moe_dispatch_workspace_size(T: int, k_max: int, E: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().moe_dispatch_workspace_size(T, k_max, E, ctypes.byref(n)),
           "moe_dispatch_workspace_size")
    return int(n.value)


def moe_dispatch(topk_ids, E, counts, offsets, sorted_token, dest_pos, workspace, d_status=None,
                 stream=None):
    """Histogram, exclusive scan and stable scatter into expert-contiguous order."""
    _need(topk_ids, torch.int32, "topk_ids", 2)
    for t, n in ((counts, "counts"), (offsets, "offsets"), (sorted_token, "sorted_token"),
                 (dest_pos, "dest_pos"), (d_status, "d_status")):
        _need(t, torch.int32, n)
    _need(workspace, torch.uint8, "workspace")
    T, k_max = topk_ids.shape
    if counts.numel() < E or offsets.numel() < E + 1 or sorted_token.numel() < T * k_max or \
            tuple(dest_pos.shape) != (T, k_max):
        raise ValueError("shape mismatch")
    _check(load_library().moe_dispatch(_ptr(topk_ids), T, k_max, E, _ptr(counts), _ptr(offsets),
                                       _ptr(sorted_token), _ptr(dest_pos), _ptr(workspace),
                                       workspace.numel(), _ptr(d_status), _stream(stream)),
           "moe_dispatch")


def moe_dispatch_limited_rows(T: int, k_max: int, E: int, capacity: int = 0, pad: int = 1) -> int:
    """Rows sorted_token and the permuted activations need under moe_dispatch_limited."""
    out = ctypes.c_int64(0)
    _check(load_library().moe_dispatch_limited_rows(T, k_max, E, capacity, pad, ctypes.byref(out)),
           "moe_dispatch_limited_rows")
    return out.value


def switch_capacity(T: int, k: int, E: int, capacity_factor: float) -> int:
    """Per-expert capacity ceil(capacity_factor * T * k / E): the fair share of
    the T*k slots times the factor (the Switch-style limit)."""
    return max(1, math.ceil(capacity_factor * T * k / E))


def moe_dispatch_limited(topk_ids, E, capacity, pad, counts, offsets, sorted_token, dest_pos,
                         workspace, dropped=None, d_status=None, stream=None):
    """moe_dispatch with a per-expert capacity (0 = none; each expert keeps its
    first `capacity` slots in flat order) and expert blocks padded to a multiple
    of `pad` rows (padding rows of sorted_token are -1)."""
    _need(topk_ids, torch.int32, "topk_ids", 2)
    for t, n in ((counts, "counts"), (offsets, "offsets"), (sorted_token, "sorted_token"),
                 (dest_pos, "dest_pos"), (dropped, "dropped"), (d_status, "d_status")):
        _need(t, torch.int32, n)
    _need(workspace, torch.uint8, "workspace")
    T, k_max = topk_ids.shape
    if counts.numel() < E or offsets.numel() < E + 1 or tuple(dest_pos.shape) != (T, k_max):
        raise ValueError("shape mismatch")
    _check(load_library().moe_dispatch_limited(
        _ptr(topk_ids), T, k_max, E, capacity, pad, _ptr(counts), _ptr(offsets),
        _ptr(sorted_token), sorted_token.numel(), _ptr(dest_pos), _ptr(dropped), _ptr(workspace),
        workspace.numel(), _ptr(d_status), _stream(stream)), "moe_dispatch_limited")


def moe_ep_layout(all_counts, topk_ids, dest_pos, offsets, rank, dest_rank, dest_row,
                  recv_offsets, d_status=None, stream=None):
    """Owner rank and receive row of every slot (expert e on rank e // (E // G))."""
    _need(all_counts, torch.int32, "all_counts", 2)
    for t, n in ((topk_ids, "topk_ids"), (dest_pos, "dest_pos"), (offsets, "offsets"),
                 (dest_rank, "dest_rank"), (dest_row, "dest_row"),
                 (recv_offsets, "recv_offsets"), (d_status, "d_status")):
        _need(t, torch.int32, n)
    G, E = all_counts.shape
    T, k_max = topk_ids.shape
    if tuple(dest_pos.shape) != (T, k_max) or tuple(dest_rank.shape) != (T, k_max) or \
            tuple(dest_row.shape) != (T, k_max) or offsets.numel() < E + 1 or \
            recv_offsets.numel() < E // G + 1:
        raise ValueError("shape mismatch")
    _check(load_library().moe_ep_layout(
        _ptr(all_counts), _ptr(topk_ids), _ptr(dest_pos), _ptr(offsets), G, rank, T, k_max, E,
        _ptr(dest_rank), _ptr(dest_row), _ptr(recv_offsets), _ptr(d_status), _stream(stream)),
        "moe_ep_layout")


def peer_table(buffers, device=None) -> torch.Tensor:
    """Device array of the G receive-buffer addresses (int64), as the EP calls
    take it; entry r must be rank r's buffer as mapped in this process."""
    addrs = [b.data_ptr() for b in buffers]
    dev = device if device is not None else buffers[0].device
    return torch.tensor(addrs, dtype=torch.int64, device=dev)


def moe_ep_permute(x, dest_rank, dest_row, peers, recv_capacity, d_status=None, stream=None):
    """Store every row of x into its owners' receive buffers (peers: a
    peer_table of G [recv_capacity, d] bf16 buffers)."""
    _need(x, torch.bfloat16, "x", 2)
    for t, n in ((dest_rank, "dest_rank"), (dest_row, "dest_row"), (d_status, "d_status")):
        _need(t, torch.int32, n)
    _need(peers, torch.int64, "peers", 1)
    T, d = x.shape
    k_max = dest_rank.shape[1]
    _check(load_library().moe_ep_permute(_ptr(x), _ptr(dest_rank), _ptr(dest_row), _ptr(peers),
                                         peers.numel(), recv_capacity, T, k_max, d,
                                         _ptr(d_status), _stream(stream)), "moe_ep_permute")


def moe_ep_combine(peers_y, dest_rank, dest_row, topk_w, shared, out, recv_capacity,
                   d_status=None, stream=None):
    """moe_combine reading each slot's expert output from its owner."""
    for t, n in ((dest_rank, "dest_rank"), (dest_row, "dest_row"), (d_status, "d_status")):
        _need(t, torch.int32, n)
    _need(peers_y, torch.int64, "peers_y", 1)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(shared, torch.bfloat16, "shared", 2)
    _need(out, torch.bfloat16, "out", 2)
    T, d = out.shape
    k_max = dest_rank.shape[1]
    _check(load_library().moe_ep_combine(_ptr(peers_y), _ptr(dest_rank), _ptr(dest_row),
                                         _ptr(topk_w), _ptr(shared), peers_y.numel(),
                                         recv_capacity, T, k_max, d, _ptr(out), _ptr(d_status),
                                         _stream(stream)), "moe_ep_combine")


MOE_ACT_SWIGLU, MOE_ACT_SWIGLU_OAI = 0, 1


def moe_expert_gate_up(xs, offsets, w1, w3, h, b1=None, b3=None, act=MOE_ACT_SWIGLU,
                       d_status=None, stream=None):
    """h = act(xs W1[e]^T + b1[e], xs W3[e]^T + b3[e]) per 128-row-aligned expert block."""
    for t, n in ((xs, "xs"), (w1, "w1"), (w3, "w3"), (h, "h")):
        _need(t, torch.bfloat16, n)
    _need(offsets, torch.int32, "offsets", 1)
    _need(b1, torch.float32, "b1")
    _need(b3, torch.float32, "b3")
    _need(d_status, torch.int32, "d_status")
    E, F, d = w1.shape
    rows = xs.shape[0]
    if tuple(w3.shape) != (E, F, d) or xs.shape[1] != d or tuple(h.shape) != (rows, F) or \
            offsets.numel() != E + 1:
        raise ValueError("shape mismatch")
    _check(load_library().moe_expert_gate_up(_ptr(xs), _ptr(offsets), _ptr(w1), _ptr(w3), _ptr(b1),
                                             _ptr(b3), E, d, F, rows, act, _ptr(h),
                                             _ptr(d_status), _stream(stream)),
           "moe_expert_gate_up")


def moe_expert_down(h, offsets, w2, y, b2=None, d_status=None, stream=None):
    """y = h W2[e]^T + b2[e] per 128-row-aligned expert block."""
    for t, n in ((h, "h"), (w2, "w2"), (y, "y")):
        _need(t, torch.bfloat16, n)
    _need(offsets, torch.int32, "offsets", 1)
    _need(b2, torch.float32, "b2")
    _need(d_status, torch.int32, "d_status")
    E, d, F = w2.shape
    rows = h.shape[0]
    if h.shape[1] != F or tuple(y.shape) != (rows, d) or offsets.numel() != E + 1:
        raise ValueError("shape mismatch")
    _check(load_library().moe_expert_down(_ptr(h), _ptr(offsets), _ptr(w2), _ptr(b2), E, d, F,
                                          rows, _ptr(y), _ptr(d_status), _stream(stream)),
           "moe_expert_down")


def moe_wait_probe(limit_ns: int, d_status, d_outcome=None, stream=None):
    """Run the library's bounded wait against a barrier nothing completes (a
    diagnostic for the timeout path): *d_status gets MOE_ERR_TIMEOUT."""
    _need(d_status, torch.int32, "d_status")
    _need(d_outcome, torch.int32, "d_outcome")
    _check(load_library().moe_wait_probe(limit_ns, _ptr(d_status), _ptr(d_outcome),
                                         _stream(stream)), "moe_wait_probe")


def moe_dispatch_static(topk_ids, E, counts, offsets, sorted_token, dest_pos, d_status=None,
                        stream=None):
    """moe_dispatch with the library's own fixed scratch (606,208 bytes: the
    largest workspace any accepted size needs) instead of a caller-allocated
    workspace, for callers that cannot allocate device memory.
    Calls that overlap on the GPU race on that scratch; the first call on a
    device should come before any stream capture."""
    _need(topk_ids, torch.int32, "topk_ids", 2)
    for t, n in ((counts, "counts"), (offsets, "offsets"), (sorted_token, "sorted_token"),
                 (dest_pos, "dest_pos"), (d_status, "d_status")):
        _need(t, torch.int32, n)
    T, k_max = topk_ids.shape
    if counts.numel() < E or offsets.numel() < E + 1 or sorted_token.numel() < T * k_max or \
            tuple(dest_pos.shape) != (T, k_max):
        raise ValueError("shape mismatch")
    _check(load_library().moe_dispatch_static(_ptr(topk_ids), T, k_max, E, _ptr(counts),
                                              _ptr(offsets), _ptr(sorted_token), _ptr(dest_pos),
                                              _ptr(d_status), _stream(stream)),
           "moe_dispatch_static")


def moe_permute(x, dest_pos, xs, stream=None):
    """xs[dest_pos[t,j]] = x[t]: rows copied into expert-contiguous order."""
    _need(x, torch.bfloat16, "x", 2)
    _need(dest_pos, torch.int32, "dest_pos", 2)
    _need(xs, torch.bfloat16, "xs", 2)
    T, d = x.shape
    if dest_pos.shape[0] != T or xs.shape[1] != d:
        raise ValueError("shape mismatch")
    _check(load_library().moe_permute(_ptr(x), _ptr(dest_pos), T, dest_pos.shape[1], d, _ptr(xs),
                                      _stream(stream)), "moe_permute")


def moe_combine(y, topk_w, dest_pos, shared, out, stream=None):
    """out[t] = bf16(sum_j w[t,j] * y[dest_pos[t,j]] + shared[t]), fp32 accumulation."""
    _need(y, torch.bfloat16, "y", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(dest_pos, torch.int32, "dest_pos", 2)
    _need(shared, torch.bfloat16, "shared", 2)
    _need(out, torch.bfloat16, "out", 2)
    T, d = out.shape
    k_max = dest_pos.shape[1]
    if dest_pos.shape[0] != T or tuple(topk_w.shape) != (T, k_max) or y.shape[1] != d or \
            (shared is not None and tuple(shared.shape) != (T, d)):
        raise ValueError("shape mismatch")
    _check(load_library().moe_combine(_ptr(y), _ptr(topk_w), _ptr(dest_pos), _ptr(shared), T,
                                      k_max, d, _ptr(out), _stream(stream)), "moe_combine")


def moe_permute_bounded(x, dest_pos, xs, d_status=None, stream=None):
    """moe_permute with every dest_pos checked against xs's rows: a value
    outside [-1, xs rows) is skipped and reported in d_status."""
    _need(x, torch.bfloat16, "x", 2)
    _need(dest_pos, torch.int32, "dest_pos", 2)
    _need(xs, torch.bfloat16, "xs", 2)
    _need(d_status, torch.int32, "d_status")
    T, d = x.shape
    if dest_pos.shape[0] != T or xs.shape[1] != d:
        raise ValueError("shape mismatch")
    _check(load_library().moe_permute_bounded(_ptr(x), _ptr(dest_pos), T, dest_pos.shape[1], d,
                                              _ptr(xs), xs.shape[0], _ptr(d_status),
                                              _stream(stream)), "moe_permute_bounded")


def moe_combine_bounded(y, topk_w, dest_pos, shared, out, d_status=None, stream=None):
    """moe_combine with every dest_pos checked against y's rows: a value
    outside [-1, y rows) is skipped (its term left out) and reported."""
    _need(y, torch.bfloat16, "y", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(dest_pos, torch.int32, "dest_pos", 2)
    _need(shared, torch.bfloat16, "shared", 2)
    _need(out, torch.bfloat16, "out", 2)
    _need(d_status, torch.int32, "d_status")
    T, d = out.shape
    k_max = dest_pos.shape[1]
    if dest_pos.shape[0] != T or tuple(topk_w.shape) != (T, k_max) or y.shape[1] != d or \
            (shared is not None and tuple(shared.shape) != (T, d)):
        raise ValueError("shape mismatch")
    _check(load_library().moe_combine_bounded(_ptr(y), _ptr(topk_w), _ptr(dest_pos), _ptr(shared),
                                              T, k_max, d, y.shape[0], _ptr(out), _ptr(d_status),
                                              _stream(stream)), "moe_combine_bounded")
