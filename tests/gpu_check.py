"""Comparison helpers for the GPU parity tests: each stage of the CUDA path
against the CPU oracle, the oracle fed with the GPU's previous-stage output.

Rules (each a tolerance derived from the arithmetic of the stage):
  gate     |g - o| <= 1e-3 * max(|o|, sigma), sigma = sum_i |x_i W_ei| * 2^-8
           (fp32 accumulation of exact products; sigma keeps cancelled
           near-zero logits from failing a purely relative test)
  route    ids identical, except rows where the oracle's fp64 keys of the two
           choices differ by < 1e-6 relative (swap of near-tied experts) or the
           last kept and first dropped group scores do (group near-tie); those
           rows are counted and must still be valid selections; weights within
           1e-5 relative, per slot
  dispatch counts, offsets, sorted_token, dest_pos bit-exact
  permute  bit-exact rows
  combine  |g - o| <= 1e-2 * max(|o|, sum_j |w_j y_j| + |s|)  (bf16 output)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

SCORE = {"softmax": oracle.SOFTMAX, "sigmoid": oracle.SIGMOID,
         "sqrt_softplus": oracle.SQRT_SOFTPLUS, "topk_softmax": oracle.TOPK_SOFTMAX}
NEAR_TIE = 1e-6
W_RTOL = 1e-5
GATE_RTOL = 1e-3
COMBINE_RTOL = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def np32(t):
    return None if t is None else t.detach().contiguous().cpu().numpy()


def check_gate(logits_gpu: torch.Tensor, x: torch.Tensor, w: torch.Tensor, rows=None) -> float:
    """Returns the largest |g-o| / max(|o|, sigma) seen (must be <= 1e-3)."""
    T = x.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    ridx = torch.as_tensor(rows, device=x.device, dtype=torch.long)
    xb = bits(x.index_select(0, ridx))
    wb = bits(w)
    o = oracle.gate_rows(xb, wb)
    g = logits_gpu.index_select(0, ridx).cpu().numpy().astype(np.float64)
    sigma = (np.abs(bits_to_f64(xb)) @ np.abs(bits_to_f64(wb)).T) * 2.0 ** -8
    scale = np.maximum(np.abs(o), sigma)
    ratio = np.abs(g - o) / np.where(scale > 0, scale, 1.0)
    worst = float(ratio.max()) if ratio.size else 0.0
    bad = np.argwhere(ratio > GATE_RTOL)
    assert bad.size == 0, f"gate: {len(bad)} logits out of tolerance, first {bad[:5]}, worst {worst}"
    return worst


def check_route(gpu_ids, gpu_w, logits, *, k_max, score, bias=None, kpt=None, n_groups=1,
                topk_groups=1, group_topn=1, renormalize=True, route_scale=1.0) -> dict:
    gpu_ids = np.asarray(gpu_ids)
    gpu_w = np.asarray(gpu_w, np.float64)
    sc = SCORE[score] if isinstance(score, str) else score
    o = oracle.route(logits, k_max=k_max, score=sc, bias=bias, k_per_token=kpt,
                     n_groups=n_groups, topk_groups=topk_groups, group_topn=group_topn,
                     renormalize=renormalize, route_scale=route_scale, want_keys=True)
    E = logits.shape[1]
    same = np.all(gpu_ids == o["ids"], axis=1)
    bad = np.nonzero(~same)[0]
    swapped = group_tied = 0
    for t in bad:
        g, oi = gpu_ids[t], o["ids"][t]
        assert np.array_equal(g < 0, oi < 0), f"route row {t}: padding differs {g} vs {oi}"
        sel = g[g >= 0]
        assert len(set(sel.tolist())) == sel.size and np.all(sel < E), f"route row {t}: {g}"
        if o["group_gap"][t] < NEAR_TIE:
            group_tied += 1
            continue
        keys = o["keys"][t]
        kg, ko = keys[g[oi >= 0]], keys[oi[oi >= 0]]
        ok = np.all(np.abs(kg - ko) <= NEAR_TIE * np.maximum(np.abs(ko), 1e-30))
        assert ok, (f"route row {t}: gpu {g} oracle {oi}; oracle keys of gpu choice {kg}, "
                    f"of oracle choice {ko}")
        swapped += 1
    # weights, slot by slot (padding must be exactly 0)
    ow = o["w"]
    if bad.size:
        ow = ow.copy()
        ow[bad] = oracle.weights_for_ids(logits[bad], gpu_ids[bad], score=sc,
                                         renormalize=renormalize, route_scale=route_scale)
    err = np.abs(gpu_w - ow)
    okw = err <= W_RTOL * np.abs(ow)
    if not okw.all():
        i = np.argwhere(~okw)[:5]
        raise AssertionError(f"route weights out of tolerance at {i.tolist()}: "
                             f"gpu {gpu_w[tuple(i.T)]} oracle {ow[tuple(i.T)]}")
    return {"rows": int(gpu_ids.shape[0]), "near_tie_swaps": swapped,
            "group_near_ties": group_tied, "status": o["status"]}


def check_dispatch(gpu_ids, counts, offsets, sorted_token, dest_pos, E):
    o = oracle.dispatch(np.asarray(gpu_ids), E)
    n = int(o["offsets"][-1])
    assert np.array_equal(np.asarray(counts), o["counts"]), "counts differ"
    assert np.array_equal(np.asarray(offsets), o["offsets"]), "offsets differ"
    assert np.array_equal(np.asarray(sorted_token)[:n], o["sorted_token"]), "sorted_token differs"
    assert np.array_equal(np.asarray(dest_pos), o["dest_pos"]), "dest_pos differs"
    return n


def check_dispatch_limited(gpu_ids, counts, offsets, sorted_token, dest_pos, dropped, E,
                           capacity, pad):
    o = oracle.dispatch_limited(np.asarray(gpu_ids), E, capacity=capacity, pad=pad)
    n = int(o["offsets"][-1])
    assert np.array_equal(np.asarray(counts), o["counts"]), "counts differ"
    assert np.array_equal(np.asarray(offsets), o["offsets"]), "offsets differ"
    assert np.array_equal(np.asarray(sorted_token)[:n], o["sorted_token"]), "sorted_token differs"
    assert np.array_equal(np.asarray(dest_pos), o["dest_pos"]), "dest_pos differs"
    assert int(dropped) == o["dropped"], "dropped differs"
    return n


def check_permute(xs_gpu, x, dest_pos, tokens=None):
    """Bit-exact: xs[dest_pos[t, j]] == x[t] (every slot of the given tokens)."""
    dp = np.asarray(dest_pos)
    if tokens is None:
        n = int(dp.max()) + 1 if dp.size and dp.max() >= 0 else 0
        want = oracle.permute(bits(x), dp, n)
        got = bits(xs_gpu[:n])
        written = np.unique(dp[dp >= 0])  # padding rows of a padded layout are not written
        assert np.array_equal(got[written], want[written]), "permute rows differ"
        return
    tokens = np.asarray(tokens)
    sub = dp[tokens]
    valid = sub >= 0
    pos = torch.as_tensor(sub[valid], device=xs_gpu.device, dtype=torch.long)
    got = bits(xs_gpu.index_select(0, pos))
    src = torch.as_tensor(np.repeat(tokens[:, None], dp.shape[1], 1)[valid], device=x.device,
                          dtype=torch.long)
    want = bits(x.index_select(0, src))
    assert np.array_equal(got, want), "permute rows differ"


def check_combine(out_gpu, y, topk_w, dest_pos, shared=None, tokens=None) -> float:
    """Returns the largest |g-o| / max(|o|, mag) seen (must be <= 1e-2)."""
    dp = np.asarray(dest_pos)
    w = np.asarray(topk_w, np.float32)
    T = dp.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    sub = dp[tokens]
    uniq = np.unique(sub[sub >= 0])
    remap = np.full(sub.shape, -1, np.int32)
    remap[sub >= 0] = np.searchsorted(uniq, sub[sub >= 0]).astype(np.int32)
    ysub = bits(y.index_select(0, torch.as_tensor(uniq, device=y.device, dtype=torch.long))) \
        if uniq.size else np.zeros((0, y.shape[1]), np.uint16)
    tt = torch.as_tensor(tokens, device=out_gpu.device, dtype=torch.long)
    sh = bits(shared.index_select(0, tt)) if shared is not None else None
    o, mag = oracle.combine(ysub if ysub.size else np.zeros((1, y.shape[1]), np.uint16),
                            w[tokens], remap, sh)
    g = bits_to_f64(bits(out_gpu.index_select(0, tt)))
    scale = np.maximum(np.abs(o), mag)
    ratio = np.abs(g - o) / np.where(scale > 0, scale, 1.0)
    worst = float(ratio.max()) if ratio.size else 0.0
    assert np.all(ratio <= COMBINE_RTOL), f"combine out of tolerance, worst {worst}"
    return worst


# ----------------------------------------------------------- expert FFN
# h  |g - o| <= 2^-8 |o| + (|u| + 1) dg + (|g| + 1) du, where dg, du =
#    1e-5 * sum_k |x_k w_k| bound the fp32 accumulation of the two products
#    (the activation's derivatives are below |u|+1 and |g|+1), and 2^-8 is one
#    bf16 rounding of h;
# y  |g - o| <= 2^-8 |o| + 1e-5 * sum_f |h_f w2_f|, fed with the device's h.
def abs_bits(b):
    return b & np.uint16(0x7FFF)


def _np(t):
    return None if t is None else t.cpu().numpy()


def check_expert_h(h, xs, offsets, w1, w3, b1, b3, act, rows):
    off = offsets.cpu().numpy()
    xb, w1b, w3b = bits(xs), bits(w1), bits(w3)
    o, g, u = oracle.expert_gate_up(xb, off, w1b, w3b, rows, act=act, b1=_np(b1), b3=_np(b3),
                                    want_pre=True)
    _, ga, ua = oracle.expert_gate_up(abs_bits(xb), off, abs_bits(w1b), abs_bits(w3b), rows,
                                      want_pre=True)
    got = bits_to_f64(bits(h)[rows])
    tol = 2.0 ** -8 * np.abs(o) + (np.abs(u) + 1) * 1e-5 * ga + (np.abs(g) + 1) * 1e-5 * ua
    bad = np.argwhere(np.abs(got - o) > tol)
    assert bad.size == 0, f"h: {len(bad)} values out of tolerance, first {bad[:5].tolist()}"


def check_expert_y(y, h, offsets, w2, b2, rows):
    off = offsets.cpu().numpy()
    hb, w2b = bits(h), bits(w2)
    o = oracle.expert_down(hb, off, w2b, rows, b2=_np(b2))
    mag = oracle.expert_down(abs_bits(hb), off, abs_bits(w2b), rows)
    got = bits_to_f64(bits(y)[rows])
    tol = 2.0 ** -8 * np.abs(o) + 1e-5 * mag
    bad = np.argwhere(np.abs(got - o) > tol)
    assert bad.size == 0, f"y: {len(bad)} values out of tolerance, first {bad[:5].tolist()}"
