"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
what the pages or the mathematics fix.  They are collected by
``test_oracle_pins.py`` and re-run against deliberately broken copies of the
oracle by ``test_oracle_mutants.py`` (every planted mistake must trip one).

Kinds of pin used here:
  * brute force on tiny inputs, written separately from the oracle: every
    subset of groups and of experts is enumerated and summed in exact rational
    arithmetic (the selection rule of "DeepSeek-V3.2-Exp - Select experts",
    applied literally as a two-stage maximisation);
  * hand-built worked cases of that page's rule (tests/golden);
  * closed forms of the scoring functions and library special cases (scipy's
    softmax / expit, numpy's bincount / cumsum / stable argsort, integer and
    torch fp64 matmul);
  * invariants: weights sum to route_scale when renormalised, k = E softmax is
    the full softmax, gpt-oss weights equal renormalised softmax weights,
    per-token k picks a prefix of the ranking ("Feature Request: dynamic
    number of experts"), the permutation is a bijection, and so on.
"""
from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

SCORE_NAMES = {"softmax": oracle.SOFTMAX, "sigmoid": oracle.SIGMOID,
               "sqrt_softplus": oracle.SQRT_SOFTPLUS, "topk_softmax": oracle.TOPK_SOFTMAX}


def _bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (inputs here are finite)."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def _rel_close(a, b, rtol, atol=0.0):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return bool(np.all(np.abs(a - b) <= rtol * np.abs(b) + atol))


# ------------------------------------------------------------------ brute force
def bf_scores(l, score):
    """Per-expert scores of one row, from Python's math module (not the oracle)."""
    if score == oracle.SOFTMAX:
        m = max(l)
        ex = [math.exp(v - m) for v in l]
        z = sum(ex)
        return [v / z for v in ex]
    if score == oracle.SIGMOID:
        return [1.0 / (1.0 + math.exp(-v)) for v in l]
    if score == oracle.SQRT_SOFTPLUS:
        return [math.sqrt(math.log1p(math.exp(v))) for v in l]
    return list(l)


def bf_select(keys, E, k, G, TG, topn):
    """Two-stage maximisation by enumeration, in exact arithmetic.

    Group score = max over topn-subsets of the group of the sum of keys; the
    kept groups = the TG-subset with the largest total group score; the
    selection = the k-subset of experts of kept groups with the largest total
    key.  Among equal totals the lexicographically smallest id tuple wins
    (itertools.combinations yields them in that order; only a strictly larger
    total replaces the incumbent).  Returns (ids ordered by key desc then id,
    kept group tuple)."""
    F = [Fraction(v) for v in keys]
    gsz = E // G
    if G > 1:
        gs = []
        for g in range(G):
            members = range(g * gsz, (g + 1) * gsz)
            gs.append(max(sum((F[i] for i in sub), Fraction(0))
                          for sub in itertools.combinations(members, topn)))
        best, kept_groups = None, None
        for sub in itertools.combinations(range(G), TG):
            s = sum((gs[g] for g in sub), Fraction(0))
            if best is None or s > best:
                best, kept_groups = s, sub
    else:
        kept_groups = (0,)
    cand = [e for e in range(E) if (e // gsz) in kept_groups]
    best, chosen = None, ()
    for sub in itertools.combinations(cand, k):
        s = sum((F[i] for i in sub), Fraction(0))
        if best is None or s > best:
            best, chosen = s, sub
    return sorted(chosen, key=lambda e: (-F[e], e)), kept_groups


def bf_weights(l, s, ids, score, renormalize, route_scale):
    if score == oracle.TOPK_SOFTMAX:
        m = max(l[e] for e in ids) if ids else 0.0
        ex = [math.exp(l[e] - m) for e in ids]
        z = sum(ex)
        w = [v / z for v in ex]
    else:
        w = [s[e] for e in ids]
    if renormalize and ids:
        z = sum(w)
        w = [v / z for v in w]
    return [v * route_scale for v in w]


BRUTE_COMBOS = [
    # E, k_max, G, TG, topn, score, bias, renormalize, route_scale, dynamic_k
    (8, 2, 1, 1, 1, oracle.SOFTMAX, False, True, 1.0, False),
    (12, 4, 1, 1, 1, oracle.SIGMOID, True, True, 2.5, False),
    (16, 4, 4, 2, 2, oracle.SIGMOID, True, True, 2.5, False),
    (16, 3, 4, 2, 1, oracle.SOFTMAX, False, False, 1.0, False),
    (12, 4, 2, 1, 2, oracle.SQRT_SOFTPLUS, True, True, 1.0, False),
    (8, 4, 1, 1, 1, oracle.TOPK_SOFTMAX, False, True, 1.0, False),
    (16, 4, 8, 3, 2, oracle.SQRT_SOFTPLUS, False, True, 1.5, False),
    (12, 4, 3, 2, 1, oracle.SOFTMAX, False, True, 1.0, True),
    (16, 5, 4, 3, 2, oracle.SIGMOID, True, False, 1.0, True),
]


def _brute_case(combo, rows, seed):
    E, k_max, G, TG, topn, score, has_bias, renorm, scale, dyn = combo
    rng = np.random.default_rng(seed)
    # A coarse grid makes equal logits (exact ties) common, so the tie rule is
    # exercised.  The grid is offset by 0.1 so that it is not symmetric about 0:
    # sigmoid(x) + sigmoid(-x) = 1 would otherwise make different groups tie in
    # real arithmetic, and such a tie is split by rounding, not by the rule.
    logits = (np.round(rng.normal(size=(rows, E)) * 4.0) / 4.0 + 0.1).astype(np.float32)
    bias = (rng.integers(-2, 3, size=E) * 0.05).astype(np.float32) if has_bias else None
    kpt = rng.integers(0, k_max + 1, size=rows).astype(np.int32) if dyn else None
    r = oracle.route(logits, k_max=k_max, score=score, bias=bias, k_per_token=kpt, n_groups=G,
                     topk_groups=TG, group_topn=topn, renormalize=renorm, route_scale=scale)
    assert r["status"] == oracle.OK, r["status"]
    for t in range(rows):
        l = [float(v) for v in logits[t]]
        s = bf_scores(l, score)
        keys = [s[e] + (float(bias[e]) if has_bias else 0.0) for e in range(E)]
        kt = int(kpt[t]) if dyn else k_max
        ids, kept = bf_select(keys, E, kt, G, TG, topn)
        got = [int(v) for v in r["ids"][t]]
        want = ids + [-1] * (k_max - kt)
        assert got == want, (combo, t, got, want, l)
        gsz = E // G
        assert all((e // gsz) in kept for e in ids)
        w = bf_weights(l, s, ids, score, renorm, scale) + [0.0] * (k_max - kt)
        assert _rel_close(r["w"][t], w, 1e-12, 1e-300), (combo, t, r["w"][t], w)


def pin_brute_force_selection():
    for i, combo in enumerate(BRUTE_COMBOS):
        _brute_case(combo, rows=120, seed=100 + i)


# -------------------------------------------------------------- golden cases
def pin_deepseek_worked_cases():
    with open(os.path.join(GOLDEN, "deepseek_select_cases.json")) as f:
        spec = json.load(f)
    for c in spec["cases"]:
        E = c["E"]
        logits = np.full((1, E), c["logit_base"], np.float32)
        for e, v in c["logit_set"].items():
            logits[0, int(e)] = v
        bias = None
        if c["bias_base"] is not None:
            bias = np.full((E,), c["bias_base"], np.float32)
            for e, v in c["bias_set"].items():
                bias[int(e)] = v
        score = SCORE_NAMES[c["score"]]
        r = oracle.route(logits, k_max=c["k"], score=score, bias=bias, n_groups=c["n_groups"],
                         topk_groups=c["topk_groups"], group_topn=c["group_topn"],
                         renormalize=c["renormalize"], route_scale=c["route_scale"],
                         want_keys=True)
        assert r["status"] == oracle.OK
        assert list(r["ids"][0]) == c["expected_ids"], (c["name"], list(r["ids"][0]))
        gsz = E // c["n_groups"]
        kept = sorted({g for g in range(c["n_groups"]) if np.isfinite(r["keys"][0, g * gsz])})
        assert kept == c["expected_kept_groups"], (c["name"], kept)
        lg = logits[0].astype(np.float64)
        sel = np.array(c["expected_ids"])
        if score == oracle.SIGMOID:
            s = 1.0 / (1.0 + np.exp(-lg[sel]))  # unbiased affinities of the selected experts
            want = s / s.sum() * c["route_scale"]
        else:
            p = np.exp(lg - lg.max())
            want = (p / p.sum())[sel] * c["route_scale"]
        assert _rel_close(r["w"][0], want, 1e-12), (c["name"], r["w"][0], want)
        if c["renormalize"]:
            assert abs(r["w"][0].sum() - c["route_scale"]) < 1e-12


# --------------------------------------------------------------- scores
def pin_score_closed_forms():
    ln3 = math.log(3.0)
    s = oracle.scores(np.array([[0.0, ln3, -ln3]], np.float32), oracle.SIGMOID)[0]
    l3 = float(np.float32(ln3))
    assert s[0] == 0.5
    assert abs(s[1] - 1.0 / (1.0 + math.exp(-l3))) < 1e-15 and abs(s[1] - 0.75) < 1e-7
    assert abs(s[1] + s[2] - 1.0) < 1e-15
    s = oracle.scores(np.array([[0.0, math.log(math.e - 1.0)]], np.float32),
                      oracle.SQRT_SOFTPLUS)[0]
    assert abs(s[0] - 0.8325546111576977) < 1e-15  # sqrt(ln 2)
    assert abs(s[1] - 1.0) < 1e-7  # softplus(ln(e-1)) = 1
    v = np.array([[-5.0, 5.0, -0.75, 0.75, 30.0, -30.0]], np.float32)
    s = oracle.scores(v, oracle.SQRT_SOFTPLUS)[0]
    for a, b, x in ((1, 0, 5.0), (3, 2, 0.75), (4, 5, 30.0)):
        assert abs((s[a] ** 2 - s[b] ** 2) - x) < 1e-13 * max(1.0, x)  # softplus(x)-softplus(-x)=x
    s = oracle.scores(np.zeros((1, 7), np.float32), oracle.SOFTMAX)[0]
    assert np.all(np.abs(s - 1.0 / 7.0) < 1e-16)
    s = oracle.scores(np.array([[0.0, math.log(2.0), math.log(5.0)]], np.float32),
                      oracle.SOFTMAX)[0]
    assert _rel_close(s, [1 / 8, 2 / 8, 5 / 8], 1e-7)
    lg = np.array([[1.5, -2.0, 0.25, 3.0]], np.float32)
    assert np.array_equal(oracle.scores(lg, oracle.TOPK_SOFTMAX)[0], lg[0].astype(np.float64))


def pin_score_library_cases():
    from scipy.special import expit, softmax
    rng = np.random.default_rng(7)
    lg = rng.normal(size=(50, 33)).astype(np.float32) * 3
    l64 = lg.astype(np.float64)
    assert _rel_close(oracle.scores(lg, oracle.SOFTMAX), softmax(l64, axis=1), 1e-13)
    assert _rel_close(oracle.scores(lg, oracle.SIGMOID), expit(l64), 1e-14)
    sp = np.sqrt(np.logaddexp(0.0, l64))
    assert _rel_close(oracle.scores(lg, oracle.SQRT_SOFTPLUS), sp, 1e-14)
    sh = oracle.scores(lg + np.float32(4.0), oracle.SOFTMAX)  # shift invariance
    assert _rel_close(sh, softmax(l64, axis=1), 1e-5)


# ------------------------------------------------------------ weight invariants
def pin_weight_invariants():
    rng = np.random.default_rng(11)
    lg = rng.normal(size=(64, 32)).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, size=32).astype(np.float32)
    for score in (oracle.SOFTMAX, oracle.SIGMOID, oracle.SQRT_SOFTPLUS, oracle.TOPK_SOFTMAX):
        r = oracle.route(lg, k_max=6, score=score, bias=b, n_groups=4, topk_groups=2,
                         group_topn=2, renormalize=True, route_scale=2.5)
        assert np.all(np.abs(r["w"].sum(1) - 2.5) < 1e-12), score
        r1 = oracle.route(lg, k_max=1, score=score, renormalize=True, route_scale=1.75)
        assert np.all(r1["w"][:, 0] == 1.75)
        assert np.array_equal(r1["ids"][:, 0], np.argmax(lg, axis=1))  # scores are monotone
    from scipy.special import softmax
    full = oracle.route(lg, k_max=32, score=oracle.SOFTMAX, renormalize=False)
    p = softmax(lg.astype(np.float64), axis=1)
    order = np.argsort(-lg, axis=1, kind="stable")
    assert np.array_equal(full["ids"], order)
    assert _rel_close(full["w"], np.take_along_axis(p, order, 1), 1e-13)
    # gpt-oss rule (softmax over the selected logits) = softmax over all, top-k, renormalised
    a = oracle.route(lg, k_max=4, score=oracle.TOPK_SOFTMAX, renormalize=False)
    c = oracle.route(lg, k_max=4, score=oracle.SOFTMAX, renormalize=True)
    assert np.array_equal(a["ids"], c["ids"])
    assert _rel_close(a["w"], c["w"], 1e-13)
    # sigmoid without renormalisation at k = 1: the weight is the raw sigmoid of the best logit
    s1 = oracle.route(lg, k_max=1, score=oracle.SIGMOID, renormalize=False)
    assert _rel_close(s1["w"][:, 0], 1.0 / (1.0 + np.exp(-lg.max(1).astype(np.float64))), 1e-14)


def pin_route_grouped():
    # Worked by hand: logits [5, 4, 3, 0, -1, -2], two groups of three, two
    # candidates per group, keep 3.  Flat top-3 would be 0, 1, 2; the groups
    # put expert 3 in place of 2.  Softmax weights over all six, renormalised
    # over the three kept: e^5, e^4, e^0 over their sum.
    lg = np.array([[5, 4, 3, 0, -1, -2]], np.float32)
    r = oracle.route_grouped(lg, k_max=3, score=oracle.SOFTMAX, n_groups=2, k_per_group=2)
    assert r["ids"].tolist() == [[0, 1, 3]]
    z = math.exp(5) + math.exp(4) + 1.0
    assert _rel_close(r["w"][0], np.array([math.exp(5) / z, math.exp(4) / z, 1.0 / z]), 1e-14)
    flat = oracle.route(lg, k_max=3, score=oracle.SOFTMAX)
    assert flat["ids"].tolist() == [[0, 1, 2]]
    # Brute force in plain Python: per group sort by (-score, id), then again.
    rng = np.random.default_rng(59)
    scores = {oracle.SOFTMAX: None, oracle.SIGMOID: lambda v: 1.0 / (1.0 + math.exp(-v)),
              oracle.SQRT_SOFTPLUS: lambda v: math.sqrt(max(v, 0.0) + math.log1p(math.exp(-abs(v)))),
              oracle.TOPK_SOFTMAX: lambda v: v}
    for E, G, kpg, k, sc, renorm, scale, integer in (
            (16, 4, 2, 5, oracle.SOFTMAX, True, 1.0, False), (16, 4, 2, 8, oracle.SIGMOID, False, 2.0, True),
            (24, 3, 3, 4, oracle.SQRT_SOFTPLUS, True, 1.5, False), (32, 8, 1, 8, oracle.TOPK_SOFTMAX, True, 1.0, True),
            (12, 1, 5, 5, oracle.SIGMOID, True, 1.0, False), (20, 5, 4, 3, oracle.SOFTMAX, False, 1.0, True)):
        lg = (rng.integers(-3, 4, size=(60, E)) if integer else rng.normal(size=(60, E))).astype(np.float32)
        r = oracle.route_grouped(lg, k_max=k, score=sc, n_groups=G, k_per_group=kpg,
                                 renormalize=renorm, route_scale=scale)
        gsz = E // G
        for t in range(lg.shape[0]):
            row = [float(v) for v in lg[t]]
            if sc == oracle.SOFTMAX:
                m = max(row)
                z = sum(math.exp(v - m) for v in row)
                sv = [math.exp(v - m) / z for v in row]
            else:
                sv = [scores[sc](v) for v in row]
            cand = []
            for g in range(G):
                members = sorted(range(g * gsz, (g + 1) * gsz), key=lambda e: (-sv[e], e))
                cand += members[:kpg]
            pick = sorted(cand, key=lambda e: (-sv[e], e))[:k]
            assert r["ids"][t].tolist() == pick, (t, r["ids"][t], pick)
            if sc == oracle.TOPK_SOFTMAX:
                m = max(row[e] for e in pick)
                ww = [math.exp(row[e] - m) for e in pick]
            else:
                ww = [sv[e] for e in pick]
            if renorm:
                tot = sum(ww)
                ww = [v / tot for v in ww]
            assert _rel_close(r["w"][t], np.array(ww) * scale, 1e-12)
        if kpg == gsz or G == 1:  # every expert is a candidate: the flat router
            f = oracle.route(lg, k_max=k, score=sc, renormalize=renorm, route_scale=scale)
            assert np.array_equal(f["ids"], r["ids"])


def pin_dynamic_k_prefix():
    """Per-token k picks a prefix of the same ranking; nothing else changes."""
    rng = np.random.default_rng(12)
    lg = rng.normal(size=(80, 64)).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, size=64).astype(np.float32)
    kpt = rng.choice([0, 1, 4, 8, 16], size=80).astype(np.int32)
    full = oracle.route(lg, k_max=16, score=oracle.SIGMOID, bias=b, n_groups=8, topk_groups=4,
                        group_topn=2, renormalize=False, route_scale=1.0)
    dyn = oracle.route(lg, k_max=16, score=oracle.SIGMOID, bias=b, n_groups=8, topk_groups=4,
                       group_topn=2, renormalize=False, route_scale=1.0, k_per_token=kpt)
    for t in range(80):
        k = kpt[t]
        assert np.array_equal(dyn["ids"][t, :k], full["ids"][t, :k])
        assert np.all(dyn["ids"][t, k:] == -1) and np.all(dyn["w"][t, k:] == 0.0)
        assert np.array_equal(dyn["w"][t, :k], full["w"][t, :k])


def pin_weights_for_ids():
    """Weights of a selection made elsewhere ("DeepSeek-V3.2-Exp - Select
    experts", gate forward: gather the unbiased scores of the chosen experts,
    divide by their sum, times route_scale; "Crate ferrox_moe",
    route_top_k_softmax_weight: softmax over the chosen logits).

    (1) Against Python's math module (bf_weights) on arbitrary id lists: slots
        in any order, -1 holes anywhere, all four scores, with and without
        renormalisation, several route_scales.
    (2) On the router's own selections (bias, groups, per-token k), the weights
        of the chosen ids are the router's weights, bit for bit: the bias only
        selects, it never weighs.
    (3) An id >= E is refused."""
    rng = np.random.default_rng(21)
    for score in (oracle.SOFTMAX, oracle.SIGMOID, oracle.SQRT_SOFTPLUS, oracle.TOPK_SOFTMAX):
        for renorm, scale in ((True, 2.5), (False, 1.0), (True, 1.0), (False, 0.75)):
            T, E, k_max = 40, 13, 5
            lg = (rng.normal(size=(T, E)) * 2.0).astype(np.float32)
            ids = np.full((T, k_max), -1, np.int32)
            for t in range(T):
                n = int(rng.integers(0, k_max + 1))
                chosen = rng.permutation(E)[:n]            # any experts, any order
                slots = np.sort(rng.permutation(k_max)[:n])  # holes anywhere
                ids[t, slots] = chosen
            w = oracle.weights_for_ids(lg, ids, score=score, renormalize=renorm,
                                       route_scale=scale)
            for t in range(T):
                l = [float(v) for v in lg[t]]
                s = bf_scores(l, score)
                live = [j for j in range(k_max) if ids[t, j] >= 0]
                want = bf_weights(l, s, [int(ids[t, j]) for j in live], score, renorm, scale)
                exp = np.zeros(k_max)
                exp[live] = want
                assert _rel_close(w[t], exp, 1e-12, 1e-300), (score, renorm, t, w[t], exp)
    # (2) the router's selections, weighed again
    T, E = 96, 64
    lg = rng.normal(size=(T, E)).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, size=E).astype(np.float32)
    kpt = rng.choice([0, 1, 3, 6, 8], size=T).astype(np.int32)
    for score in (oracle.SOFTMAX, oracle.SIGMOID, oracle.SQRT_SOFTPLUS, oracle.TOPK_SOFTMAX):
        for bias, G, TG, topn, kp, renorm, scale in (
                (b, 8, 4, 2, None, True, 2.5), (None, 1, 1, 1, kpt, True, 1.0),
                (b, 4, 2, 2, kpt, False, 1.0), (None, 8, 3, 1, None, False, 1.5)):
            r = oracle.route(lg, k_max=8, score=score, bias=bias, k_per_token=kp, n_groups=G,
                             topk_groups=TG, group_topn=topn, renormalize=renorm,
                             route_scale=scale)
            w = oracle.weights_for_ids(lg, r["ids"], score=score, renormalize=renorm,
                                       route_scale=scale)
            assert np.array_equal(w, r["w"]), (score, G, renorm)
            # a permutation of the slots permutes the weights and nothing else
            perm = rng.permutation(8)
            wp = oracle.weights_for_ids(lg, r["ids"][:, perm], score=score, renormalize=renorm,
                                        route_scale=scale)
            assert _rel_close(wp, r["w"][:, perm], 1e-13, 1e-300), (score, G, renorm)
    # (3) an id past the last expert
    import ctypes
    bad = np.array([[0, 3]], np.int32)
    lg1 = np.zeros((1, 3), np.float32)
    out = np.empty((1, 2), np.float64)
    st = oracle._load().oracle_weights_for_ids(lg1.ctypes.data, bad.ctypes.data, 1, 3, 2,
                                              oracle.SOFTMAX, 1, ctypes.c_double(1.0),
                                              out.ctypes.data)
    assert st == oracle.ERR_INDEX, st


def pin_status_and_nan():
    lg = np.array([[0.5, np.nan, 2.0, -1.0]], np.float32)
    r = oracle.route(lg, k_max=3, score=oracle.SIGMOID, renormalize=False)
    assert r["status"] == oracle.ERR_NAN
    assert list(r["ids"][0]) == [2, 0, 3]
    r = oracle.route(lg, k_max=4, score=oracle.TOPK_SOFTMAX, renormalize=False)
    assert list(r["ids"][0]) == [2, 0, 3, 1]
    ok = np.zeros((2, 4), np.float32)
    r = oracle.route(ok, k_max=2, score=oracle.SOFTMAX, k_per_token=np.array([1, 3], np.int32))
    assert r["status"] == oracle.ERR_ARG
    r = oracle.route(np.array([[0.0, -0.0, 0.0]], np.float32), k_max=3, score=oracle.TOPK_SOFTMAX)
    assert list(r["ids"][0]) == [0, 1, 2]  # -0 and +0 tie, lower id first


# --------------------------------------------------------------------- gate
def pin_gate_integer_exact():
    rng = np.random.default_rng(21)
    for T, d, E in ((5, 24, 3), (9, 2048, 16), (3, 64, 96)):
        xi = rng.integers(-4, 5, size=(T, d))
        wi = rng.integers(-4, 5, size=(E, d))
        got = oracle.gate_rows(_bf16_bits_from_f32(xi.astype(np.float32)),
                               _bf16_bits_from_f32(wi.astype(np.float32)))
        assert np.array_equal(got, (xi @ wi.T).astype(np.float64)), (T, d, E)
    rows = np.array([4, 0, 2], np.int64)
    xi = rng.integers(-4, 5, size=(5, 40))
    wi = rng.integers(-4, 5, size=(7, 40))
    got = oracle.gate_rows(_bf16_bits_from_f32(xi.astype(np.float32)),
                           _bf16_bits_from_f32(wi.astype(np.float32)), rows)
    assert np.array_equal(got, (xi[rows] @ wi.T).astype(np.float64))


def pin_gate_torch_fp64():
    import torch
    rng = np.random.default_rng(22)
    x = _bf16_bits_from_f32(rng.normal(size=(17, 200)).astype(np.float32))
    w = _bf16_bits_from_f32((rng.normal(size=(24, 200)) * 0.02).astype(np.float32))
    xf, wf = _bits_to_f64(x), _bits_to_f64(w)
    ref = (torch.from_numpy(xf) @ torch.from_numpy(wf).T).numpy()
    got = oracle.gate_rows(x, w)
    assert np.all(np.abs(got - ref) <= 1e-13 * (np.abs(xf) @ np.abs(wf).T))


# ------------------------------------------------------------------- hash
def pin_hash_lookup():
    rng = np.random.default_rng(31)
    vocab, k, E, T = 1000, 6, 384, 300
    table = rng.integers(0, E, size=(vocab, k)).astype(np.int32)
    table[5] = [7, 7, 3, 9, 7, 1]  # repeated ids keep every slot
    tok = rng.integers(0, vocab, size=T).astype(np.int32)
    tok[:3] = 5
    r = oracle.hash_route(tok, table, num_experts=E, route_scale=2.0)
    assert r["status"] == oracle.OK
    assert np.array_equal(r["ids"], table[tok])
    assert np.all(r["w"] == 2.0 / k)
    lg = rng.normal(size=(T, E)).astype(np.float32)
    r = oracle.hash_route(tok, table, num_experts=E, logits=lg, score=oracle.SOFTMAX,
                          renormalize=True, route_scale=1.0)
    ex = np.exp(np.take_along_axis(lg.astype(np.float64), table[tok].astype(np.int64), 1))
    assert _rel_close(r["w"], ex / ex.sum(1, keepdims=True), 1e-12)
    r = oracle.hash_route(tok, table, num_experts=E, logits=lg, score=oracle.SIGMOID,
                          renormalize=False, route_scale=1.0)
    l_sel = np.take_along_axis(lg.astype(np.float64), table[tok].astype(np.int64), 1)
    assert _rel_close(r["w"], 1.0 / (1.0 + np.exp(-l_sel)), 1e-14)
    bad = tok.copy()
    bad[10] = vocab
    r = oracle.hash_route(bad, table, num_experts=E)
    assert r["status"] == oracle.ERR_INDEX and np.all(r["ids"][10] == -1)
    assert np.all(r["w"][10] == 0.0) and np.array_equal(r["ids"][11], table[bad[11]])


# ---------------------------------------------------------------- dispatch
def pin_dispatch_library():
    rng = np.random.default_rng(41)
    for T, k_max, E in ((1, 1, 1), (37, 4, 8), (500, 8, 64), (300, 16, 128)):
        ids = rng.integers(0, E, size=(T, k_max)).astype(np.int32)
        ids[rng.random(size=(T, k_max)) < 0.2] = -1
        r = oracle.dispatch(ids, E)
        assert r["status"] == oracle.OK
        flat = ids.reshape(-1)
        valid = np.nonzero(flat >= 0)[0]
        assert np.array_equal(r["counts"], np.bincount(flat[valid], minlength=E))
        assert np.array_equal(r["offsets"], np.concatenate([[0], np.cumsum(r["counts"])]))
        order = valid[np.argsort(flat[valid], kind="stable")]
        assert np.array_equal(r["sorted_token"], order // k_max)
        dp = r["dest_pos"].reshape(-1)
        assert np.array_equal(np.sort(dp[valid]), np.arange(valid.size))  # bijection
        assert np.all(dp[flat < 0] == -1)
        assert np.array_equal(dp[order], np.arange(valid.size))
        for e in range(E):
            seg = r["sorted_token"][r["offsets"][e]:r["offsets"][e + 1]]
            assert np.all(np.diff(seg) >= 0)
    r = oracle.dispatch(np.array([[0, 5], [1, -1]], np.int32), 4)
    assert r["status"] == oracle.ERR_INDEX


def pin_dispatch_limited():
    # Worked by hand: six top-1 tokens on three experts, capacity 2, blocks
    # padded to 4 rows.  Expert 0 is asked for by tokens 0, 2, 3, 5 and keeps
    # the first two; experts 1 and 2 keep their one token each.
    ids = np.array([[0], [1], [0], [0], [2], [0]], np.int32)
    r = oracle.dispatch_limited(ids, 3, capacity=2, pad=4)
    assert r["status"] == oracle.OK and r["dropped"] == 2
    assert r["counts"].tolist() == [4, 1, 1]
    assert r["offsets"].tolist() == [0, 4, 8, 12]
    assert r["sorted_token"].tolist() == [0, 2, -1, -1, 1, -1, -1, -1, 4, -1, -1, -1]
    assert r["dest_pos"].reshape(-1).tolist() == [0, 4, 1, -1, 8, -1]
    # Brute force: each expert's kept slots are its first `cap` in flat order.
    rng = np.random.default_rng(43)
    for T, k_max, E, cap, pad in ((1, 1, 1, 0, 1), (40, 2, 5, 7, 1), (300, 4, 16, 50, 8),
                                  (500, 8, 64, 0, 128), (257, 1, 8, 20, 16), (64, 6, 12, 1, 3)):
        ids = rng.integers(0, E, size=(T, k_max)).astype(np.int32)
        ids[rng.random(size=(T, k_max)) < 0.15] = -1
        r = oracle.dispatch_limited(ids, E, capacity=cap, pad=pad)
        flat = ids.reshape(-1)
        dp = r["dest_pos"].reshape(-1)
        st = r["sorted_token"]
        base, dropped = 0, 0
        for e in range(E):
            slots = np.nonzero(flat == e)[0]
            assert r["counts"][e] == slots.size
            keep = slots if cap <= 0 else slots[:cap]
            dropped += slots.size - keep.size
            block = -(-keep.size // pad) * pad
            assert r["offsets"][e] == base and r["offsets"][e + 1] == base + block
            assert np.array_equal(st[base:base + keep.size], keep // k_max)
            assert np.all(st[base + keep.size:base + block] == -1)
            assert np.array_equal(dp[keep], base + np.arange(keep.size))
            assert np.all(dp[slots[keep.size:]] == -1)
            base += block
        assert r["dropped"] == dropped and st.size == base
        assert np.all(dp[flat < 0] == -1)
        if cap <= 0 and pad == 1:  # no limit, no padding: the plain dispatch
            q = oracle.dispatch(ids, E)
            for key in ("counts", "offsets", "sorted_token", "dest_pos"):
                assert np.array_equal(r[key], q[key])
    r = oracle.dispatch_limited(np.array([[0, 5], [1, -1]], np.int32), 4, capacity=1, pad=2)
    assert r["status"] == oracle.ERR_INDEX


def pin_ep_layout():
    # Worked by hand: 2 ranks, 4 experts (rank 0 owns 0-1, rank 1 owns 2-3),
    # 3 tokens x 2 slots each.  Owner 0 receives expert 0 from rank 0 (slots
    # 0, 5) then rank 1 (slot 2), then expert 1 from rank 0 (slot 4) and rank 1
    # (slot 1); owner 1 receives expert 2 (rank 0 slot 2, rank 1 slot 3), then
    # expert 3 (rank 0 slot 1, rank 1 slots 0, 4, 5).
    ids = np.array([[[0, 3], [2, -1], [1, 0]], [[3, 1], [0, 2], [3, 3]]], np.int32)
    r = oracle.ep_layout(ids, 4)
    assert r["status"] == oracle.OK
    assert r["dest_rank"].tolist() == [[[0, 1], [1, -1], [0, 0]], [[1, 0], [0, 1], [1, 1]]]
    assert r["dest_row"].tolist() == [[[0, 2], [0, -1], [3, 1]], [[3, 4], [2, 1], [4, 5]]]
    assert r["recv_rows"].tolist() == [5, 6]
    # One rank: the plain dispatch.  Several: the order of a sort by
    # (expert, source rank, flat slot) restricted to each owner.
    rng = np.random.default_rng(47)
    for G, T, k_max, E in ((1, 50, 3, 8), (2, 40, 2, 8), (4, 64, 4, 16), (8, 33, 6, 64)):
        ids = rng.integers(0, E, size=(G, T, k_max)).astype(np.int32)
        ids[rng.random(size=ids.shape) < 0.1] = -1
        r = oracle.ep_layout(ids, E)
        if G == 1:
            assert np.array_equal(r["dest_row"][0], oracle.dispatch(ids[0], E)["dest_pos"])
        el = E // G
        src_r, src_a = np.nonzero(ids.reshape(G, -1) >= 0)
        e = ids.reshape(G, -1)[src_r, src_a]
        order = np.lexsort((src_a, src_r, e))
        owner = e[order] // el
        for d in range(G):
            mine = order[owner == d]
            rows = r["dest_row"].reshape(G, -1)[src_r[mine], src_a[mine]]
            assert np.array_equal(rows, np.arange(mine.size))
            assert np.all(r["dest_rank"].reshape(G, -1)[src_r[mine], src_a[mine]] == d)
            assert r["recv_rows"][d] == mine.size
        assert np.all(r["dest_rank"][ids < 0] == -1) and np.all(r["dest_row"][ids < 0] == -1)
    # The exchange round trip: identity experts (y = received x) and weights
    # summing to 1 give every token back exactly.
    G, T, k_max, E, d = 4, 24, 3, 16, 16
    ids = np.stack([np.stack([rng.permutation(E)[:k_max] for _ in range(T)]) for _ in range(G)])
    r = oracle.ep_layout(ids.astype(np.int32), E)
    x = _bf16_bits_from_f32(rng.normal(size=(G, T, d)).astype(np.float32))
    recv = oracle.ep_permute(x, r["dest_rank"], r["dest_row"], r["recv_rows"])
    w = np.full((G, T, k_max), 0.25, np.float32)
    w[..., 0] = 0.5
    outs = oracle.ep_combine(recv, w, r["dest_rank"], r["dest_row"], want_mag=False)
    for g in range(G):
        assert np.array_equal(outs[g], _bits_to_f64(x[g]))


def pin_expert_ffn():
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    # Activation closed forms through 1-wide experts: xs = [1], so g = w1, u = w3.
    off = np.array([0, 1], np.int32)
    one = _bf16_bits_from_f32(np.array([[1.0] + [0.0] * 15], np.float32))
    for act, g, u, want in ((oracle.SWIGLU, 0.0, 5.0, 0.0),
                            (oracle.SWIGLU, 2.0, 3.0, 2.0 * sig(2.0) * 3.0),
                            (oracle.SWIGLU_OAI, 10.0, 2.0, 7.0 * sig(1.702 * 7.0) * 3.0),
                            (oracle.SWIGLU_OAI, 3.0, -20.0, 3.0 * sig(1.702 * 3.0) * -6.0),
                            (oracle.SWIGLU_OAI, -20.0, 1.0, -20.0 * sig(-1.702 * 20.0) * 2.0),
                            (oracle.SWIGLU_OAI, 1.0, -1.0, 0.0)):
        w1 = _bf16_bits_from_f32(np.array([[[g] + [0.0] * 15]], np.float32))
        w3 = _bf16_bits_from_f32(np.array([[[u] + [0.0] * 15]], np.float32))
        h = oracle.expert_gate_up(one, off, w1, w3, [0], act=act)
        assert abs(h[0, 0] - want) <= 1e-14 * max(1.0, abs(want)), (act, g, u, h[0, 0], want)
    # Integer-valued operands: the products are exact, so g, u and y equal an
    # integer matmul; each row uses the weights of the block holding it.
    rng = np.random.default_rng(67)
    E, d, F = 3, 16, 8
    offsets = np.array([0, 4, 4, 9], np.int32)  # expert 1 holds no rows
    R = 9
    xi = rng.integers(-3, 4, size=(R, d))
    w1i = rng.integers(-2, 3, size=(E, F, d))
    w3i = rng.integers(-2, 3, size=(E, F, d))
    w2i = rng.integers(-2, 3, size=(E, d, F))
    b1 = rng.integers(-4, 5, size=(E, F)).astype(np.float32)
    b3 = rng.integers(-4, 5, size=(E, F)).astype(np.float32)
    b2 = rng.integers(-4, 5, size=(E, d)).astype(np.float32)
    bits = lambda a: _bf16_bits_from_f32(a.astype(np.float32))  # noqa: E731
    rows = np.arange(R)
    for act in (oracle.SWIGLU, oracle.SWIGLU_OAI):
        h, g, u = oracle.expert_gate_up(bits(xi), offsets, bits(w1i), bits(w3i), rows, act=act,
                                        b1=b1, b3=b3, want_pre=True)
        for r in rows:
            e = 0 if r < 4 else 2
            gi = w1i[e] @ xi[r] + b1[e]
            ui = w3i[e] @ xi[r] + b3[e]
            assert np.array_equal(g[r], gi) and np.array_equal(u[r], ui)
            for f in range(F):
                gv, uv = float(gi[f]), float(ui[f])
                if act == oracle.SWIGLU:
                    want = gv * sig(gv) * uv
                else:
                    gc, uc = min(gv, 7.0), min(max(uv, -7.0), 7.0)
                    want = gc * sig(1.702 * gc) * (uc + 1.0)
                assert abs(h[r, f] - want) <= 1e-12 * max(1.0, abs(want))
    hi = rng.integers(-3, 4, size=(R, F))
    y = oracle.expert_down(bits(hi), offsets, bits(w2i), rows, b2=b2)
    for r in rows:
        e = 0 if r < 4 else 2
        assert np.array_equal(y[r], w2i[e] @ hi[r] + b2[e])
    try:
        oracle.expert_down(bits(hi), offsets, bits(w2i), [R])  # row past the last block
        raise AssertionError("a row outside every block must be refused")
    except ValueError:
        pass


# ---------------------------------------------------------------- permute
def pin_permute_copy():
    rng = np.random.default_rng(51)
    T, k_max, E, d = 40, 3, 6, 24
    ids = rng.integers(0, E, size=(T, k_max)).astype(np.int32)
    ids[::7, 2] = -1
    r = oracle.dispatch(ids, E)
    x = rng.integers(0, 1 << 16, size=(T, d)).astype(np.uint16)
    n = int(r["offsets"][-1])
    xs = oracle.permute(x, r["dest_pos"], n)
    assert np.array_equal(xs, x[r["sorted_token"]])


# ---------------------------------------------------------------- combine
def pin_combine_cases():
    rng = np.random.default_rng(61)
    T, k_max, d = 30, 4, 16
    N = T * k_max
    y = _bf16_bits_from_f32(rng.normal(size=(N, d)).astype(np.float32))
    sh = _bf16_bits_from_f32(rng.normal(size=(T, d)).astype(np.float32))
    dp = rng.permutation(N).astype(np.int32).reshape(T, k_max)
    dp[::5, 3] = -1
    onehot = np.zeros((T, k_max), np.float32)
    pick = rng.integers(0, 3, size=T)
    onehot[np.arange(T), pick] = 1.0
    out = oracle.combine(y, onehot, dp, want_mag=False)
    assert np.array_equal(out, _bits_to_f64(y)[dp[np.arange(T), pick]])
    zero = np.zeros((T, k_max), np.float32)
    assert np.array_equal(oracle.combine(y, zero, dp, sh, want_mag=False), _bits_to_f64(sh))
    # padded slots are skipped even if their weight is not zero
    wbig = rng.uniform(0.5, 1.5, size=(T, k_max)).astype(np.float32)
    yc = _bf16_bits_from_f32(np.repeat(rng.integers(-8, 9, size=(N, 1)), d, 1).astype(np.float32))
    out, mag = oracle.combine(yc, wbig, dp, sh)
    yv = _bits_to_f64(yc)[:, 0]
    for t in range(T):
        want = sum(float(wbig[t, j]) * yv[dp[t, j]] for j in range(k_max) if dp[t, j] >= 0)
        assert np.allclose(out[t] - _bits_to_f64(sh)[t], want, rtol=1e-12, atol=1e-12)
    assert np.all(mag >= np.abs(out) - 1e-12)
    # identity experts (y = permuted x) with weights summing to s give s * x
    ids = np.stack([rng.permutation(8)[:k_max] for _ in range(T)]).astype(np.int32)
    r = oracle.dispatch(ids, 8)
    x = _bf16_bits_from_f32(rng.normal(size=(T, d)).astype(np.float32))
    xs = oracle.permute(x, r["dest_pos"], int(r["offsets"][-1]))
    w = np.full((T, k_max), 0.625, np.float32)  # sums to 2.5, exactly representable
    out = oracle.combine(xs, w, r["dest_pos"], want_mag=False)
    assert np.array_equal(out, 2.5 * _bits_to_f64(x))


PINS = [pin_score_closed_forms, pin_score_library_cases, pin_status_and_nan,
        pin_gate_integer_exact, pin_gate_torch_fp64, pin_hash_lookup, pin_dispatch_library,
        pin_dispatch_limited, pin_ep_layout, pin_route_grouped, pin_expert_ffn,
        pin_permute_copy, pin_combine_cases, pin_weight_invariants, pin_weights_for_ids,
        pin_dynamic_k_prefix, pin_deepseek_worked_cases, pin_brute_force_selection]


def run_all(stop_at_first: bool = True) -> list[str]:
    """Names of the pins that fail (all of them run unless stop_at_first)."""
    failed = []
    for p in PINS:
        try:
            p()
        except Exception as exc:  # noqa: BLE001 - any failure counts as a caught mistake
            failed.append(f"{p.__name__}: {type(exc).__name__}")
            if stop_at_first:
                break
    return failed
