"""Stage-by-stage parity of the CUDA path with the oracle on small and edge
shapes: ragged tiles, scalar and vector layouts, maximum sizes, empty inputs,
ties, NaN, out-of-range ids.  All calls go through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_moe_b200 as moe
from gpu_check import (bits, check_combine, check_dispatch, check_gate, check_permute,
                       check_route)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


# ------------------------------------------------------------------ gate GEMM
@pytest.mark.parametrize("T,d,E", [(1, 64, 128), (300, 200, 8), (257, 2048, 128),
                                   (129, 512, 30), (200, 1024, 256), (131, 7168, 384),
                                   (140, 256, 512), (128, 8, 16), (333, 128, 300)])
def test_gate_gemm_integer_exact(T, d, E):
    """Integer-valued x, W in [-4, 4]: every product and partial sum is exact in
    fp32, so the logits must equal the oracle bit for bit whatever the order."""
    g = _gen(T * 7 + d + E)
    x = torch.randint(-4, 5, (T, d), generator=g, device=DEV).to(torch.bfloat16)
    w = torch.randint(-4, 5, (E, d), generator=g, device=DEV).to(torch.bfloat16)
    logits = torch.full((T, E), float("nan"), device=DEV)
    st = _status()
    moe.moe_gate_gemm(x, w, logits, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    o = oracle.gate_rows(bits(x), bits(w))
    assert np.array_equal(logits.cpu().numpy().astype(np.float64), o)


@pytest.mark.parametrize("T,d,E", [(515, 2048, 128), (300, 7168, 256), (260, 7168, 384)])
def test_gate_gemm_random(T, d, E):
    g = _gen(T + d + E)
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    w = (torch.randn((E, d), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    logits = torch.empty((T, E), device=DEV)
    moe.moe_gate_gemm(x, w, logits)
    torch.cuda.synchronize()
    check_gate(logits, x, w)


@pytest.mark.parametrize("T,d,E", [(20000, 512, 384), (19500, 256, 300), (40000, 256, 256),
                                   (30001, 128, 128)])
def test_gate_gemm_several_waves(T, d, E):
    """More tiles than SMs (two CTAs per SM where the accumulator takes at most
    half the TMEM): every logit is written, and sampled rows (the first and
    last tiles included) match the oracle."""
    g = _gen(T + d + E)
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    w = (torch.randn((E, d), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    logits = torch.full((T, E), float("nan"), device=DEV)
    moe.moe_gate_gemm(x, w, logits)
    torch.cuda.synchronize()
    assert not torch.isnan(logits).any()
    rows = np.unique(np.concatenate([np.arange(130), np.arange(T - 130, T),
                                     np.random.default_rng(T).choice(T, 600, replace=False)]))
    check_gate(logits, x, w, rows)


def test_gate_gemm_validation():
    x = torch.zeros((4, 12), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((4, 12), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moe.MoeError):
        moe.moe_gate_gemm(x, w, torch.empty((4, 4), device=DEV))  # d % 8 != 0
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    moe.moe_gate_gemm(x, torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV),
                      torch.empty((0, 4), device=DEV))  # T = 0 is a no-op


# ---------------------------------------------------------------------- route
ROUTE_CASES = [
    # E, k_max, score, bias, G, TG, topn, renorm, scale, dyn
    (8, 2, "softmax", False, 1, 1, 1, True, 1.0, False),
    (128, 16, "softmax", False, 1, 1, 1, True, 1.0, True),
    (128, 8, "softmax", False, 1, 1, 1, False, 1.0, False),
    (256, 8, "sigmoid", True, 8, 4, 2, True, 2.5, False),
    (256, 8, "sigmoid", False, 8, 4, 1, True, 1.0, False),
    (384, 6, "sqrt_softplus", False, 1, 1, 1, True, 1.0, False),
    (384, 6, "sqrt_softplus", True, 4, 2, 2, True, 1.5, False),
    (128, 1, "sigmoid", False, 1, 1, 1, False, 1.0, False),
    (128, 4, "topk_softmax", False, 1, 1, 1, True, 1.0, False),
    (128, 4, "topk_softmax", True, 1, 1, 1, False, 1.0, False),
    (30, 5, "softmax", True, 3, 2, 2, True, 1.0, True),      # scalar layout, odd groups
    (7, 7, "sigmoid", False, 1, 1, 1, True, 1.0, False),      # k = E
    (512, 32, "softmax", False, 1, 1, 1, True, 1.0, False),   # maximum E and k
    (512, 32, "sigmoid", True, 32, 8, 2, True, 1.0, True),    # 32 groups of 16
    (96, 12, "sqrt_softplus", False, 6, 4, 2, False, 2.0, True),
]


@pytest.mark.parametrize("case", ROUTE_CASES, ids=lambda c: "-".join(map(str, c)))
def test_route_parity(case):
    E, k_max, score, has_bias, G, TG, topn, renorm, scale, dyn = case
    T = 1003
    g = _gen(E * 31 + k_max)
    logits = torch.randn((T, E), generator=g, device=DEV) * 2
    logits[::17] = torch.round(logits[::17] * 2) / 2  # rows with many exact ties
    logits[5] = 0.0                                   # a row where every key ties
    bias = (torch.rand((E,), generator=g, device=DEV) * 0.2 - 0.1) if has_bias else None
    if dyn == "seg":
        kpt = _seg_k(T, k_max)
    else:
        kpt = torch.randint(0, k_max + 1, (T,), generator=g, device=DEV,
                            dtype=torch.int32) if dyn else None
    p = moe.RouteParams.make(E, k_max, score, G, TG, topn, renorm, scale)
    ids = torch.full((T, k_max), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k_max), 7.0, device=DEV)
    st = _status()
    moe.moe_route(logits, bias, kpt, p, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    r = check_route(ids.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy(), k_max=k_max,
                    score=score, bias=None if bias is None else bias.cpu().numpy(),
                    kpt=None if kpt is None else kpt.cpu().numpy(), n_groups=G, topk_groups=TG,
                    group_topn=topn, renormalize=renorm, route_scale=scale)
    print(case, r)


NEAR_TIE_CASES = [
    # E, k_max, score, G, TG, topn, logit step giving keys about 2e-5 apart (relative)
    (128, 4, "topk_softmax", 1, 1, 1, 8e-5),     # keys are the logits
    (128, 8, "softmax", 1, 1, 1, 8e-5),
    (256, 8, "sigmoid", 8, 4, 2, 1.1e-3),        # deepseek-v3 layout, scored keys
    (384, 6, "sqrt_softplus", 4, 2, 2, 1.6e-4),
]


@pytest.mark.parametrize("case", NEAR_TIE_CASES, ids=lambda c: "-".join(map(str, c)))
def test_route_prefix_near_ties(case):
    """Rows whose leading experts' keys are 2e-5 apart: closer than the 2^-14
    relative resolution of the 23-bit key prefix of the selection words, so
    the rows tie on prefixes and are ordered again on the whole key; wider
    than the 1e-6 near-tie band, so the order must be exactly the oracle's."""
    E, k_max, score, G, TG, topn, step = case
    T = 515
    g = _gen(E + k_max * 7)
    logits = torch.randn((T, E), generator=g, device=DEV)
    rows = torch.arange(0, T, 3, device=DEV)
    for t in rows.tolist():
        who = torch.randperm(E, generator=g, device=DEV)[:12]  # ids in random order
        logits[t, who] = 4.0 + step * torch.arange(12, device=DEV, dtype=torch.float32)
    p = moe.RouteParams.make(E, k_max, score, G, TG, topn, True, 1.0)
    ids = torch.full((T, k_max), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k_max), 7.0, device=DEV)
    st = _status()
    moe.moe_route(logits, None, None, p, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    lg = logits.cpu().numpy()
    if score in ("topk_softmax", "softmax"):  # keys are the logits: count prefix ties
        u = lg.view(np.uint32)
        img = np.where(u >> 31, ~u, u | np.uint32(0x80000000)) >> 9
        top = np.sort(img, axis=1)[:, ::-1][:, :k_max + 1]
        tied = (np.diff(top, axis=1) == 0).any(axis=1)
        assert tied[::3].mean() > 0.5
    # (a swap is accepted only below a 1e-6 relative key gap: never between
    # the crafted experts)
    check_route(ids.cpu().numpy(), w.cpu().numpy(), lg, k_max=k_max, score=score,
                n_groups=G, topk_groups=TG, group_topn=topn, renormalize=True)


@pytest.mark.parametrize("spread", [50.0, 1e-3])
def test_route_fixed_point_words_bias_range(spread):
    """Sigmoid keys with a bias spread far wider (50) and far narrower (1e-3)
    than the scores: the fixed-point selection words scale to the bias range,
    so their step is coarse in the first case (many prefix ties, settled by the
    exact routine) and fine in the second."""
    T, E, k = 1003, 256, 8
    g = _gen(int(spread * 1000) + 7)
    logits = torch.randn((T, E), generator=g, device=DEV) * 2
    bias = (torch.rand((E,), generator=g, device=DEV) * 2 - 1) * spread
    bias[::37] = bias[0]  # some equal biases
    p = moe.RouteParams.make(E, k, "sigmoid", 8, 4, 2, True, 2.5)
    ids = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k), 7.0, device=DEV)
    st = _status()
    moe.moe_route(logits, bias, None, p, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    check_route(ids.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy(), k_max=k,
                score="sigmoid", bias=bias.cpu().numpy(), n_groups=8, topk_groups=4,
                group_topn=2, renormalize=True, route_scale=2.5)


def test_route_nan_and_bad_k():
    E, k = 16, 4
    logits = torch.randn((3, E), device=DEV)
    logits[1, 3] = float("nan")
    kpt = torch.tensor([2, 4, 9], dtype=torch.int32, device=DEV)  # 9 > k_max: clamped
    p = moe.RouteParams.make(E, k, "sigmoid", renormalize=False)
    ids = torch.empty((3, k), dtype=torch.int32, device=DEV)
    w = torch.empty((3, k), device=DEV)
    st = _status()
    moe.moe_route(logits, None, kpt, p, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() in (moe.MOE_ERR_NAN_LOGIT, moe.MOE_ERR_DEVICE_INDEX)
    assert 3 not in ids[1].tolist()  # NaN ranks below every number
    assert (ids[2] >= 0).all()       # clamped to k_max
    assert (ids[0, 2:] == -1).all() and (w[0, 2:] == 0).all()


def test_route_validation():
    logits = torch.zeros((2, 12), device=DEV)
    ids = torch.empty((2, 4), dtype=torch.int32, device=DEV)
    w = torch.empty((2, 4), device=DEV)
    for p in (moe.RouteParams.make(12, 4, "softmax", n_groups=5, topk_groups=1),  # E % G
              moe.RouteParams.make(12, 4, "softmax", n_groups=4, topk_groups=1),  # k > kept
              moe.RouteParams.make(12, 4, 9)):                                    # bad score
        with pytest.raises(moe.MoeError):
            moe.moe_route(logits, None, None, p, ids, w)
    moe.moe_route(torch.zeros((0, 12), device=DEV), None, None,
                  moe.RouteParams.make(12, 4, "softmax"), ids[:0], w[:0])
    with pytest.raises(moe.MoeError):  # logits not 16-byte aligned
        moe.moe_route(torch.zeros((2 * 12 + 1,), device=DEV)[1:].view(2, 12), None, None,
                      moe.RouteParams.make(12, 4, "softmax"), ids, w)


# ----------------------------------------------------------------- hash route
@pytest.mark.parametrize("score,with_logits,renorm", [("sqrt_softplus", True, True),
                                                      ("softmax", True, False),
                                                      ("softmax", True, True),
                                                      ("topk_softmax", True, True),
                                                      ("sigmoid", False, True)])
def test_hash_route_parity(score, with_logits, renorm):
    T, E, k, vocab = 777, 384, 6, 5000
    g = _gen(99)
    tok = torch.randint(0, vocab, (T,), generator=g, device=DEV, dtype=torch.int32)
    table = torch.randint(0, E, (vocab, k), generator=g, device=DEV, dtype=torch.int32)
    table[tok[0]] = torch.tensor([3, 3, 5, 3, 9, 1], dtype=torch.int32, device=DEV)
    logits = torch.randn((T, E), generator=g, device=DEV) if with_logits else None
    p = moe.RouteParams.make(E, k, score, renormalize=renorm, route_scale=1.25)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), device=DEV)
    st = _status()
    moe.moe_hash_route(tok, table, logits, p, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    o = oracle.hash_route(tok.cpu().numpy(), table.cpu().numpy(), num_experts=E,
                          logits=None if logits is None else logits.cpu().numpy(),
                          score=oracle_score(score), renormalize=renorm, route_scale=1.25)
    assert np.array_equal(ids.cpu().numpy(), o["ids"])
    wg = w.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(wg - o["w"]) <= 1e-5 * np.abs(o["w"]))


@pytest.mark.parametrize("T,k,score,renorm", [(1001, 1, "softmax", True),
                                               (1001, 4, "sigmoid", False),
                                               (1001, 5, "sqrt_softplus", True),
                                               (1001, 8, "topk_softmax", True),
                                               (1001, 9, "softmax", True),
                                               (1001, 16, "sigmoid", True),
                                               (1001, 17, "sqrt_softplus", False),
                                               (1001, 32, "softmax", True),
                                               (200003, 2, "sqrt_softplus", True)])
def test_hash_route_lanes_per_token(T, k, score, renorm):
    """Every lane width (4, 8, 16, 32 lanes a token), a ragged last warp and,
    at 200003 tokens, more rows than one pass of the grid."""
    E, vocab = 64, 3000
    g = _gen(100 + k)
    tok = torch.randint(0, vocab, (T,), generator=g, device=DEV, dtype=torch.int32)
    table = torch.randint(0, E, (vocab, k), generator=g, device=DEV, dtype=torch.int32)
    logits = torch.randn((T, E), generator=g, device=DEV)
    p = moe.RouteParams.make(E, k, score, renormalize=renorm, route_scale=0.75)
    ids = torch.full((T, k), -9, dtype=torch.int32, device=DEV)
    w = torch.full((T, k), -9.0, device=DEV)
    st = _status()
    moe.moe_hash_route(tok, table, logits, p, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    o = oracle.hash_route(tok.cpu().numpy(), table.cpu().numpy(), num_experts=E,
                          logits=logits.cpu().numpy(), score=oracle_score(score),
                          renormalize=renorm, route_scale=0.75)
    assert np.array_equal(ids.cpu().numpy(), o["ids"])
    wg = w.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(wg - o["w"]) <= 1e-5 * np.abs(o["w"]))


def oracle_score(name):
    return {"softmax": oracle.SOFTMAX, "sigmoid": oracle.SIGMOID,
            "sqrt_softplus": oracle.SQRT_SOFTPLUS, "topk_softmax": oracle.TOPK_SOFTMAX}[name]


def test_hash_route_bad_entries():
    E, k, vocab = 16, 3, 10
    tok = torch.tensor([1, 10, 2, -1], dtype=torch.int32, device=DEV)
    table = torch.randint(0, E, (vocab, k), device=DEV, dtype=torch.int32)
    table[2, 1] = E  # out of range slot
    p = moe.RouteParams.make(E, k, "softmax")
    ids = torch.empty((4, k), dtype=torch.int32, device=DEV)
    w = torch.empty((4, k), device=DEV)
    st = _status()
    moe.moe_hash_route(tok, table, None, p, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_DEVICE_INDEX
    o = oracle.hash_route(tok.cpu().numpy(), table.cpu().numpy(), num_experts=E)
    assert np.array_equal(ids.cpu().numpy(), o["ids"])
    assert np.allclose(w.cpu().numpy(), o["w"], rtol=1e-6, atol=0)


# ------------------------------------------------------------------- dispatch
def _dispatch(ids, E):
    T, k = ids.shape
    counts = torch.full((E,), -5, dtype=torch.int32, device=DEV)
    offsets = torch.full((E + 1,), -5, dtype=torch.int32, device=DEV)
    st_tok = torch.full((max(T * k, 1),), -5, dtype=torch.int32, device=DEV)
    dest = torch.full((T, k), -5, dtype=torch.int32, device=DEV)
    ws = torch.full((max(moe.moe_dispatch_workspace_size(T, k, E), 256),), 0xAB,
                    dtype=torch.uint8, device=DEV)  # garbage: no initialisation needed
    st = _status()
    moe.moe_dispatch(ids, E, counts, offsets, st_tok, dest, ws, st)
    torch.cuda.synchronize()
    return counts, offsets, st_tok, dest, st.item()


@pytest.mark.parametrize("T,k,E,empty_frac,hot", [
    (1, 1, 1, 0.0, False), (1000, 8, 256, 0.0, False), (3001, 4, 128, 0.0, True),
    (777, 16, 128, 0.4, False), (5000, 6, 384, 0.0, False), (20000, 32, 512, 0.1, True),
    (333, 3, 7, 0.2, False), (70000, 8, 256, 0.0, True),
    # 200 K slots: eight items a lane; E = 130: 33 quads of the segment-total rows
    (25000, 8, 128, 0.3, True), (4000, 5, 130, 0.1, False),
    # around the one-block launch (at most 1024 slots)
    (128, 8, 64, 0.1, True), (1024, 1, 64, 0.1, True), (1025, 1, 16, 0.0, True),
    (512, 8, 64, 0.1, True),
    # over 296 segments of 4096 slots: segments of 2 and 7 rounds, ragged last round
    (200003, 8, 256, 0.1, True), (40001, 32, 512, 0.05, False), (1048577, 8, 128, 0.0, True)])
def test_dispatch_parity(T, k, E, empty_frac, hot):
    g = _gen(T + k + E)
    ids = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
    if hot:  # skewed load: a third of the slots on two experts
        m = torch.rand((T, k), generator=g, device=DEV) < 0.33
        ids[m] = torch.randint(0, 2, (int(m.sum()),), generator=g, device=DEV,
                               dtype=torch.int32) * (E - 1)
    if empty_frac:
        ids[torch.rand((T, k), generator=g, device=DEV) < empty_frac] = -1
    counts, offsets, st_tok, dest, st = _dispatch(ids, E)
    assert st == 0
    check_dispatch(ids.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy(),
                   st_tok.cpu().numpy(), dest.cpu().numpy(), E)


def test_dispatch_edge_cases():
    for ids in (torch.full((5, 3), -1, dtype=torch.int32, device=DEV),  # all empty
                torch.zeros((6, 0), dtype=torch.int32, device=DEV),     # k_max = 0
                torch.zeros((0, 4), dtype=torch.int32, device=DEV)):    # T = 0
        counts, offsets, st_tok, dest, st = _dispatch(ids, 9)
        assert st == 0
        assert (counts == 0).all() and (offsets == 0).all()
        if ids.numel():
            assert (dest == -1).all()
    ids = torch.tensor([[0, 9], [3, -2], [1, 1]], dtype=torch.int32, device=DEV)
    counts, offsets, st_tok, dest, st = _dispatch(ids, 4)
    assert st == moe.MOE_ERR_DEVICE_INDEX
    o = oracle.dispatch(ids.cpu().numpy(), 4)
    assert np.array_equal(dest.cpu().numpy(), o["dest_pos"])
    assert np.array_equal(counts.cpu().numpy(), o["counts"])


# ---------------------------------------------------------- permute / combine
@pytest.mark.parametrize("T,k,E,cap,pad,hot", [
    (1, 1, 4, 0, 1, False), (3001, 1, 128, 0, 128, True), (70000, 1, 128, 547, 128, True),
    (5000, 8, 64, 400, 16, False), (777, 6, 384, 3, 1, True), (40000, 4, 128, 1, 7, True),
    (20000, 16, 512, 0, 64, False), (9000, 2, 8, 2250, 128, True),
    (200, 2, 8, 0, 4096, False), (3000, 32, 16, 5, 1, True),
    # segments of several rounds, with capacity and padding
    (200003, 8, 256, 5000, 128, True), (160001, 8, 64, 0, 1, False)])
def test_dispatch_limited_parity(T, k, E, cap, pad, hot):
    """Capacity cut and block padding, bit-exact against the oracle."""
    g = _gen(T * 7 + E + cap + pad)
    ids = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
    if hot:  # a few experts take most of the demand, so the cut bites
        sel = torch.rand((T, k), generator=g, device=DEV) < 0.5
        ids = torch.where(sel, ids % 4, ids)
    ids[torch.rand((T, k), generator=g, device=DEV) < 0.1] = -1
    rows = moe.moe_dispatch_limited_rows(T, k, E, cap, pad)
    counts = torch.full((E,), -7, dtype=torch.int32, device=DEV)
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=DEV)
    sorted_token = torch.full((max(rows, 1),), -7, dtype=torch.int32, device=DEV)
    dest = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    dropped = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    ws = torch.empty((max(moe.moe_dispatch_workspace_size(T, k, E), 256),), dtype=torch.uint8,
                     device=DEV)
    st = _status()
    moe.moe_dispatch_limited(ids, E, cap, pad, counts, offsets, sorted_token, dest, ws, dropped, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    o = oracle.dispatch_limited(ids.cpu().numpy(), E, capacity=cap, pad=pad)
    n = int(o["offsets"][-1])
    assert np.array_equal(counts.cpu().numpy(), o["counts"])
    assert np.array_equal(offsets.cpu().numpy(), o["offsets"])
    assert np.array_equal(sorted_token.cpu().numpy()[:n], o["sorted_token"])
    assert np.array_equal(dest.cpu().numpy(), o["dest_pos"])
    assert dropped.item() == o["dropped"]
    if cap == 0 and pad == 1:
        ref = _dispatch(ids, E)
        assert torch.equal(dest, ref[3])


def test_dispatch_limited_then_permute_combine():
    """Dropped slots are skipped by permute and combine; padding rows untouched."""
    T, k, E, d, cap, pad = 2000, 2, 16, 256, 200, 128
    g = _gen(99)
    ids = torch.randint(0, 4, (T, k), generator=g, device=DEV, dtype=torch.int32)
    rows = moe.moe_dispatch_limited_rows(T, k, E, cap, pad)
    counts = torch.empty((E,), dtype=torch.int32, device=DEV)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=DEV)
    sorted_token = torch.empty((rows,), dtype=torch.int32, device=DEV)
    dest = torch.empty((T, k), dtype=torch.int32, device=DEV)
    ws = torch.empty((max(moe.moe_dispatch_workspace_size(T, k, E), 256),), dtype=torch.uint8,
                     device=DEV)
    moe.moe_dispatch_limited(ids, E, cap, pad, counts, offsets, sorted_token, dest, ws)
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    xs = torch.full((rows, d), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_permute(x, dest, xs)
    w = torch.rand((T, k), generator=g, device=DEV)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(xs, w, dest, None, out)
    torch.cuda.synchronize()
    n = int(offsets[-1].item())
    st = sorted_token[:n].cpu().numpy()
    xs_c = xs[:n].cpu()
    x_c = x.cpu()
    kept = st >= 0
    assert torch.equal(xs_c[torch.from_numpy(kept)], x_c[torch.from_numpy(st[kept]).long()])
    assert torch.all(xs_c[torch.from_numpy(~kept)] == 3.0)
    dropped_rows = (dest.cpu().numpy() < 0).all(axis=1)
    assert dropped_rows.any() and np.all(out.float().cpu().numpy()[dropped_rows] == 0.0)
    check_combine(out, xs, w.cpu().numpy(), dest.cpu().numpy())


@pytest.mark.parametrize("T,k,d,E", [(1, 1, 8, 4), (999, 8, 2048, 64), (500, 6, 7168, 384),
                                     (1234, 4, 2880, 128), (100, 32, 136, 512),
                                     (257, 2, 128, 8),
                                     # several rows a warp through both row buffers
                                     (10007, 3, 2048, 64), (2000, 8, 7168, 256)])
def test_permute_combine_parity(T, k, d, E):
    g = _gen(T * 3 + d)
    ids = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
    ids[::9, k - 1] = -1  # some empty slots
    counts, offsets, st_tok, dest, st = _dispatch(ids, E)
    n = int(offsets[-1].item())
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    xs = torch.zeros((max(n, 1), d), dtype=torch.bfloat16, device=DEV)
    moe.moe_permute(x, dest, xs)
    torch.cuda.synchronize()
    check_permute(xs, x, dest.cpu().numpy())
    y = torch.randn((max(n, 1), d), generator=g, device=DEV).to(torch.bfloat16)
    w = torch.rand((T, k), generator=g, device=DEV) * (dest >= 0)
    for shared in (None, torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)):
        out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
        moe.moe_combine(y, w, dest, shared, out)
        torch.cuda.synchronize()
        check_combine(out, y, w.cpu().numpy(), dest.cpu().numpy(), shared)


def test_permute_combine_validation():
    x = torch.zeros((4, 17), dtype=torch.bfloat16, device=DEV)
    dest = torch.zeros((4, 2), dtype=torch.int32, device=DEV)
    xs = torch.zeros((8, 16), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moe.MoeError):  # x not 16-byte aligned (offset by one element)
        moe.moe_permute(x.view(-1)[1:65].view(4, 16), dest, xs)
    out = torch.zeros((4, 16), dtype=torch.bfloat16, device=DEV)
    sh = torch.ones((4, 16), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(xs, torch.zeros((4, 0), device=DEV),
                    torch.zeros((4, 0), dtype=torch.int32, device=DEV), sh, out)
    torch.cuda.synchronize()
    assert torch.equal(out, sh)  # k_max = 0: the shared expert alone


@pytest.mark.parametrize("k_max,score,has_bias", [(1, "sigmoid", False), (4, "topk_softmax", False),
                                                  (8, "softmax", True), (16, "softmax", False)])
def test_route_keys_equal_in_high_bits(k_max, score, has_bias):
    """Rows whose keys differ only in their lowest mantissa bits: any scheme
    that compares shortened keys must still reach the exact selection."""
    T, E = 515, 128
    g = _gen(777 + k_max)
    base = torch.randn((T, 1), generator=g, device=DEV) * 2
    steps = torch.randint(-40, 41, (T, E), generator=g, device=DEV).float()
    logits = (base * (1 + steps * 2.0 ** -21)).contiguous()  # neighbours a few ulps apart
    logits[::3, 5] = logits[::3, 9]                          # and some exact ties
    bias = (torch.rand((E,), generator=g, device=DEV) * 1e-6) if has_bias else None
    p = moe.RouteParams.make(E, k_max, score)
    ids = torch.empty((T, k_max), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k_max), device=DEV)
    moe.moe_route(logits, bias, None, p, ids, w)
    torch.cuda.synchronize()
    r = check_route(ids.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy(), k_max=k_max,
                    score=score, bias=None if bias is None else bias.cpu().numpy())
    print(r)


# ------------------------------------------------------- fused gate + route
FUSED_CASES = [
    # T, d, E, k_max, score, bias, G, TG, topn, renorm, scale, dyn, integer_inputs
    (515, 2048, 128, 16, "softmax", False, 1, 1, 1, True, 1.0, True, False),
    (300, 7168, 256, 8, "sigmoid", True, 8, 4, 2, True, 2.5, False, False),
    (260, 7168, 384, 6, "sqrt_softplus", False, 1, 1, 1, True, 1.0, False, False),
    (333, 512, 128, 4, "topk_softmax", False, 1, 1, 1, True, 1.0, False, False),
    (129, 256, 128, 1, "sigmoid", False, 1, 1, 1, False, 1.0, False, False),
    (200, 1024, 8, 2, "softmax", False, 1, 1, 1, True, 1.0, False, False),
    (140, 512, 30, 5, "softmax", True, 3, 2, 2, True, 1.0, True, False),
    (257, 256, 512, 16, "sigmoid", True, 32, 8, 2, True, 1.0, False, False),
    (300, 128, 128, 8, "softmax", False, 1, 1, 1, False, 1.0, False, True),   # many exact ties
    (300, 256, 256, 8, "sigmoid", True, 8, 4, 2, True, 2.5, True, True),      # ties + groups
    # k fixed per 128-token block (the kernel narrows its selection per tile)
    (900, 2048, 128, 16, "softmax", False, 1, 1, 1, True, 1.0, "seg", False),
    (900, 512, 64, 8, "sigmoid", True, 1, 1, 1, True, 1.0, "seg", False),
    (700, 1024, 256, 16, "sigmoid", True, 8, 4, 2, True, 2.5, "seg", True),
]

SEG_K = [4, 1, 16, 8, 3, 0, 2]


def _seg_k(T, k_max):
    return torch.tensor([min(SEG_K[(i // 128) % len(SEG_K)], k_max) for i in range(T)],
                        dtype=torch.int32, device=DEV)


@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: "-".join(map(str, c)))
def test_gate_route_fused(case):
    """moe_gate_route must pick exactly the ids moe_gate_gemm + moe_route pick,
    with weights equal to rounding, and both must match the oracle."""
    T, d, E, k_max, score, has_bias, G, TG, topn, renorm, scale, dyn, integer = case
    g = _gen(T + d + E + k_max)
    if integer:
        x = torch.randint(-2, 3, (T, d), generator=g, device=DEV).to(torch.bfloat16)
        w = torch.randint(-2, 3, (E, d), generator=g, device=DEV).to(torch.bfloat16)
    else:
        x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
        w = (torch.randn((E, d), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    bias = (torch.rand((E,), generator=g, device=DEV) * 0.2 - 0.1) if has_bias else None
    if dyn == "seg":
        kpt = _seg_k(T, k_max)
    else:
        kpt = torch.randint(0, k_max + 1, (T,), generator=g, device=DEV,
                            dtype=torch.int32) if dyn else None
    p = moe.RouteParams.make(E, k_max, score, G, TG, topn, renorm, scale)
    ids = torch.full((T, k_max), -7, dtype=torch.int32, device=DEV)
    wts = torch.full((T, k_max), 7.0, device=DEV)
    logits = torch.full((T, E), float("nan"), device=DEV)
    st = _status()
    moe.moe_gate_route(x, w, bias, kpt, p, ids, wts, logits, st)
    ref_logits = torch.empty((T, E), device=DEV)
    ref_ids = torch.empty_like(ids)
    ref_w = torch.empty_like(wts)
    moe.moe_gate_gemm(x, w, ref_logits)
    moe.moe_route(ref_logits, bias, kpt, p, ref_ids, ref_w)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(logits, ref_logits)
    assert torch.equal(ids, ref_ids)
    assert torch.allclose(wts, ref_w, rtol=2e-6, atol=0)
    check_route(ids.cpu().numpy(), wts.cpu().numpy(), logits.cpu().numpy(), k_max=k_max,
                score=score, bias=None if bias is None else bias.cpu().numpy(),
                kpt=None if kpt is None else kpt.cpu().numpy(), n_groups=G, topk_groups=TG,
                group_topn=topn, renormalize=renorm, route_scale=scale)


def test_gate_route_without_logits_and_nan():
    T, d, E, k = 150, 256, 64, 4
    g = _gen(4242)
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    x[7, 3] = float("inf")  # row 7's logits become +-inf ...
    w = (torch.randn((E, d), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w[5, 3] = 0.0           # ... and inf * 0 = NaN for expert 5
    p = moe.RouteParams.make(E, k, "sigmoid", renormalize=False)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    wts = torch.empty((T, k), device=DEV)
    st = _status()
    moe.moe_gate_route(x, w, None, None, p, ids, wts, None, st)  # logits not written
    logits = torch.empty((T, E), device=DEV)
    ref_ids = torch.empty_like(ids)
    ref_w = torch.empty_like(wts)
    moe.moe_gate_gemm(x, w, logits)
    moe.moe_route(logits, None, None, p, ref_ids, ref_w)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_NAN_LOGIT
    assert torch.equal(ids, ref_ids)
    ok = torch.isfinite(ref_w)
    assert torch.allclose(wts[ok], ref_w[ok], rtol=2e-6, atol=0)
    with pytest.raises(moe.MoeError):  # k_max above the fused limit
        moe.moe_gate_route(x, w, None, None, moe.RouteParams.make(E, 17, "softmax"),
                           torch.empty((T, 17), dtype=torch.int32, device=DEV),
                           torch.empty((T, 17), device=DEV))


GROUPED_CASES = [
    # T, E, G, k_per_group, k, score, renorm, scale, integer logits
    (1000, 128, 8, 2, 8, "softmax", True, 1.0, False),
    (777, 256, 8, 4, 8, "sigmoid", True, 2.5, False),
    (500, 384, 6, 2, 6, "sqrt_softplus", True, 1.0, False),
    (300, 64, 4, 3, 12, "topk_softmax", True, 1.0, True),   # every candidate kept
    (257, 512, 32, 1, 32, "sigmoid", False, 1.0, False),
    (100, 8, 1, 2, 2, "softmax", True, 1.0, False),         # one group: the flat rule
    (333, 96, 3, 32, 5, "softmax", True, 1.0, True),        # whole groups: the flat rule
    (200, 30, 3, 2, 4, "softmax", False, 1.0, True),        # E not a multiple of 32
    # quad path (whole 16-expert chunks and groups, k and k_per_group <= 8)
    (1003, 256, 16, 1, 8, "sigmoid", True, 2.5, False),     # groups of 16, one candidate each
    (515, 128, 1, 8, 8, "softmax", True, 1.0, False),       # one group: the flat rule
    (600, 512, 8, 3, 7, "sqrt_softplus", False, 1.0, False),
    (300, 128, 8, 2, 4, "topk_softmax", True, 1.0, True),   # integer logits: many ties
    (70001, 384, 6, 2, 6, "sqrt_softplus", True, 1.0, False),  # more rows than one grid pass
]


@pytest.mark.parametrize("case", GROUPED_CASES, ids=lambda c: "-".join(map(str, c)))
def test_route_grouped_parity(case):
    T, E, G, kpg, k, score, renorm, scale, integer = case
    g = _gen(T + E + kpg)
    if integer:
        logits = torch.randint(-3, 4, (T, E), generator=g, device=DEV).float()
    else:
        logits = torch.randn((T, E), generator=g, device=DEV)
    p = moe.RouteParams.make(E, k, score, G, 1, 1, renorm, scale)
    ids = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k), 7.0, device=DEV)
    st = _status()
    moe.moe_route_grouped(logits, p, kpg, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    sc = oracle_score(score)
    o = oracle.route_grouped(logits.cpu().numpy(), k_max=k, score=sc, n_groups=G, k_per_group=kpg,
                             renormalize=renorm, route_scale=scale, want_keys=True)
    gi, gw = ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)
    rows = np.nonzero(~np.all(gi == o["ids"], axis=1))[0]
    for t in rows:  # only a tie in the oracle's fp64 scores may order them otherwise
        kg = o["keys"][t][gi[t]]
        ko = o["keys"][t][o["ids"][t]]
        assert np.array_equal(np.sort(kg), np.sort(ko)) and np.all(np.isfinite(kg)), \
            f"row {t}: gpu {gi[t]} oracle {o['ids'][t]}"
    ow = o["w"].copy()
    if rows.size:
        ow[rows] = oracle.weights_for_ids(logits.cpu().numpy()[rows], gi[rows], score=sc,
                                          renormalize=renorm, route_scale=scale)
    assert np.all(np.abs(gw - ow) <= 1e-5 * np.abs(ow)), np.max(np.abs(gw - ow) / np.abs(ow))
    if G == 1 or kpg == E // G:  # the flat router gives the same ids
        fids = torch.empty_like(ids)
        fw = torch.empty_like(w)
        moe.moe_route(logits, None, None, moe.RouteParams.make(E, k, score, 1, 1, 1, renorm, scale),
                      fids, fw)
        torch.cuda.synchronize()
        assert torch.equal(fids, ids)


@pytest.mark.parametrize("E,G,kpg,k", [(128, 8, 2, 4),    # quad kernel
                                      (30, 3, 2, 4)])    # warp kernel
def test_route_grouped_nan_logits(E, G, kpg, k):
    """A NaN logit ranks below every number, as the header states (the
    ranking is of the logits, which every score orders alike), and the call
    reports MOE_ERR_NAN_LOGIT.  The ids of NaN rows are checked against that
    rule written out here; rows without NaN against the oracle."""
    T = 64
    g = _gen(E + G)
    logits = torch.randn((T, E), generator=g, device=DEV)
    nan_rows = [1, 7, 30]
    logits[1, 5] = float("nan")
    logits[7, :E // G] = float("nan")  # a whole group
    logits[30, ::3] = float("nan")
    p = moe.RouteParams.make(E, k, "softmax", G, 1, 1, True, 1.0)
    ids = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k), 7.0, device=DEV)
    st = _status()
    moe.moe_route_grouped(logits, p, kpg, ids, w, st)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_NAN_LOGIT
    lg, gi = logits.cpu().numpy(), ids.cpu().numpy()
    gsz = E // G
    order = lambda e, row: (0 if np.isnan(row[e]) else 1, -np.inf if np.isnan(row[e]) else row[e], -e)  # noqa: E731
    for t in nan_rows:
        row = lg[t]
        cand = []
        for q in range(G):
            grp = sorted(range(q * gsz, (q + 1) * gsz), key=lambda e: order(e, row), reverse=True)
            cand += grp[:kpg]
        want = sorted(cand, key=lambda e: order(e, row), reverse=True)[:k]
        assert gi[t].tolist() == want, (t, gi[t], want)
    ok = np.array([t not in nan_rows for t in range(T)])
    o = oracle.route_grouped(lg[ok], k_max=k, score=oracle.SOFTMAX, n_groups=G, k_per_group=kpg,
                             renormalize=True, route_scale=1.0, want_keys=True)
    assert np.array_equal(gi[ok], o["ids"])


def test_route_grouped_validation():
    logits = torch.zeros((4, 16), device=DEV)
    ids = torch.empty((4, 4), dtype=torch.int32, device=DEV)
    w = torch.empty((4, 4), device=DEV)
    for E_, G, kpg, k in ((16, 3, 1, 2), (16, 4, 0, 2), (16, 4, 5, 4), (16, 2, 1, 4)):
        p = moe.RouteParams.make(E_, k, "softmax", G, 1, 1, True, 1.0)
        with pytest.raises((moe.MoeError, ValueError)):
            moe.moe_route_grouped(logits, p, kpg, ids[:, :k].contiguous(), w[:, :k].contiguous())


def test_bounded_wait_times_out_and_context_survives():
    """The wait every kernel uses gives up on a barrier that nothing completes,
    records MOE_ERR_TIMEOUT and returns; the next calls run normally."""
    st = _status()
    outcome = torch.zeros((1,), dtype=torch.int32, device=DEV)
    moe.moe_wait_probe(20_000_000, st, outcome)  # 20 ms
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_TIMEOUT and outcome.item() == 2
    with pytest.raises(moe.MoeError):
        moe.moe_wait_probe(0, st)
    logits = torch.randn((64, 16), generator=_gen(5), device=DEV)
    p = moe.RouteParams.make(16, 2, "softmax")
    ids = torch.empty((64, 2), dtype=torch.int32, device=DEV)
    w = torch.empty((64, 2), device=DEV)
    st2 = _status()
    moe.moe_route(logits, None, None, p, ids, w, st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    assert torch.equal(ids[:, 0], logits.argmax(dim=1).to(torch.int32))
