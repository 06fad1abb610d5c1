"""Parity of the whole chain on every workload, through the same RouterDispatch
object the benchmark times.

* reduced: the workload's d, E, k and scoring with a ragged token count the
  oracle finishes in seconds; every output of every stage is checked.
* full: the workload at its full size; route and dispatch are checked on every
  row, the gate, permute and combine on sampled tokens (first, last, random).
Each stage's oracle is fed the GPU's previous-stage output.
"""
import numpy as np
import pytest
import torch

from gpu_check import (check_combine, check_dispatch, check_dispatch_limited, check_expert_h,
                       check_expert_y, check_gate, check_permute, check_route, np32)
from token_dispatch_moe_b200.path import RouterDispatch
from token_dispatch_moe_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

REDUCED_T = {"mixtral_tiny": 253, "qwen3_dynk": 1500, "deepseek_v3": 777,
             "deepseek_v4": 777, "llama4_top1": 3001, "gptoss_top4": 3001,
             "llama4_top1_capacity": 3001}


def _sample(T, n, seed):
    rng = np.random.default_rng(seed)
    pick = rng.choice(T, size=min(n, T), replace=False)
    return np.unique(np.concatenate([pick, [0, T - 1]]))


def _run_and_check(wl, sampled: bool, fused=None):
    inp = make_inputs(wl, "cuda")
    path = RouterDispatch(wl, fused=fused, keep_logits=True)
    path.run(inp)
    torch.cuda.synchronize()
    assert path.status.item() == 0, path.status.item()
    report = {}
    logits = path.logits if wl.gate else inp["logits"]
    if wl.gate:
        rows = _sample(wl.T, 192, 1) if sampled else None
        report["gate_worst"] = check_gate(logits, inp["x"], inp["w"], rows)
    ids, w = np32(path.topk_ids), np32(path.topk_w)
    report["route"] = check_route(ids, w, np32(logits), k_max=wl.k_max, score=wl.score,
                                  bias=np32(inp["bias"]), kpt=np32(inp["k_per_token"]),
                                  n_groups=wl.n_groups, topk_groups=wl.topk_groups,
                                  group_topn=wl.group_topn, renormalize=wl.renormalize,
                                  route_scale=wl.route_scale)
    dest = np32(path.dest_pos)
    if wl.limited:
        n = check_dispatch_limited(ids, np32(path.counts), np32(path.offsets),
                                   np32(path.sorted_token), dest, path.dropped.item(), wl.E,
                                   path.capacity, wl.pad)
        report["dropped"] = path.dropped.item()
    else:
        n = check_dispatch(ids, np32(path.counts), np32(path.offsets), np32(path.sorted_token),
                           dest, wl.E)
    tokens = _sample(wl.T, 1024, 2) if sampled else None
    check_permute(path.xs, inp["x"], dest, tokens)
    if wl.combine:
        assert inp["y"].shape[0] >= n
        tokens = _sample(wl.T, 512, 3) if sampled else None
        report["combine_worst"] = check_combine(path.out, inp["y"], w, dest, inp["shared"], tokens)
    if wl.hash_vocab:
        path.run_hash_layer(inp, logits)
        torch.cuda.synchronize()
        assert path.status.item() == 0
        import oracle
        o = oracle.hash_route(np32(inp["token_ids"]), np32(inp["tid2eid"]), num_experts=wl.E,
                              logits=np32(logits), score=oracle.SQRT_SOFTPLUS,
                              renormalize=wl.renormalize, route_scale=wl.route_scale)
        hid = np32(path.hash_ids)
        assert np.array_equal(hid, o["ids"])
        hw = np32(path.hash_w).astype(np.float64)
        assert np.all(np.abs(hw - o["w"]) <= 1e-5 * np.abs(o["w"]))
        hdest = np32(path.dest_pos)
        check_dispatch(hid, np32(path.counts), np32(path.offsets), np32(path.sorted_token),
                       hdest, wl.E)
        check_permute(path.xs, inp["x"], hdest, _sample(wl.T, 1024, 4) if sampled else None)
    print(wl.name, wl.T, report)
    return report


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "separate"])
@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_reduced(name, fused):
    if not fused and not WORKLOADS[name].gate:
        pytest.skip("no gate: the fused and separate paths are the same")
    _run_and_check(WORKLOADS[name].scaled(REDUCED_T[name]), sampled=False, fused=fused)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_full(name):
    _run_and_check(WORKLOADS[name], sampled=True)
    torch.cuda.empty_cache()


FFN_T = {"mixtral_tiny": 253, "qwen3_dynk": 1500, "gptoss_top4": 700}


@pytest.mark.parametrize("name", list(FFN_T))
def test_workload_with_expert_ffn(name):
    """The chain with the experts' FFN on the permuted rows (expert blocks
    padded to 128): dispatch bit-exact, h and y against the oracle on sampled
    token rows (fed the device's previous stage), combine against the oracle
    over every token."""
    from token_dispatch_moe_b200 import MOE_ACT_SWIGLU, MOE_ACT_SWIGLU_OAI
    from token_dispatch_moe_b200.workloads import make_expert_weights
    wl = WORKLOADS[name].scaled(FFN_T[name]).with_ffn()
    inp = make_inputs(wl, "cuda", with_y=False)
    ex = make_expert_weights(wl, "cuda")
    path = RouterDispatch(wl, keep_logits=True)
    path.run(inp, experts=ex)
    torch.cuda.synchronize()
    assert path.status.item() == 0
    ids = np32(path.topk_ids)
    n = check_dispatch_limited(ids, np32(path.counts), np32(path.offsets), np32(path.sorted_token),
                               np32(path.dest_pos), path.dropped.item(), wl.E, 0, 128)
    st = np32(path.sorted_token)[:n]
    real = np.nonzero(st >= 0)[0]
    rows = np.unique(np.concatenate([_sample(real.size, 96, 5), [0, real.size - 1]]))
    rows = real[rows]
    act = MOE_ACT_SWIGLU_OAI if wl.ffn_act == "swiglu_oai" else MOE_ACT_SWIGLU
    check_expert_h(path.h, path.xs, path.offsets, ex["w1"], ex["w3"], ex["b1"], ex["b3"], act, rows)
    check_expert_y(path.y, path.h, path.offsets, ex["w2"], ex["b2"], rows)
    check_combine(path.out, path.y, np32(path.topk_w), np32(path.dest_pos), inp["shared"])


@pytest.mark.parametrize("name", ["qwen3_dynk", "deepseek_v4", "mixtral_tiny"])
def test_graph_replay_matches_eager(name):
    """The chain captured as a CUDA graph (as bench.py times it) gives the same
    bits as the same chain launched from the host: the kernels' programmatic
    dependent launches keep every producer/consumer order inside the graph."""
    wl = WORKLOADS[name].scaled(REDUCED_T[name])
    inp = make_inputs(wl, "cuda")
    eager = RouterDispatch(wl)
    eager.run(inp)
    torch.cuda.synchronize()
    assert eager.status.item() == 0
    path = RouterDispatch(wl)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
        path.run(inp)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert path.status.item() == 0
    for attr in ("topk_ids", "topk_w", "counts", "offsets", "dest_pos"):
        assert torch.equal(getattr(path, attr), getattr(eager, attr)), attr
    n = int(eager.offsets[-1].item())
    assert torch.equal(path.sorted_token[:n], eager.sorted_token[:n])
    assert torch.equal(path.xs[:n], eager.xs[:n])
    if wl.combine:
        assert torch.equal(path.out, eager.out)
    del g
