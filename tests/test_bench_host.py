"""bench.py's host-side pieces without a GPU: the byte model each roofline
fraction divides by, and the oracle chain its CPU baseline and reference arm
time (run here on small CPU-generated samples of every workload)."""
import importlib.util
import os

import numpy as np
import pytest

from token_dispatch_moe_b200.workloads import WORKLOADS, expert_rows, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_stage_bytes_qwen3(bench):
    wl = WORKLOADS["qwen3_dynk"]
    T, d, E, k = 16384, 2048, 128, 16
    n = 150000
    b = bench.stage_bytes(wl, n, fused=False)
    assert b["gate_gemm"] == T * d * 2 + E * d * 2 + T * E * 4
    assert b["route"] == T * E * 4 + T * k * 8 + T * 4
    assert b["permute"] == T * d * 2 + n * d * 2 + T * k * 4
    assert b["combine"] == n * d * 2 + T * d * 2 + 8 * T * k
    f = bench.stage_bytes(wl, n, fused=True)
    assert "gate_gemm" not in f and "route" not in f
    assert f["gate_route"] == T * d * 2 + E * d * 2 + T * k * 8 + T * 4


def test_ep_stage_bytes_match_the_local_kernels(bench):
    """The exchange moves the same rows as permute and combine; its only extra
    bytes are the second routing table (dest_rank beside dest_row)."""
    wl = WORKLOADS["qwen3_dynk"]
    T, d, k = wl.T, wl.d, wl.k_max
    n = 150000
    local = bench.stage_bytes(wl, n, fused=False)
    ep = bench.ep_stage_bytes(T, d, k, n, shared=False)
    assert ep["ep_permute"] - local["permute"] == 4 * T * k
    assert ep["ep_combine"] - local["combine"] == 4 * T * k
    assert ep["ep_layout"] == 16 * T * k
    v3 = WORKLOADS["deepseek_v3"]
    with_shared = bench.ep_stage_bytes(v3.T, v3.d, v3.k_max, n, shared=True)
    without = bench.ep_stage_bytes(v3.T, v3.d, v3.k_max, n, shared=False)
    assert with_shared["ep_combine"] - without["ep_combine"] == v3.T * v3.d * 2


def test_ep_emulate_refuses_uneven_splits(bench):
    """Checked before any device work: mixtral_tiny's 8 experts do not split
    over 3 ranks, and 16384 tokens do not split over 3 either."""
    for argv in (["--ep-emulate", "3", "--workload", "mixtral_tiny"],
                 ["--ep-emulate", "3"]):
        with pytest.raises(SystemExit) as err:
            bench.main(argv)
        assert "must split over 3 ranks" in str(err.value)


def test_stage_bytes_capacity(bench):
    wl = WORKLOADS["llama4_top1_capacity"]
    T, d, E = wl.T, wl.d, wl.E
    kept, t_read, pad_rows = 250000, 250000, 5000
    b = bench.stage_bytes(wl, T, limited=(kept, t_read, pad_rows))
    assert b["permute"] == t_read * d * 2 + kept * d * 2 + T * 4
    assert b["combine"] == kept * d * 2 + T * d * 2 + T * d * 2 + 8 * T
    assert b["dispatch"] == T * 4 + kept * 4 + T * 4 + 8 * E + pad_rows * 4
    assert wl.capacity == T // E  # factor 1.0: the fair share


def test_expert_rows_bound():
    wl = WORKLOADS["llama4_top1_capacity"].scaled(1000)
    assert wl.capacity == 8  # ceil(1000 / 128)
    assert expert_rows(wl, None) == min(1000, 128 * 8) + 128 * 127
    assert expert_rows(WORKLOADS["gptoss_top4"].scaled(10), None) == 40


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_oracle_chain_runs_on_cpu_inputs(bench, name):
    wl = WORKLOADS[name].scaled(300)
    inp = make_inputs(wl, "cpu")
    h = bench.oracle_inputs(wl, inp, 40)
    assert h["T"] == 40 and h["x"].shape == (40, wl.d)
    n = int(h["kpt"].sum()) if wl.k_choices else 40 * wl.k_max
    assert h["y"].shape[0] >= n
    stage_s = {}
    bench.oracle_chain(wl, h, stage_s=stage_s)
    # the oracle's per-stage wall times carry the GPU stages' names
    assert set(stage_s) == set(bench.stage_bytes(wl, n))
    assert all(v >= 0.0 for v in stage_s.values())
    assert bench.oracle_sample_size(wl, inp, 0.05) >= 8
    if wl.k_choices:
        assert set(np.unique(h["kpt"])) <= set(wl.k_choices)


def test_oracle_chain_with_experts_on_cpu(bench):
    from token_dispatch_moe_b200.workloads import make_expert_weights
    for name in ("mixtral_tiny", "gptoss_top4"):
        wl = WORKLOADS[name].scaled(200).with_ffn()
        if name == "gptoss_top4":  # keep the fp64 FFN small on CPU
            import dataclasses
            wl = dataclasses.replace(wl, d=64, ffn_dim=32)
        inp = make_inputs(wl, "cpu", with_y=False)
        ex = make_expert_weights(wl, "cpu")
        assert (ex["b1"] is not None) == (wl.ffn_act == "swiglu_oai")
        h = bench.oracle_inputs(wl, inp, 12, ex)
        bench.oracle_chain(wl, h)
        b = bench.stage_bytes(wl, 24, limited=(24, 12, 100))
        f = bench.stage_flops(wl, 24)
        assert f["expert_gate_up"] == 2.0 * 24 * 2 * wl.ffn_dim * wl.d
        assert b["expert_down"] >= wl.E * wl.d * wl.ffn_dim * 2


def test_hash_layer_chain_on_cpu(bench):
    wl = WORKLOADS["deepseek_v4"].scaled(64)
    import dataclasses
    wl = dataclasses.replace(wl, d=256)  # small enough for the fp64 gate on CPU
    inp = make_inputs(wl, "cpu", with_y=False)
    h = bench.oracle_inputs(wl, inp, 16)
    assert h["token_ids"].shape == (16,) and h["tid2eid"].shape == (wl.hash_vocab, wl.k_max)
    bench.oracle_chain(wl, h, hash_layer=True)
    b = bench.hash_stage_bytes(wl)
    assert list(b) == ["gate_gemm", "hash_route", "dispatch", "permute"]
    assert b["permute"] == wl.T * wl.d * 2 + wl.T * wl.k_max * wl.d * 2 + wl.T * wl.k_max * 4


def test_expert_load_max_vio(bench):
    import torch
    r = bench.expert_load(torch.tensor([1, 1, 1, 5], dtype=torch.int32))
    assert r == {"max_vio": 1.5, "max_count": 5, "mean_count": 2.0}
    assert bench.expert_load(torch.tensor([3, 3, 3], dtype=torch.int32))["max_vio"] == 0.0
