"""Benchmark of the B200 MoE router-and-dispatch path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path over one batch of synthetic tokens:
gate GEMM -> route -> dispatch -> permute -> combine (the chain the workload
defines), inputs resident in HBM.  L2 is flushed (a write larger than L2)
before every timed step, outside the step's events.  Timing: CUDA events on the
launching stream, barrier + synchronize around the K timed steps, max over
ranks.  value = routed tokens/s of the whole job (T tokens per rank per step).

Multi-GPU: the path shards by tokens with no exchange step, so each rank runs
its own T-token batch (weak scaling, different seeds per rank, no collective in
the data path; the only collectives are the barrier and the max-over-ranks of
the timings).

Extra keys: roofline (dominant kernel, algorithmic bytes / event time against
the measured HBM copy bandwidth), stages (every kernel), clocks (nvidia-smi
sampled during the timed steps), e2e (same metric through the C ABI with the
inputs copied from pinned host memory and the output copied back inside the
timed region), cpu_baseline (the fp64 CPU oracle on a bounded sample of the
same workload), gpu_launches.

--impl reference times the CPU oracle alone (the reference arm for this build:
there is no upstream implementation to run), rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
DEFAULT_WORKLOAD = "deepseek_v3"
METRIC = "routed tokens/s (gate->top-k->permute->combine); % of HBM/tensor roofline"


# ----------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime
    if world > 1 and not torch.distributed.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def barrier(world: int, device=None):
    if world > 1:
        if device is not None and torch.distributed.get_backend() == "nccl":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def reduce_max(value: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, seconds_per_step_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / seconds_per_step_max


def rank_seed_offset(rank: int) -> int:
    return 100000 * rank


# ------------------------------------------------------------------ byte model
def hash_stage_bytes(wl) -> dict:
    """The hash-routed layer's chain: gate GEMM (its logits give the weights),
    hash_route, dispatch, permute (every token takes k = k_max slots)."""
    T, d, E, k = wl.T, wl.d, wl.E, wl.k_max
    n = T * k
    return {"gate_gemm": T * d * 2 + E * d * 2 + T * E * 4,
            # token ids, the looked-up table rows, the logits of the k looked-up
            # experts, ids and weights out
            "hash_route": T * 4 + n * 4 + n * 4 + n * 8,
            "dispatch": n * 4 + n * 4 + n * 4 + 8 * E,
            "permute": T * d * 2 + n * d * 2 + n * 4}


def stage_bytes(wl, n_assign: int, fused: bool = False, limited=None) -> dict:
    """Algorithmic DRAM bytes per launch of each kernel (each read once, each
    write once) and the gate's FLOPs.  limited = (kept slots, tokens with a
    kept slot, padding rows) of a capacity-limited dispatch: only kept slots
    move rows, only tokens with one are read, padding rows cost a 4-byte -1."""
    T, d, E, k = wl.T, wl.d, wl.E, wl.k_max
    t_read, pad_rows = T, 0
    if limited is not None:
        n_assign, t_read, pad_rows = limited
    b = {}
    if wl.gate and fused:
        b["gate_route"] = (T * d * 2 + E * d * 2 + T * k * 8 + (T * 4 if wl.k_choices else 0)
                           + (E * 4 if wl.bias else 0))
    else:
        if wl.gate:
            b["gate_gemm"] = T * d * 2 + E * d * 2 + T * E * 4
        b["route"] = (T * E * 4 + T * k * 8 + (T * 4 if wl.k_choices else 0)
                      + (E * 4 if wl.bias else 0))
    b["dispatch"] = T * k * 4 + n_assign * 4 + T * k * 4 + 8 * E + pad_rows * 4
    b["permute"] = t_read * d * 2 + n_assign * d * 2 + T * k * 4
    if wl.ffn_dim and wl.pad % 128 == 0:  # the experts' FFN on the kept rows
        F = wl.ffn_dim
        bias = wl.ffn_act == "swiglu_oai"
        b["expert_gate_up"] = (n_assign * d * 2 + 2 * E * F * d * 2 + n_assign * F * 2
                               + (2 * E * F * 4 if bias else 0))
        b["expert_down"] = n_assign * F * 2 + E * d * F * 2 + n_assign * d * 2 + (E * d * 4 if bias else 0)
    if wl.combine:
        b["combine"] = n_assign * d * 2 + T * d * 2 + (T * d * 2 if wl.shared else 0) + 8 * T * k
    return b


def stage_flops(wl, n_assign: int) -> dict:
    """Algorithmic FLOPs of the tensor-core stages (padding rows excluded)."""
    f = {}
    if wl.gate:
        f["gate_route"] = f["gate_gemm"] = 2.0 * wl.T * wl.E * wl.d
    if wl.ffn_dim and wl.pad % 128 == 0:
        f["expert_gate_up"] = 2.0 * n_assign * 2 * wl.ffn_dim * wl.d
        f["expert_down"] = 2.0 * n_assign * wl.ffn_dim * wl.d
    return f


def host_env(device) -> dict:
    """What the numbers were taken on (reported, not used)."""
    cpu = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    cpu = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    driver = None
    try:
        driver = subprocess.run(["nvidia-smi", "--query-gpu=driver_version", "--format=csv,noheader",
                                 "-i", str(device.index or 0)], capture_output=True, text=True,
                                timeout=20).stdout.strip() or None
    except (OSError, subprocess.SubprocessError):
        pass
    return {"gpu": torch.cuda.get_device_name(device), "driver": driver,
            "torch": torch.__version__, "torch_cuda": torch.version.cuda, "host_cpu": cpu,
            "host_threads": os.cpu_count(), "seeds": "1000*workload + tensor (+100000*rank)"}


def launch_floor_us(device, stream, reps: int = 200) -> float:
    """Device time of a one-element kernel replayed from a CUDA graph on the
    bench's stream: the floor under any single stage's time."""
    t = torch.zeros((1,), device=device)
    cap = torch.cuda.Stream(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        t.add_(1.0)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    del g
    return round(us, 2)


def expert_load(counts) -> dict:
    """Per-expert load of the routed slots and its MaxVio = (max - mean) / mean,
    the balance measure of the aux-loss-free balancing the pages cite."""
    c = counts.detach().cpu().double()
    mean = float(c.mean())
    mx = float(c.max())
    return {"max_vio": round((mx - mean) / mean, 4) if mean > 0 else None,
            "max_count": int(mx), "mean_count": round(mean, 2)}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get(
            "bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "token_dispatch_moe_b200", "csrc")
    for name in files:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    kernel's current source files; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        entry = rec["workloads"][workload][kernel]
    except (OSError, ValueError, KeyError):
        return None
    if entry.get("sha") != kernel_source_hash(entry.get("files", [])):
        return None
    return entry.get("bytes")


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- oracle chain
def oracle_inputs(wl, inp: dict, n_tokens: int, experts=None) -> dict:
    """Host copies of the first n_tokens tokens of a workload's inputs, with
    expert outputs for the sample's own assignments (or, given the experts'
    weights, host copies of those)."""
    from token_dispatch_moe_b200.workloads import normal_bf16

    def bits(t):
        return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    h = {"T": n_tokens}
    h["x"] = bits(inp["x"][:n_tokens])
    h["w"] = bits(inp["w"]) if wl.gate else None
    h["logits"] = inp["logits"][:n_tokens].cpu().numpy() if not wl.gate else None
    h["bias"] = inp["bias"].cpu().numpy() if inp["bias"] is not None else None
    kpt = inp["k_per_token"]
    h["kpt"] = kpt[:n_tokens].cpu().numpy() if kpt is not None else None
    n = int(h["kpt"].sum()) if kpt is not None else n_tokens * wl.k_max
    n += wl.E * (wl.pad - 1)  # padded expert blocks
    h["y"] = bits(normal_bf16((max(n, 1), wl.d), 1.0, "cpu", 1000 * wl.index + 44))
    h["shared"] = bits(inp["shared"][:n_tokens]) if inp["shared"] is not None else None
    h["token_ids"] = (inp["token_ids"][:n_tokens].cpu().numpy()
                      if inp.get("token_ids") is not None else None)
    h["tid2eid"] = inp["tid2eid"].cpu().numpy() if inp.get("tid2eid") is not None else None
    h["experts"] = None
    if experts is not None:
        h["experts"] = {k: (None if v is None else
                            (bits(v) if v.dtype == torch.bfloat16 else v.cpu().numpy()))
                        for k, v in experts.items()}
    return h


def oracle_chain(wl, h: dict, hash_layer: bool = False, stage_s: dict | None = None) -> None:
    """The path computed by the fp64 CPU oracle (single thread): gate, route,
    dispatch, permute, [the experts' FFN when h holds their weights], combine,
    on the sample held in h; or the hash-routed layer's chain (gate, hash
    route, dispatch, permute).  stage_s, if given, receives each stage's wall
    seconds."""
    import oracle
    t_last = [time.perf_counter()]

    def lap(name):
        now = time.perf_counter()
        if stage_s is not None:
            stage_s[name] = stage_s.get(name, 0.0) + now - t_last[0]
        t_last[0] = now

    score = {"softmax": oracle.SOFTMAX, "sigmoid": oracle.SIGMOID,
             "sqrt_softplus": oracle.SQRT_SOFTPLUS, "topk_softmax": oracle.TOPK_SOFTMAX}[wl.score]
    logits = oracle.gate_rows(h["x"], h["w"]).astype(np.float32) if wl.gate else h["logits"]
    if wl.gate:
        lap("gate_gemm")
    if hash_layer:
        r = oracle.hash_route(h["token_ids"], h["tid2eid"], num_experts=wl.E, logits=logits,
                              score=score, renormalize=wl.renormalize,
                              route_scale=wl.route_scale)
        lap("hash_route")
        dsp = oracle.dispatch(r["ids"], wl.E)
        lap("dispatch")
        oracle.permute(h["x"], dsp["dest_pos"], int(dsp["offsets"][-1]))
        lap("permute")
        return
    r = oracle.route(logits, k_max=wl.k_max, score=score, bias=h["bias"], k_per_token=h["kpt"],
                     n_groups=wl.n_groups, topk_groups=wl.topk_groups, group_topn=wl.group_topn,
                     renormalize=wl.renormalize, route_scale=wl.route_scale)
    lap("route")
    if wl.limited:  # the same capacity rule, applied to the sample's own tokens
        dsp = oracle.dispatch_limited(r["ids"], wl.E, capacity=wl.scaled(h["T"]).capacity,
                                      pad=wl.pad)
    else:
        dsp = oracle.dispatch(r["ids"], wl.E)
    lap("dispatch")
    n = int(dsp["offsets"][-1])
    xs = oracle.permute(h["x"], dsp["dest_pos"], n)
    lap("permute")
    y = h["y"]
    if h.get("experts") is not None:
        ex = h["experts"]
        act = oracle.SWIGLU_OAI if wl.ffn_act == "swiglu_oai" else oracle.SWIGLU
        rows = np.nonzero(dsp["sorted_token"] >= 0)[0]
        hid = np.zeros((max(n, 1), wl.ffn_dim), np.uint16)
        hv = oracle.expert_gate_up(xs, dsp["offsets"], ex["w1"], ex["w3"], rows, act=act,
                                   b1=ex["b1"], b3=ex["b3"])
        hid[rows] = torch.from_numpy(hv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        lap("expert_gate_up")
        yv = oracle.expert_down(hid, dsp["offsets"], ex["w2"], rows, b2=ex["b2"])
        y = np.zeros((max(n, 1), wl.d), np.uint16)
        y[rows] = torch.from_numpy(yv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        lap("expert_down")
    if wl.combine:
        oracle.combine(y[:max(n, 1)], r["w"].astype(np.float32), dsp["dest_pos"],
                       h["shared"], want_mag=False)
        lap("combine")


def oracle_sample_size(wl, inp, budget_s: float, experts=None, hash_layer=False) -> int:
    """Tokens of CPU work that take about budget_s seconds (calibrated on a small run)."""
    n0 = min(64 if experts is None else 8, wl.T)
    h = oracle_inputs(wl, inp, n0, experts)
    t0 = time.perf_counter()
    oracle_chain(wl, h, hash_layer)
    per_token = (time.perf_counter() - t0) / n0
    return int(max(8, min(wl.T, budget_s / max(per_token, 1e-9))))


# ----------------------------------------------------------------- our arm
def dispatch_launches(n_slots: int) -> int:
    """Kernels one dispatch launches: one block for at most 1024 slots, else
    count + scatter."""
    return 1 if n_slots <= 1024 else 2


def chain_launches(wl, fused: bool) -> int:
    """Kernels of this library launched by one step of the chain."""
    gate_route = 1 if fused else (1 if wl.gate else 0) + 1
    return gate_route + dispatch_launches(wl.T * wl.k_max) + 1 + (1 if wl.combine else 0)


def run_ours(args):
    world, rank, local = dist_env()
    init_dist(world, "nccl")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import token_dispatch_moe_b200 as moe
    from token_dispatch_moe_b200.path import RouterDispatch
    from token_dispatch_moe_b200.workloads import WORKLOADS, make_inputs, num_assignments

    moe.load_library()  # no fallback: fails loudly if the library is missing
    wl = WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.scaled(args.tokens)
    experts = None
    if args.ffn:
        from token_dispatch_moe_b200.workloads import make_expert_weights
        if not wl.ffn_dim:
            raise SystemExit(f"--ffn: {wl.name} has no expert FFN shape; use --workload with one "
                             f"of {', '.join(n for n, w in WORKLOADS.items() if w.ffn_dim)}")
        wl = wl.with_ffn()
        experts = make_expert_weights(wl, device, seed_offset=rank_seed_offset(rank))
    inp = make_inputs(wl, device, with_y=experts is None, seed_offset=rank_seed_offset(rank))
    n_assign = num_assignments(wl, inp["k_per_token"])
    if args.hash_layer:
        if not wl.hash_vocab or experts is not None:
            raise SystemExit("--hash-layer needs a workload with a hash-routed layer, without --ffn")
        path = RouterDispatch(wl, device, fused=False, keep_logits=True)
    else:
        path = RouterDispatch(wl, device,
                              fused=False if args.separate else (True if args.fused else None))
    stream = torch.cuda.current_stream(device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)
    bytes_per = hash_stage_bytes(wl) if args.hash_layer else stage_bytes(wl, n_assign, path.fused)
    names = list(bytes_per)

    def run_step(mark):
        """One pass of the chain; mark(i) records the i-th stage boundary."""
        i = 0

        def boundary():
            nonlocal i
            if mark is not None:
                mark(i)
            i += 1

        boundary()
        if args.hash_layer:
            logits = path.gate(inp["x"], inp["w"])
            boundary()
            path.hash_route(inp["token_ids"], inp["tid2eid"], logits)
            boundary()
            path.dispatch(path.hash_ids)
            boundary()
            path.permute(inp["x"])
            boundary()
            return
        if path.fused:
            path.gate_route(inp["x"], inp["w"], inp["bias"], inp["k_per_token"])
            boundary()
        else:
            logits = inp["logits"]
            if wl.gate:
                logits = path.gate(inp["x"], inp["w"])
                boundary()
            path.route(logits, inp["bias"], inp["k_per_token"])
            boundary()
        path.dispatch()
        boundary()
        path.permute(inp["x"])
        boundary()
        y = inp["y"]
        if experts is not None:
            path.expert_gate_up(experts)
            boundary()
            path.expert_down(experts)
            boundary()
            y = path.y
        if wl.combine:
            path.combine(y, inp["shared"])
            boundary()

    for _ in range(args.warmup):
        flush.zero_()
        run_step(None)
    torch.cuda.synchronize()
    if path.status.item() != 0:
        raise RuntimeError(f"device status {moe.moe_status_string(path.status.item())}")
    limited = None
    if wl.limited:  # what the capacity kept decides the bytes moved
        kept = n_assign - path.dropped.item()
        t_read = int((path.dest_pos >= 0).any(dim=1).sum().item())
        limited = (kept, t_read, int(path.offsets[-1].item()) - kept)
        bytes_per = stage_bytes(wl, n_assign, path.fused, limited)

    K = args.steps
    nb = len(names) + 1
    if args.eager:
        # Stream launches, one set of events per step.
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nb)] for _ in range(K)]
        cur = {"s": 0}

        def mark(i):
            evs[cur["s"]][i].record(stream)

        def timed_step(s):
            cur["s"] = s
            run_step(mark)
    else:
        # The step captured as CUDA graphs (no host launch overhead); event-record
        # nodes inside them are read after each replay.
        gev = [torch.cuda.Event(enable_timing=True) for _ in range(nb)]
        for e in gev:
            e.record(stream)
        torch.cuda.synchronize()
        cudart = ctypes.CDLL("libcudart.so.12")
        cudart.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_uint]
        cap = torch.cuda.Stream(device)

        def mark(i):
            err = cudart.cudaEventRecordWithFlags(gev[i].cuda_event, cap.cuda_stream, 1)
            if err != 0:
                raise RuntimeError(f"cudaEventRecordWithFlags failed ({err})")

        def make_graph(every_stage):
            # An event node between two kernels replaces their programmatic
            # (PDL) edge by a full dependency, so the timed step carries events
            # at its two ends only; a second graph of the same step marks every
            # stage boundary for the per-stage breakdown.
            def m(i):
                if every_stage or i in (0, nb - 1):
                    mark(i)

            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
                run_step(m)
            g.replay()
            torch.cuda.synchronize()
            return g

        graph = make_graph(False)
        graph_stages = make_graph(True)
        step_times, times = [], []

        def timed_step(s):
            graph.replay()
            torch.cuda.synchronize()
            step_times.append(gev[0].elapsed_time(gev[nb - 1]))

        def stage_step(s):
            graph_stages.replay()
            torch.cuda.synchronize()
            times.append([gev[0].elapsed_time(gev[i]) for i in range(nb)])

    with ClockSampler(device.index) as clk:
        t_warm = time.perf_counter()
        while time.perf_counter() - t_warm < 0.3:  # let the sampler start under load (untimed)
            flush.zero_()
            run_step(None)
            torch.cuda.synchronize()
        barrier(world, device)
        torch.cuda.synchronize()
        for s in range(K):
            flush.zero_()  # L2 flush between timed steps, outside the step's events
            timed_step(s)
        torch.cuda.synchronize()
        barrier(world, device)
        if not args.eager:
            for s in range(K):  # the per-stage breakdown, after the timed region
                flush.zero_()
                stage_step(s)
            torch.cuda.synchronize()
    if args.eager:
        marks = [[evs[s][0].elapsed_time(evs[s][i]) for i in range(nb)] for s in range(K)]
        step_ms = [m[-1] for m in marks]
    else:
        marks = times
        step_ms = step_times
    stage_ms = {n: statistics.fmean(m[i + 1] - m[i] for m in marks) for i, n in enumerate(names)}
    ms = statistics.fmean(step_ms)
    srt = sorted(step_ms)
    ms_p50, ms_p90 = srt[len(srt) // 2], srt[min(len(srt) - 1, (9 * len(srt)) // 10)]
    ms_max = reduce_max(ms, world, device)
    value = job_throughput(wl.T, world, ms_max / 1e3)

    hbm, tf_burst, tf_sust, peak_kind = load_peaks()
    stages = {}
    for n in names:
        gbs = bytes_per[n] / (stage_ms[n] / 1e3) / 1e9
        stages[n] = {"us": round(stage_ms[n] * 1e3, 2), "bytes": bytes_per[n],
                     "GB_s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}
    kept = limited[0] if limited else n_assign
    flops = stage_flops(wl, kept)
    for n in names:
        if n in flops:
            stages[n]["TFLOP_s"] = round(flops[n] / (stage_ms[n] / 1e3) / 1e12, 1)
            stages[n]["frac_tensor"] = round(stages[n]["TFLOP_s"] / tf_sust, 4)
    dom = max(stage_ms, key=stage_ms.get)
    if dom.startswith("expert_"):  # a dense contraction: bound by the tensor pipe
        achieved = flops[dom] / (stage_ms[dom] / 1e3) / 1e12
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": tf_sust, "unit": "TFLOP/s", "frac": round(achieved / tf_sust, 4),
                    "traffic": recorded_traffic(wl.name + "+ffn", dom),
                    "algorithmic_flops": flops[dom], "peak_source": peak_kind + " (sustained)"}
    else:
        achieved = bytes_per[dom] / (stage_ms[dom] / 1e3) / 1e9
        roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                    "unit": "GB/s", "frac": round(achieved / hbm, 4),
                    "traffic": recorded_traffic(wl.name, dom),
                    "algorithmic_bytes": bytes_per[dom], "peak_source": peak_kind}

    e2e = None
    if not args.no_e2e:
        if args.hash_layer:
            def make_path():
                return RouterDispatch(wl, device, fused=False, keep_logits=True)
        else:
            def make_path():
                return RouterDispatch(wl, device, fused=path.fused)
        e2e = measure_e2e(wl, inp, path, device, stream, min(K, args.e2e_steps), world, experts,
                          args.hash_layer, make_path)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_max, 5),
        "ms_p50": round(ms_p50, 5), "ms_p90": round(ms_p90, 5),
        "launch_floor_us": launch_floor_us(device, stream),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
        "data": "synthetic",
        "config": {"workload": (wl.name + ("+ffn" if experts is not None else "")
                                + ("/hash-layer" if args.hash_layer else "")
                                + (f"@T={wl.T}" if args.tokens else "")),
                   "tokens_per_gpu": wl.T, "hidden": wl.d, "experts": wl.E,
                   "k": (f"{'/'.join(map(str, wl.k_choices))} per {wl.segment}-token request"
                         if wl.k_choices else wl.k_max),
                   "score": wl.score, "assignments_per_gpu": n_assign,
                   "inputs": "bf16 x / W / expert outputs, fp32 logits",
                   "l2": f"flushed before every timed step ({flush.numel() * 4 >> 20} MiB write)",
                   "parallelism": f"token-sharded replicas x{world}",
                   "launch": "stream (eager)" if args.eager else "CUDA graph of the step",
                   "gate_route": "fused (one kernel)" if path.fused else "separate kernels",
                   **({"capacity": path.capacity, "capacity_factor": wl.capacity_factor,
                       "pad_rows_to": wl.pad, "kept_slots": limited[0],
                       "dropped_slots": n_assign - limited[0]} if limited else {})},
        "roofline": roofline, "stages": stages,
        "stages_timed": ("events on the stream around each stage" if args.eager else
                         "a second graph of the step with an event node at every stage "
                         "boundary, replayed K times after the timed region"),
        "ms_per_step_stage_marked": round(statistics.fmean(m[-1] for m in marks), 5),
        "clocks": clk.summary(),
        "load": expert_load(path.counts), "env": host_env(device),
        "gpu_launches": (3 + dispatch_launches(wl.T * wl.k_max) if args.hash_layer else
                         chain_launches(wl, path.fused) + (2 if experts is not None else 0)) * K,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, inp, args.cpu_budget, experts, args.hash_layer)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def measure_e2e(wl, inp, path, device, stream, steps, world, experts=None, hash_layer=False,
                make_path=None):
    """Same metric through the C ABI with host buffers: each step copies its
    inputs from pinned host memory, runs the chain and copies the result back.
    Two step slots (device inputs and a RouterDispatch each) alternate, so one
    step's copies overlap its neighbours' work the way a serving loop would:
    host->device on a copy stream, the chain on the compute stream,
    device->host on a third stream (the two copy directions run at once)."""
    keys = ("x", "w", "token_ids") if hash_layer else \
        ("x", "w", "logits", "bias", "k_per_token", "y", "shared")
    names = [k for k in keys if inp[k] is not None]
    # pinned host copies, made without a pageable intermediate (deepseek_v3's
    # x, y and shared rows are 9.4 GB)
    host = {k: torch.empty(inp[k].shape, dtype=inp[k].dtype, pin_memory=True).copy_(inp[k])
            for k in names}
    paths = [path, make_path() if make_path is not None else path]
    devs = [{k: torch.empty_like(inp[k]) for k in names} for _ in range(2)]
    fulls = []
    for dv in devs:
        f = dict(inp)
        f.update(dv)
        fulls.append(f)
    results = [(p.out if (wl.combine and not hash_layer) else p.xs) for p in paths]
    outs_host = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in results]
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "comp", "d2h")}

    def one(step):
        i = step % 2 if make_path is not None else 0
        h2d_s.wait_event(ev["comp"][i])  # this slot's inputs are no longer read
        with torch.cuda.stream(h2d_s):
            for k in names:
                devs[i][k].copy_(host[k], non_blocking=True)
        ev["h2d"][i].record(h2d_s)
        stream.wait_event(ev["h2d"][i])
        stream.wait_event(ev["d2h"][i])  # this slot's result has been read back
        with torch.cuda.stream(stream):
            pth, full = paths[i], fulls[i]
            if hash_layer:
                pth.run_hash_layer(full, pth.gate(full["x"], full["w"]))
            else:
                pth.run(full, experts=experts)
        ev["comp"][i].record(stream)
        d2h_s.wait_event(ev["comp"][i])
        with torch.cuda.stream(d2h_s):
            outs_host[i].copy_(results[i], non_blocking=True)
        ev["d2h"][i].record(d2h_s)

    for e in ev.values():
        for x in e:
            x.record(stream)
    one(0)
    one(1)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(steps):
        one(s)
    for i in range(2):  # every copy of the last steps has landed
        stream.wait_event(ev["d2h"][i])
        stream.wait_event(ev["h2d"][i])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world, device)
    ms = reduce_max(e0.elapsed_time(e1) / steps, world, device)
    return {"value": round(job_throughput(wl.T, world, ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "steps": steps, "overlap": "two step slots; copies of both directions beside the chain"}


def cpu_baseline(wl, inp, budget_s: float, experts=None, hash_layer=False) -> dict:
    n = oracle_sample_size(wl, inp, budget_s, experts, hash_layer)
    h = oracle_inputs(wl, inp, n, experts)
    stage_s = {}
    t0 = time.perf_counter()
    oracle_chain(wl, h, hash_layer, stage_s)
    dt = time.perf_counter() - t0
    return {"value": round(n / dt, 2), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"first {n} of {wl.T} tokens of {wl.name}, full chain in fp64, "
                      f"{dt:.1f} s on one host core",
            "stage_s": {k: round(v, 3) for k, v in stage_s.items()}}


# ---------------------------------------------------------- reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return  # the CPU oracle runs once, on rank 0
    from token_dispatch_moe_b200.workloads import WORKLOADS, make_expert_weights, make_inputs
    wl = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    experts = None
    if args.ffn:
        wl = wl.with_ffn()
        experts = make_expert_weights(wl, dev)
    inp = make_inputs(wl, dev, with_y=experts is None)
    total_budget = args.cpu_budget
    hl = bool(args.hash_layer and wl.hash_vocab)
    per_step = oracle_sample_size(wl, inp, total_budget / max(1, args.steps + args.warmup),
                                  experts, hl)
    h = oracle_inputs(wl, inp, per_step, experts)
    for _ in range(args.warmup):
        oracle_chain(wl, h, hl)
    stage_s = {}
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_chain(wl, h, hl, stage_s)
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": (wl.name + ("+ffn" if experts is not None else "")
                                    + ("/hash-layer" if hl else "")),
                       "tokens_per_step": per_step,
                       "parallelism": "single host core"},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": 1,
                             "kind": "oracle",
                             "sample": f"first {per_step} of {wl.T} tokens per step",
                             "stage_ms_per_step": {k: round(v / args.steps * 1e3, 3)
                                                   for k, v in stage_s.items()}},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def ep_stage_bytes(T: int, d: int, k_max: int, n_assign: int, shared: bool) -> dict:
    """Algorithmic bytes of the expert-parallel exchange kernels over all ranks:
    layout reads ids and dest_pos and writes dest_rank and dest_row; permute
    reads every token row once and writes each of its N copies; combine reads
    the N expert rows (and the shared rows) and writes one row per token."""
    slots = T * k_max
    return {"ep_layout": 16 * slots,
            "ep_permute": T * d * 2 + n_assign * d * 2 + 8 * slots,
            "ep_combine": n_assign * d * 2 + T * d * 2 + (T * d * 2 if shared else 0) + 12 * slots}


def run_ep_emulated(args):
    """The expert-parallel exchange kernels with G ranks emulated on one GPU.

    The workload's tokens are routed once, then split over G ranks.  Every
    rank's buffers live on this device and the peer tables hold their
    addresses, so each rank's moe_ep_permute stores into all G receive
    buffers and its moe_ep_combine gathers from all G expert-output buffers,
    exactly as over NVLink, but the rows cross HBM instead.  The ranks'
    kernels run one after another on one stream (none waits on another)."""
    import token_dispatch_moe_b200 as moe
    from token_dispatch_moe_b200.ep import EpRank, recv_rows
    from token_dispatch_moe_b200.path import RouterDispatch
    from token_dispatch_moe_b200.workloads import WORKLOADS, make_inputs

    G = args.ep_emulate
    wl = WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.scaled(args.tokens)
    if G < 1 or wl.E % G or wl.T % G:
        raise SystemExit(f"{wl.name}: E = {wl.E} and T = {wl.T} must split over {G} ranks")
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    moe.load_library()
    inp = make_inputs(wl, device, with_y=False)
    path = RouterDispatch(wl, device, fused=False)
    logits = path.gate(inp["x"], inp["w"]) if wl.gate else inp["logits"]
    path.route(logits, inp["bias"], inp["k_per_token"])
    torch.cuda.synchronize()
    Tr, k, d = wl.T // G, wl.k_max, wl.d
    rows_of = lambda t, r: t[r * Tr:(r + 1) * Tr]  # noqa: E731
    xs = [rows_of(inp["x"], r) for r in range(G)]
    ids = [rows_of(path.topk_ids, r) for r in range(G)]
    wts = [rows_of(path.topk_w, r) for r in range(G)]
    sh = [rows_of(inp["shared"], r) if inp["shared"] is not None else None for r in range(G)]
    ranks = [EpRank(Tr, k, wl.E, G, r, device) for r in range(G)]
    for r in range(G):
        ranks[r].dispatch(ids[r])
    all_counts = torch.stack([rs.counts for rs in ranks])
    rows = recv_rows(all_counts)
    cap = max(max(rows), 1)
    g = torch.Generator(device=device)
    g.manual_seed(1000 * wl.index + 77)
    recv = [torch.empty((cap, d), dtype=torch.bfloat16, device=device) for _ in range(G)]
    ybuf = [torch.randn((cap, d), generator=g, device=device).to(torch.bfloat16) for _ in range(G)]
    outs = [torch.empty((Tr, d), dtype=torch.bfloat16, device=device) for _ in range(G)]
    recv_tab, y_tab = moe.peer_table(recv), moe.peer_table(ybuf)
    stream = torch.cuda.current_stream(device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)
    names = ["ep_layout", "ep_permute", "ep_combine"]

    def one(mark):
        mark(0)
        for r in range(G):
            ranks[r].layout(all_counts, ids[r])
        mark(1)
        for r in range(G):
            ranks[r].permute(xs[r], recv_tab, cap)
        mark(2)
        for r in range(G):
            ranks[r].combine(y_tab, wts[r], sh[r], outs[r], cap)
        mark(3)

    for _ in range(args.warmup):
        flush.zero_()
        one(lambda i: None)
    torch.cuda.synchronize()
    bad = [r for r in range(G) if ranks[r].status.item() != 0]
    if bad:
        raise RuntimeError(f"device status on ranks {bad}: "
                           f"{moe.moe_status_string(ranks[bad[0]].status.item())}")
    # The 3 x G launches captured as one CUDA graph, so that host launch time
    # does not open gaps between the short kernels; event-record nodes at the
    # stage boundaries are read after each replay.
    gev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in gev:
        e.record(stream)
    torch.cuda.synchronize()
    cudart = ctypes.CDLL("libcudart.so.12")
    cudart.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
    cap_stream = torch.cuda.Stream(device)

    def mark(i):
        if cudart.cudaEventRecordWithFlags(gev[i].cuda_event, cap_stream.cuda_stream, 1) != 0:
            raise RuntimeError("cudaEventRecordWithFlags failed")

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap_stream, capture_error_mode="relaxed"):
        one(mark)
    graph.replay()
    torch.cuda.synchronize()
    times = {n: [] for n in names}
    with ClockSampler(device.index) as clk:
        t_warm = time.perf_counter()
        while time.perf_counter() - t_warm < 0.3:  # let the sampler start under load (untimed)
            graph.replay()
            torch.cuda.synchronize()
        for _ in range(args.steps):
            flush.zero_()  # L2 flush before every timed pass, outside its events
            graph.replay()
            torch.cuda.synchronize()
            for i, n in enumerate(names):
                times[n].append(gev[i].elapsed_time(gev[i + 1]))
    n_assign = int(sum(rows))
    nbytes = ep_stage_bytes(wl.T, d, k, n_assign, inp["shared"] is not None)
    hbm, _, _, peak_kind = load_peaks()
    stages = {}
    for n in names:
        ms = statistics.fmean(times[n])
        gbs = nbytes[n] / (ms / 1e3) / 1e9
        stages[n] = {"us": round(ms * 1e3, 2), "bytes": nbytes[n], "GB_s": round(gbs, 1),
                     "frac_hbm": round(gbs / hbm, 4)}
    print(json.dumps({
        "metric": "expert-parallel exchange kernels, ranks emulated on one GPU",
        "unit": "GB/s per kernel", "ranks": G, "steps": args.steps, "warmup": args.warmup,
        "launch": "CUDA graph of the G ranks' launches, one stage after another",
        "config": {"workload": wl.name, "tokens_per_rank": Tr, "hidden": d, "experts": wl.E,
                   "experts_per_rank": wl.E // G, "rows_sent": n_assign,
                   "recv_rows_per_rank": rows,
                   "l2": f"flushed before every timed pass ({flush.numel() * 4 >> 20} MiB write)",
                   "links": "none: every buffer is on this GPU, so rows cross HBM, not NVLink"},
        "stages": stages, "peak": {"hbm_gbs": hbm, "source": peak_kind},
        "clocks": clk.summary()}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (profiling of smaller cases)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--separate", action="store_true",
                    help="run the gate GEMM and the route as two kernels instead of one")
    ap.add_argument("--fused", action="store_true",
                    help="route inside the gate GEMM even where two kernels are faster")
    ap.add_argument("--ffn", action="store_true",
                    help="run the experts' SwiGLU FFN (synthetic weights) on the permuted rows "
                         "instead of reading synthetic expert outputs")
    ap.add_argument("--hash-layer", action="store_true",
                    help="time the hash-routed layer's chain (gate, hash_route, dispatch, "
                         "permute) of a workload that has one")
    ap.add_argument("--eager", action="store_true",
                    help="launch from the host every step instead of replaying a CUDA graph")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of single-core oracle work for the CPU baseline")
    ap.add_argument("--ep-emulate", type=int, default=0, metavar="G",
                    help="time the expert-parallel exchange kernels with G ranks emulated on "
                         "this one GPU (a separate measurement, not the chain)")
    args = ap.parse_args(argv)
    if args.ep_emulate:
        run_ep_emulated(args)
        return
    world, _, _ = dist_env()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
