"""Time one stage of the chain on its own (the driver of the per-kernel ncu
captures and of kernel A/B comparisons).

    python -m token_dispatch_moe_b200.stage_timer --workload llama4_top1 --stage route
        [--tokens T] [--iters N] [--warmup W] [--lib PATH]

Only the inputs the stage reads are made (its producers run once, untimed):
route reads the workload's logits (the gate GEMM's, for gate workloads),
dispatch the route's ids, permute x and the dispatch's dest_pos, combine the
synthetic expert outputs, weights and dest_pos.  Each timed launch is
bracketed by CUDA events on the launching stream, with L2 flushed (a 256 MiB
write) before it; the line printed gives the mean time per launch and the
stage's algorithmic bytes per launch (the bench's byte model) over that time.
--lib loads another build of libmoe_dispatch.so (same ABI) in place of the
package's own.  route_grouped runs moe_route_grouped on the route's logits,
with the workload's groups (8 where it has none) and --kpg candidates a group.
expert_gate_up and expert_down run the experts' FFN GEMMs (workloads with an
FFN shape; expert blocks padded to 128 rows, synthetic weights) on the
permuted rows, and print TFLOP/s beside the bytes.
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

STAGES = ("gate_gemm", "gate_route", "route", "route_grouped", "hash_route", "dispatch", "permute",
          "combine", "expert_gate_up", "expert_down")


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workload", required=True)
    ap.add_argument("--stage", required=True, choices=STAGES)
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--iters", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--lib", default=None)
    ap.add_argument("--kpg", type=int, default=2,
                    help="route_grouped: candidates a group (groups: the workload's, else 8)")
    args = ap.parse_args(argv)

    import token_dispatch_moe_b200 as moe
    from token_dispatch_moe_b200.path import RouterDispatch
    from token_dispatch_moe_b200.workloads import WORKLOADS, make_inputs, num_assignments

    if args.lib:
        moe._lib = moe.load_library(args.lib, strict=False)
    moe.load_library()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wl = WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.scaled(args.tokens)
    st = args.stage
    experts = None
    if st.startswith("expert_"):
        from token_dispatch_moe_b200.workloads import make_expert_weights
        wl = wl.with_ffn()
        experts = make_expert_weights(wl, device)
    need_x = wl.gate or st in ("permute", "expert_gate_up", "expert_down")
    inp = make_inputs(wl, device, with_y=(st == "combine"), with_x=need_x)
    fused = st == "gate_route"
    path = RouterDispatch(wl, device, fused=fused, keep_logits=not fused)
    n_assign = num_assignments(wl, inp["k_per_token"])

    logits = inp["logits"]
    if wl.gate and st not in ("gate_gemm", "gate_route"):
        logits = path.gate(inp["x"], inp["w"])
    if st in ("dispatch", "permute", "combine") or experts is not None:
        path.route(logits, inp["bias"], inp["k_per_token"])
        path.dispatch()
    if experts is not None:
        path.permute(inp["x"])
        path.expert_gate_up(experts)
    if st != "permute" and not wl.gate:
        inp["x"] = None
    torch.cuda.synchronize()

    steps = {
        "gate_gemm": lambda: path.gate(inp["x"], inp["w"]),
        "gate_route": lambda: path.gate_route(inp["x"], inp["w"], inp["bias"], inp["k_per_token"]),
        "route": lambda: path.route(logits, inp["bias"], inp["k_per_token"]),
        "hash_route": lambda: path.hash_route(inp["token_ids"], inp["tid2eid"], logits),
        "dispatch": lambda: path.dispatch(),
        "permute": lambda: path.permute(inp["x"]),
        "combine": lambda: path.combine(inp["y"], inp["shared"]),
        "expert_gate_up": lambda: path.expert_gate_up(experts),
        "expert_down": lambda: path.expert_down(experts),
    }
    if st == "route_grouped":
        G = wl.n_groups if wl.n_groups > 1 else 8
        gp = moe.RouteParams.make(wl.E, wl.k_max, wl.score, G, 1, 1, wl.renormalize,
                                  wl.route_scale)
        gids = torch.empty((wl.T, wl.k_max), dtype=torch.int32, device=device)
        gw = torch.empty((wl.T, wl.k_max), dtype=torch.float32, device=device)
        steps[st] = lambda: moe.moe_route_grouped(logits, gp, args.kpg, gids, gw, path.status)
    step = steps[st]
    stream = torch.cuda.current_stream(device)
    flush = torch.empty((256 << 20) // 4, dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if path.status.item() != 0:
        raise RuntimeError(f"device status {moe.moe_status_string(path.status.item())}")
    from bench import ClockSampler, hash_stage_bytes, stage_bytes, stage_flops  # the bench's models
    times = []
    with ClockSampler(device.index) as clk:
        for _ in range(args.iters):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3)
    model = hash_stage_bytes(wl) if st == "hash_route" else stage_bytes(wl, n_assign, fused)
    model["route_grouped"] = wl.T * (4 * wl.E + 8 * wl.k_max)  # logits in, ids and weights out
    us = statistics.fmean(times)
    nbytes = model.get(st)
    flops = stage_flops(wl, n_assign).get(st)
    print(json.dumps({
        "workload": wl.name, "tokens": wl.T, "stage": st, "lib": args.lib or "package",
        "us": round(us, 2), "us_min": round(min(times), 2), "iters": args.iters,
        "bytes": nbytes, "GB_s": round(nbytes / (us * 1e-6) / 1e9, 1) if nbytes else None,
        "TFLOP_s": round(flops / (us * 1e-6) / 1e12, 1) if flops else None,
        "clocks": clk.summary()}))


if __name__ == "__main__":
    main()
