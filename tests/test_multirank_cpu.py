"""Host-side multi-rank logic of bench.py on CPU ranks (gloo, world size 2):
the path shards by tokens with no exchange step, so the only cross-rank steps
are the barrier, the max over ranks of the step time and the job-wide
throughput built from it."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_env()
    assert (w, r) == (world, rank)
    bench.init_dist(w, "gloo")
    bench.barrier(w)
    ms = 2.0 + 3.0 * rank                      # rank 1 is the slow one
    ms_max = bench.reduce_max(ms, w, torch.device("cpu"))
    value = bench.job_throughput(16384, w, ms_max / 1e3)
    out[rank] = (ms_max, value, bench.rank_seed_offset(rank))
    dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of a threaded process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (m0, v0, s0), (m1, v1, s1) = out[0], out[1]
    assert m0 == m1 == 5.0                      # every rank sees the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 16384 / 5e-3)
    assert s0 != s1                             # each rank routes its own batch


def test_inputs_differ_per_rank_but_not_per_run():
    from token_dispatch_moe_b200.workloads import WORKLOADS, make_inputs
    wl = WORKLOADS["mixtral_tiny"]
    a = make_inputs(wl, "cpu", seed_offset=0)
    b = make_inputs(wl, "cpu", seed_offset=100000)
    c = make_inputs(wl, "cpu", seed_offset=0)
    assert not torch.equal(a["logits"], b["logits"])
    assert torch.equal(a["logits"], c["logits"]) and torch.equal(a["y"], c["y"])
