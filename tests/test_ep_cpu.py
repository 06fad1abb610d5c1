"""Host side of the expert-parallel exchange on CPU ranks (gloo, world size 2):
the count all-gather every rank runs before moe_ep_layout, and the receive
sizes derived from it, checked against the oracle's layout of both ranks'
slots."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

T, K, E = 300, 4, 16


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ids(rank):
    g = torch.Generator().manual_seed(4000 + rank)
    ids = torch.randint(0, E, (T, K), generator=g, dtype=torch.int32)
    ids[torch.rand((T, K), generator=g) < 0.1] = -1
    if rank == 1:  # a skewed rank: half its slots on expert 3
        ids[::2, 0] = 3
    return ids


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from token_dispatch_moe_b200.ep import exchange_counts, recv_rows
    ids = _ids(rank)
    flat = ids.reshape(-1)
    counts = torch.bincount(flat[flat >= 0].long(), minlength=E).to(torch.int32)
    all_counts = exchange_counts(counts)
    out[rank] = (all_counts.numpy().copy(), recv_rows(all_counts))
    dist.destroy_process_group()


def test_count_exchange_and_receive_sizes():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of a threaded process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (c0, r0), (c1, r1) = out[0], out[1]
    assert np.array_equal(c0, c1) and r0 == r1  # every rank holds the same plan
    ids_all = np.stack([_ids(r).numpy() for r in range(world)])
    for r in range(world):
        f = ids_all[r].reshape(-1)
        assert np.array_equal(c0[r], np.bincount(f[f >= 0], minlength=E))
    lay = oracle.ep_layout(ids_all, E)
    assert list(lay["recv_rows"]) == r0
    assert r0[0] > r0[1]  # expert 3 (rank 0's) is the hot one


def test_recv_rows_split():
    from token_dispatch_moe_b200.ep import experts_per_rank, recv_rows
    c = torch.tensor([[1, 2, 3, 4], [10, 20, 30, 40]], dtype=torch.int32)
    assert recv_rows(c) == [33, 77]
    assert experts_per_rank(8, 4) == 2
    try:
        experts_per_rank(6, 4)
        raise AssertionError("6 experts cannot split over 4 ranks")
    except ValueError:
        pass
