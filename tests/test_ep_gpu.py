"""Expert-parallel exchange kernels against the oracle, G ranks emulated on one
GPU: every rank's buffers live on this device, the peer tables hold their
addresses, and the ranks' calls run one after another (no kernel waits on
another).  The same kernels take real peer addresses on G GPUs."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_moe_b200 as moe
from gpu_check import bits, bits_to_f64
from token_dispatch_moe_b200.ep import EpRank, recv_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _ranks_inputs(G, T, k, E, d, seed, hot=False):
    g = _gen(seed)
    xs, ids, ws, sh = [], [], [], []
    for _ in range(G):
        i = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
        if hot:
            i[:, 0] = i[:, 0] % 2
        i[torch.rand((T, k), generator=g, device=DEV) < 0.1] = -1
        ids.append(i)
        xs.append(torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16))
        ws.append(torch.rand((T, k), generator=g, device=DEV))
        sh.append(torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16))
    return xs, ids, ws, sh


def _emulated_exchange(G, T, k, E, d, seed, hot=False, cap_extra=0):
    xs, ids, ws, sh = _ranks_inputs(G, T, k, E, d, seed, hot)
    ranks = [EpRank(T, k, E, G, r) for r in range(G)]
    for r in range(G):
        ranks[r].dispatch(ids[r])
    all_counts = torch.stack([rs.counts for rs in ranks])  # the all-gather
    rows = recv_rows(all_counts)
    cap = max(rows) + cap_extra
    recv = [torch.full((max(cap, 1), d), 7.0, dtype=torch.bfloat16, device=DEV) for _ in range(G)]
    table = moe.peer_table(recv)
    for r in range(G):
        ranks[r].layout(all_counts, ids[r])
        ranks[r].permute(xs[r], table, cap)
    torch.cuda.synchronize()
    return xs, ids, ws, sh, ranks, all_counts, rows, cap, recv


@pytest.mark.parametrize("G,T,k,E,d,hot", [(1, 300, 4, 8, 64, False), (2, 500, 2, 8, 128, False),
                                           (4, 1000, 8, 64, 256, True),
                                           (8, 777, 6, 256, 7168, False),
                                           (8, 64, 1, 8, 2048, True),
                                           (2, 300, 3, 16, 768, False)])  # two vectors a lane
def test_ep_exchange_parity(G, T, k, E, d, hot):
    xs, ids, ws, sh, ranks, all_counts, rows, cap, recv = _emulated_exchange(
        G, T, k, E, d, 77 + G * 13 + T, hot)
    for rs in ranks:
        assert rs.status.item() == 0
    ids_all = np.stack([i.cpu().numpy() for i in ids])
    lay = oracle.ep_layout(ids_all, E)
    assert list(lay["recv_rows"]) == rows
    for r in range(G):
        assert np.array_equal(ranks[r].dest_rank.cpu().numpy(), lay["dest_rank"][r])
        assert np.array_equal(ranks[r].dest_row.cpu().numpy(), lay["dest_row"][r])
        el = E // G
        want_off = np.concatenate([[0], np.cumsum(all_counts.cpu().numpy()[:, r * el:(r + 1) * el]
                                                  .sum(axis=0))])
        assert np.array_equal(ranks[r].recv_offsets.cpu().numpy(), want_off)
    x_all = np.stack([bits(x) for x in xs])
    want = oracle.ep_permute(x_all, lay["dest_rank"], lay["dest_row"], lay["recv_rows"])
    for dd in range(G):
        assert np.array_equal(bits(recv[dd][:rows[dd]]), want[dd]), f"receive buffer of rank {dd}"
    # Experts: synthetic outputs in each owner's receive layout; combine reads them back.
    g = _gen(5)
    y = [torch.randn((max(cap, 1), d), generator=g, device=DEV).to(torch.bfloat16)
         for _ in range(G)]
    ytab = moe.peer_table(y)
    outs = [torch.empty((T, d), dtype=torch.bfloat16, device=DEV) for _ in range(G)]
    for r in range(G):
        ranks[r].combine(ytab, ws[r], sh[r], outs[r], cap)
    torch.cuda.synchronize()
    o = oracle.ep_combine([bits(y[dd][:rows[dd]]) for dd in range(G)],
                          np.stack([w.cpu().numpy() for w in ws]), lay["dest_rank"],
                          lay["dest_row"], np.stack([bits(s) for s in sh]))
    for r in range(G):
        assert ranks[r].status.item() == 0
        ref, mag = o[r]
        got = bits_to_f64(bits(outs[r]))
        scale = np.maximum(np.abs(ref), mag)
        assert np.all(np.abs(got - ref) <= 1e-2 * np.where(scale > 0, scale, 1.0))


def test_ep_round_trip_identity_experts():
    """y = received x and weights 1/k per kept slot give x back (to bf16)."""
    G, T, k, E, d = 4, 400, 4, 32, 512
    xs, ids, ws, sh, ranks, all_counts, rows, cap, recv = _emulated_exchange(G, T, k, E, d, 9)
    table = moe.peer_table(recv)
    for r in range(G):
        kept = (ids[r] >= 0).float()
        w = kept / kept.sum(dim=1, keepdim=True).clamp(min=1)
        out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
        ranks[r].combine(table, w.contiguous(), None, out, cap)
        torch.cuda.synchronize()
        has = (ids[r] >= 0).any(dim=1)
        assert torch.allclose(out[has].float(), xs[r][has].float(), rtol=1e-2, atol=1e-2)
        assert torch.all(out[~has] == 0)


def test_ep_bounds_are_reported_not_written():
    """A receive capacity below the rows sent: the overflowing slots are
    skipped (nothing lands past the buffers' end) and the status says so."""
    G, T, k, E, d = 2, 256, 2, 8, 64
    xs, ids, ws, sh = _ranks_inputs(G, T, k, E, d, 31)
    ranks = [EpRank(T, k, E, G, r) for r in range(G)]
    for r in range(G):
        ranks[r].dispatch(ids[r])
    all_counts = torch.stack([rs.counts for rs in ranks])
    cap = min(recv_rows(all_counts)) // 2
    guard = 64
    bufs = [torch.full((cap + guard, d), 5.0, dtype=torch.bfloat16, device=DEV) for _ in range(G)]
    table = moe.peer_table(bufs)
    for r in range(G):
        ranks[r].layout(all_counts, ids[r])
        ranks[r].permute(xs[r], table, cap)
    torch.cuda.synchronize()
    assert all(rs.status.item() == moe.MOE_ERR_DEVICE_INDEX for rs in ranks)
    for b in bufs:
        assert torch.all(b[cap:] == 5.0)


def test_ep_validation():
    rs = EpRank(10, 2, 8, 2, 0)
    x = torch.zeros((10, 64), dtype=torch.bfloat16, device=DEV)
    tab = moe.peer_table([x, x])
    with pytest.raises(moe.MoeError):
        moe.moe_ep_permute(x, rs.dest_rank, rs.dest_row, tab, -1)   # negative capacity
    with pytest.raises(moe.MoeError):
        moe.moe_ep_layout(torch.zeros((3, 8), dtype=torch.int32, device=DEV),  # 8 % 3 != 0
                          torch.zeros((10, 2), dtype=torch.int32, device=DEV), rs.dest_pos,
                          rs.offsets, 0, rs.dest_rank, rs.dest_row,
                          torch.zeros((4,), dtype=torch.int32, device=DEV))


def test_ep_step_one_rank_over_nccl():
    """The whole exchange step of ep.py (count all-gather and barriers over
    NCCL, layout, peer stores, experts, peer loads) on a one-rank group, with
    plain device buffers standing in for the symmetric ones."""
    import socket

    import torch.distributed as dist

    from token_dispatch_moe_b200.ep import ep_step
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device(DEV, torch.cuda.current_device()))
    try:
        T, k, E, d = 500, 4, 16, 256
        xs, ids, ws, sh = _ranks_inputs(1, T, k, E, d, 123)
        rs = EpRank(T, k, E, 1, 0)
        cap = T * k
        recv = torch.zeros((cap, d), dtype=torch.bfloat16, device=DEV)
        y = torch.zeros((cap, d), dtype=torch.bfloat16, device=DEV)
        out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)

        def experts(recv_buf, y_buf, recv_offsets):
            y_buf.copy_(recv_buf)  # identity experts

        all_counts = ep_step(rs, xs[0], ids[0], ws[0], sh[0], out, recv, moe.peer_table([recv]), y,
                             moe.peer_table([y]), experts)
        torch.cuda.synchronize()
        assert rs.status.item() == 0
        flat = ids[0].reshape(-1)
        assert torch.equal(all_counts[0], torch.bincount(flat[flat >= 0].long(), minlength=E)
                           .to(torch.int32))
        lay = oracle.ep_layout(ids[0].cpu().numpy()[None], E)
        o = oracle.ep_combine([bits(recv[:int(lay["recv_rows"][0])])], ws[0].cpu().numpy()[None],
                              lay["dest_rank"], lay["dest_row"], bits(sh[0])[None])
        ref, mag = o[0]
        got = bits_to_f64(bits(out))
        assert np.all(np.abs(got - ref) <= 1e-2 * np.maximum(np.abs(ref), mag))
        # identity experts: the received rows are the tokens' own rows
        want = oracle.ep_permute(bits(xs[0])[None], lay["dest_rank"], lay["dest_row"],
                                 lay["recv_rows"])
        assert np.array_equal(bits(recv[:int(lay["recv_rows"][0])]), want[0])
    finally:
        dist.destroy_process_group()
