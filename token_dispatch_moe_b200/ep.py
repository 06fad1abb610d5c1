"""Expert-parallel exchange around the C-ABI calls: G ranks, expert e on rank
e // (E // G), rows moved over peer memory by moe_ep_permute / moe_ep_combine.

Only orchestration lives here: the count all-gather and the barriers are
torch.distributed collectives, the receive buffers come from torch's symmetric
memory (every rank maps every other rank's buffer), and every row movement is
a call into libmoe_dispatch.so.
"""
from __future__ import annotations

import torch

from . import moe_dispatch, moe_dispatch_workspace_size, moe_ep_combine, moe_ep_layout, \
    moe_ep_permute


def experts_per_rank(E: int, G: int) -> int:
    if E % G:
        raise ValueError(f"{E} experts do not split over {G} ranks")
    return E // G


def recv_rows(all_counts: torch.Tensor) -> list[int]:
    """Rows each rank receives: the demand of all ranks for its experts."""
    G, E = all_counts.shape
    el = experts_per_rank(E, G)
    demand = all_counts.sum(dim=0)
    return [int(demand[d * el:(d + 1) * el].sum().item()) for d in range(G)]


def exchange_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's per-expert counts: [G][E] on every rank."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    out = torch.empty((G, counts.numel()), dtype=counts.dtype, device=counts.device)
    if counts.device.type == "cuda":
        dist.all_gather_into_tensor(out, counts.contiguous(), group=group)
    else:  # gloo has no all_gather_into_tensor
        parts = list(out.unbind(0))
        dist.all_gather(parts, counts.contiguous(), group=group)
        out = torch.stack(parts)
    return out


def symmetric_buffer(rows: int, d: int, device, group=None):
    """A [rows, d] bf16 buffer every rank of the group can address, and the
    device table of the G addresses as this process maps them."""
    import torch.distributed as dist
    import torch.distributed._symmetric_memory as symm_mem
    buf = symm_mem.empty((rows, d), dtype=torch.bfloat16, device=device)
    hdl = symm_mem.rendezvous(buf, group if group is not None else dist.group.WORLD)
    table = torch.tensor(list(hdl.buffer_ptrs), dtype=torch.int64, device=device)
    return buf, table, hdl


class EpRank:
    """One rank's state: local dispatch outputs and its exchange layout."""

    def __init__(self, T: int, k_max: int, E: int, G: int, rank: int, device="cuda"):
        self.T, self.k_max, self.E, self.G, self.rank = T, k_max, E, G, rank
        self.el = experts_per_rank(E, G)
        i32 = dict(dtype=torch.int32, device=device)
        self.counts = torch.empty((E,), **i32)
        self.offsets = torch.empty((E + 1,), **i32)
        self.sorted_token = torch.empty((max(T * k_max, 1),), **i32)
        self.dest_pos = torch.empty((T, k_max), **i32)
        self.dest_rank = torch.empty((T, k_max), **i32)
        self.dest_row = torch.empty((T, k_max), **i32)
        self.recv_offsets = torch.empty((self.el + 1,), **i32)
        ws = moe_dispatch_workspace_size(T, k_max, E)
        self.workspace = torch.empty((max(ws, 256),), dtype=torch.uint8, device=device)
        self.status = torch.zeros((1,), **i32)

    def dispatch(self, topk_ids, stream=None):
        moe_dispatch(topk_ids, self.E, self.counts, self.offsets, self.sorted_token,
                     self.dest_pos, self.workspace, self.status, stream)

    def layout(self, all_counts, topk_ids, stream=None):
        moe_ep_layout(all_counts, topk_ids, self.dest_pos, self.offsets, self.rank,
                      self.dest_rank, self.dest_row, self.recv_offsets, self.status, stream)

    def permute(self, x, peers_recv, recv_capacity: int, stream=None):
        moe_ep_permute(x, self.dest_rank, self.dest_row, peers_recv, recv_capacity, self.status,
                       stream)

    def combine(self, peers_y, topk_w, shared, out, recv_capacity: int, stream=None):
        moe_ep_combine(peers_y, self.dest_rank, self.dest_row, topk_w, shared, out,
                       recv_capacity, self.status, stream)


def ep_step(rank_state: EpRank, x, topk_ids, topk_w, shared, out, recv_buf, recv_table,
            y_buf, y_table, experts, group=None, stream=None):
    """One exchange on G processes (one GPU each): local dispatch, count
    all-gather, layout, rows to the owners, barrier, experts(recv rows ->
    y rows, in place on this rank's buffers), barrier, combine from the owners.
    recv_buf / y_buf: this rank's symmetric buffers; *_table their peer tables."""
    import torch.distributed as dist
    rank_state.dispatch(topk_ids, stream)
    all_counts = exchange_counts(rank_state.counts, group)
    rank_state.layout(all_counts, topk_ids, stream)
    cap = recv_buf.shape[0]
    s = torch.cuda.current_stream() if stream is None else stream
    rank_state.permute(x, recv_table, cap, stream)
    s.synchronize()           # this rank's stores have landed ...
    dist.barrier(group=group)  # ... and so have everyone else's
    experts(recv_buf, y_buf, rank_state.recv_offsets)
    s.synchronize()
    dist.barrier(group=group)  # every owner's outputs are complete
    rank_state.combine(y_table, topk_w, shared, out, cap, stream)
    return all_counts
