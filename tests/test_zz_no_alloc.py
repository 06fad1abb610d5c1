"""moe_dispatch_static: dispatch for callers that cannot allocate device memory
(its scratch is a fixed array inside the library).  Checked through the C ABI
against moe_dispatch with a caller-allocated workspace, bit for bit, on two
calls in a row; oversize requests must be refused without a launch.

This file is collected last on purpose: it must pass both alone in a fresh
process and after every other test."""
import pytest
import torch

import token_dispatch_moe_b200 as moe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(T, k, E):
    i32 = dict(dtype=torch.int32, device=DEV)
    return (torch.full((E,), -3, **i32), torch.full((E + 1,), -3, **i32),
            torch.full((max(T * k, 1),), -3, **i32), torch.full((T, k), -3, **i32),
            torch.zeros((1,), **i32))


def _reference(ids, E):
    T, k = ids.shape
    counts, offsets, st_tok, dest, status = _outputs(T, k, E)
    ws = torch.empty((max(moe.moe_dispatch_workspace_size(T, k, E), 256),), dtype=torch.uint8,
                     device=DEV)
    moe.moe_dispatch(ids, E, counts, offsets, st_tok, dest, ws, status)
    return counts, offsets, st_tok, dest, status


@pytest.mark.parametrize("T,k,E", [(16384, 16, 128), (3001, 6, 384), (65536, 8, 256)])
def test_static_scratch_matches_workspace_dispatch(T, k, E):
    g = torch.Generator(device=DEV)
    for call in range(2):  # two calls in a row: the scratch keeps the first call's contents
        g.manual_seed(1000 * call + T + k + E)
        ids = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
        ids[torch.rand((T, k), generator=g, device=DEV) < 0.1] = -1
        got = _outputs(T, k, E)
        moe.moe_dispatch_static(ids, E, *got)
        want = _reference(ids, E)
        torch.cuda.synchronize()
        n = int(want[1][-1].item())
        assert got[4].item() == 0 and want[4].item() == 0
        assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])
        assert torch.equal(got[2][:n], want[2][:n]) and torch.equal(got[3], want[3])


def test_static_scratch_refuses_oversize():
    T, k, E = 524288, 32, 512  # needs more than the fixed 4 MiB
    assert moe.moe_dispatch_workspace_size(T, k, E) > 4 << 20
    ids = torch.zeros((T, k), dtype=torch.int32, device=DEV)
    out = _outputs(T, k, E)
    with pytest.raises(moe.MoeError) as err:
        moe.moe_dispatch_static(ids, E, *out)
    assert err.value.status == moe.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (out[0] == -3).all()  # nothing was launched
