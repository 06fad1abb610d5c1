"""Bounds-checked row movers.

moe_permute_bounded / moe_combine_bounded (in every build) check each dest_pos
against the rows the caller's buffer holds, skip a slot outside [-1, rows) and
report MOE_ERR_DEVICE_INDEX; the plain moe_permute / moe_combine of the
MOE_CHECKED build (libmoe_dispatch_checked.so) check against T * k_max rows.

Every out-of-range dest_pos planted here points at a slack row the buffer
really has, past the bound the call is given, so even an unchecked access
would stay inside allocated memory.  The tests check that the slack rows are
left alone, that the skipped slots are the only difference from the oracle,
and that valid input gives the default build's results bit for bit."""
import numpy as np
import pytest
import torch

import token_dispatch_moe_b200 as moe
from gpu_check import bits, check_combine
from token_dispatch_moe_b200 import build as build_mod

pytestmark = pytest.mark.gpu
DEV = "cuda"
SLACK = 8
SENTINEL = 0x7E57  # a bf16 bit pattern no input row holds


def _case(T, k, d, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    n = T * k
    dest = torch.randperm(n, generator=g, device=DEV).to(torch.int32).view(T, k).contiguous()
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    y = torch.randn((n + SLACK, d), generator=g, device=DEV).to(torch.bfloat16)
    y[n:] = 1000.0  # a slack row read by mistake would dominate its token's output
    w = torch.rand((T, k), generator=g, device=DEV)
    sh = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    return dest, x, y, w, sh


def _plant(dest, bound):
    """Two bad slots: one at the bound itself (a slack row), one below -1."""
    bad = dest.clone()
    lost = [int(bad[3, 1].item()), int(bad[5, 0].item())]  # rows these slots would have filled
    bad[3, 1] = bound
    bad[5, 0] = -9
    skipped = dest.clone()
    skipped[3, 1] = -1
    skipped[5, 0] = -1
    return bad, skipped, lost


def _xs_buffer(n, d):
    xs = torch.empty((n + SLACK, d), dtype=torch.bfloat16, device=DEV)
    xs.view(torch.int16).fill_(SENTINEL)
    return xs


def _check_permute_skipped(xs, x, skipped, lost, n):
    dp = skipped.cpu().numpy()
    got = bits(xs)
    xb = bits(x)
    for t in range(dp.shape[0]):
        for j in range(dp.shape[1]):
            if dp[t, j] >= 0:
                assert np.array_equal(got[dp[t, j]], xb[t]), (t, j)
    for r in lost + list(range(n, n + SLACK)):
        assert np.all(got[r] == SENTINEL), f"row {r} was written"


@pytest.mark.parametrize("d", [64, 1024, 4096])
def test_bounded_calls_skip_and_report(d):
    T, k = 64, 2
    n = T * k
    dest, x, y, w, sh = _case(T, k, d, 11 + d)
    bad, skipped, lost = _plant(dest, n)
    xs = _xs_buffer(n, d)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_permute_bounded(x, bad, xs[:n], st)  # the call sees n rows; the slack is beyond
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_DEVICE_INDEX
    _check_permute_skipped(xs, x, skipped, lost, n)

    out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    st.zero_()
    moe.moe_combine_bounded(y[:n], w, bad, sh, out, st)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_DEVICE_INDEX
    check_combine(out, y, w.cpu().numpy(), skipped.cpu().numpy(), sh)

    # valid input: nothing reported, the plain calls' results bit for bit
    xs2, xs3 = _xs_buffer(n, d), _xs_buffer(n, d)
    out2 = torch.empty_like(out)
    st.zero_()
    moe.moe_permute_bounded(x, dest, xs2[:n], st)
    moe.moe_permute(x, dest, xs3)
    moe.moe_combine_bounded(y[:n], w, dest, sh, out2, st)
    moe.moe_combine(y, w, dest, sh, out)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(xs2.view(torch.int16), xs3.view(torch.int16))
    assert torch.equal(out2.view(torch.int16), out.view(torch.int16))


@pytest.fixture(scope="module")
def checked_lib():
    return moe.load_library(build_mod.build(checked=True))


@pytest.mark.parametrize("d", [64, 4096])
def test_checked_build_plain_calls(checked_lib, d):
    """The MOE_CHECKED library's plain moe_permute / moe_combine skip a
    dest_pos at T * k_max (and below -1); on valid input they match the
    default library bit for bit."""
    T, k = 64, 2
    n = T * k
    dest, x, y, w, sh = _case(T, k, d, 23 + d)
    bad, skipped, lost = _plant(dest, n)
    stream = torch.cuda.current_stream().cuda_stream
    xs = _xs_buffer(n, d)
    assert checked_lib.moe_permute(x.data_ptr(), bad.data_ptr(), T, k, d, xs.data_ptr(),
                                   stream) == moe.MOE_OK
    out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    assert checked_lib.moe_combine(y.data_ptr(), w.data_ptr(), bad.data_ptr(), sh.data_ptr(), T, k,
                                   d, out.data_ptr(), stream) == moe.MOE_OK
    torch.cuda.synchronize()
    _check_permute_skipped(xs, x, skipped, lost, n)
    check_combine(out, y, w.cpu().numpy(), skipped.cpu().numpy(), sh)

    xs_c, xs_d = _xs_buffer(n, d), _xs_buffer(n, d)
    out_c, out_d = torch.empty_like(out), torch.empty_like(out)
    assert checked_lib.moe_permute(x.data_ptr(), dest.data_ptr(), T, k, d, xs_c.data_ptr(),
                                   stream) == moe.MOE_OK
    assert checked_lib.moe_combine(y.data_ptr(), w.data_ptr(), dest.data_ptr(), sh.data_ptr(), T,
                                   k, d, out_c.data_ptr(), stream) == moe.MOE_OK
    moe.moe_permute(x, dest, xs_d)
    moe.moe_combine(y, w, dest, sh, out_d)
    torch.cuda.synchronize()
    assert torch.equal(xs_c.view(torch.int16), xs_d.view(torch.int16))
    assert torch.equal(out_c.view(torch.int16), out_d.view(torch.int16))
