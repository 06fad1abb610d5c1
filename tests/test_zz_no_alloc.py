"""moe_dispatch_static: dispatch for callers that cannot allocate device memory
(its scratch is a fixed array inside the library).  Checked through the C ABI
against moe_dispatch with a caller-allocated workspace, bit for bit, on two
calls in a row, up to the largest workspace any size needs (the size of the
fixed array); the sizes it refuses are refused on the host (test_abi).

This file is collected last on purpose: it must pass both alone in a fresh
process and after every other test."""
import os
import subprocess
import sys
import textwrap

import numpy as np
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


LIMIT = 296 * 512 * 4  # bytes of the library's fixed scratch: the largest workspace of any size


@pytest.mark.parametrize("T,k,E", [(37888, 32, 512),    # 296 segments: the whole array
                                   (262144, 32, 512)])  # 8.4 M slots: 7 rounds a segment
def test_static_scratch_at_its_limit(T, k, E):
    """The request that fills the scratch to its last byte, and one of the
    largest slot counts, match the workspace dispatch bit for bit."""
    assert moe.moe_dispatch_workspace_size(T, k, E) <= LIMIT
    if T == 37888:
        assert moe.moe_dispatch_workspace_size(T, k, E) == LIMIT  # the whole array is used
    g = torch.Generator(device=DEV)
    g.manual_seed(4242 + T)
    ids = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
    ids[:, -1] = E - 1  # the last expert's column of every segment is written
    ids[::7, 0] = -1
    got = _outputs(T, k, E)
    moe.moe_dispatch_static(ids, E, *got)
    want = _reference(ids, E)
    torch.cuda.synchronize()
    assert got[4].item() == 0 and want[4].item() == 0
    for a, b in zip(got[:4], want[:4]):
        assert torch.equal(a, b)


# Run in a child process with no torch: the library and the CUDA driver API
# only.  The first dispatch runs in the device's primary context, the second
# in a second context created on the same device with its own buffers; each
# context has its own copy of the scratch array, so the address the first
# call found must not be reused by the second.
_TWO_CONTEXTS = textwrap.dedent(r"""
    import ctypes, sys
    import numpy as np
    sys.path.insert(0, sys.argv[1])
    import token_dispatch_moe_b200 as moe
    lib = moe.load_library()
    cu = ctypes.CDLL("libcuda.so.1")
    def ck(r, what):
        if r != 0:
            raise SystemExit(f"{what} failed: CUresult {r}")
    P, u64 = ctypes.c_void_p, ctypes.c_uint64
    ck(cu.cuInit(0), "cuInit")
    dev = ctypes.c_int(0)
    ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
    T, k, E = 20000, 8, 256
    rng = np.random.default_rng(7)
    def run_in(ctx):
        ck(cu.cuCtxSetCurrent(ctx), "cuCtxSetCurrent")
        ids = rng.integers(-1, E, size=(T, k)).astype(np.int32)
        sizes = {"ids": T * k, "counts": E, "offsets": E + 1, "sorted": T * k, "dest": T * k,
                 "status": 1}
        buf = {}
        for n, c in sizes.items():
            p = u64(0)
            ck(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(4 * c)), "cuMemAlloc")
            buf[n] = p.value
        ck(cu.cuMemcpyHtoD_v2(u64(buf["ids"]), ids.ctypes.data, ctypes.c_size_t(ids.nbytes)),
           "cuMemcpyHtoD")
        ck(cu.cuMemsetD32_v2(u64(buf["status"]), 0, ctypes.c_size_t(1)), "cuMemsetD32")
        st = lib.moe_dispatch_static(buf["ids"], T, k, E, buf["counts"], buf["offsets"],
                                     buf["sorted"], buf["dest"], buf["status"], None)
        if st != 0:
            raise SystemExit(f"moe_dispatch_static: status {st}")
        ck(cu.cuCtxSynchronize(), "cuCtxSynchronize")
        out = {}
        for n in ("counts", "offsets", "sorted", "dest", "status"):
            a = np.empty(sizes[n], np.int32)
            ck(cu.cuMemcpyDtoH_v2(a.ctypes.data, u64(buf[n]), ctypes.c_size_t(a.nbytes)),
               "cuMemcpyDtoH")
            out[n] = a
        for p in buf.values():
            ck(cu.cuMemFree_v2(u64(p)), "cuMemFree")
        flat = ids.reshape(-1)
        counts = np.bincount(flat[flat >= 0], minlength=E)
        offsets = np.concatenate([[0], np.cumsum(counts)])
        order = np.argsort(np.where(flat >= 0, flat, E), kind="stable")[:offsets[-1]]
        dest = np.full(T * k, -1, np.int64)
        dest[order] = np.arange(offsets[-1])
        assert out["status"][0] == 0, out["status"]
        assert np.array_equal(out["counts"], counts)
        assert np.array_equal(out["offsets"], offsets)
        assert np.array_equal(out["sorted"][:offsets[-1]], order // k)
        assert np.array_equal(out["dest"], dest)
    primary = P()
    ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "cuDevicePrimaryCtxRetain")
    run_in(primary)
    second = P()
    ck(cu.cuCtxCreate_v2(ctypes.byref(second), 0, dev), "cuCtxCreate")
    run_in(second)
    run_in(primary)
    ck(cu.cuCtxSetCurrent(None), "cuCtxSetCurrent")
    ck(cu.cuCtxDestroy_v2(second), "cuCtxDestroy")
    ck(cu.cuDevicePrimaryCtxRelease_v2(dev), "cuDevicePrimaryCtxRelease")
    print("OK")
""")


def test_static_scratch_per_context():
    """The scratch address is looked up per CUDA context: a second context on
    the same device (with its own copy of the array) gets its own address, and
    the primary context's cached one still serves the primary context."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _TWO_CONTEXTS, root], capture_output=True,
                         text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip().endswith("OK"), res.stdout + res.stderr
