"""Build libmoe_dispatch.so in-tree with nvcc for sm_100a.

    python -m token_dispatch_moe_b200.build [--force] [--verbose] [--checked]

Each .cu under csrc/ is compiled to an object under _build/ (in parallel) and
linked into token_dispatch_moe_b200/libmoe_dispatch.so.  The CUDA runtime is
linked statically, so the library needs only the NVIDIA driver at run time.

--checked builds the MOE_CHECKED variant (every index read bounds-checked,
including the plain permute / combine) as libmoe_dispatch_checked.so, with its
objects under _build_checked/; the default library is left as it is.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmoe_dispatch.so")
LIB_CHECKED = os.path.join(PKG, "libmoe_dispatch_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3",
                     "-I" + INCLUDE, "-I" + CSRC]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) +
            glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          checked: bool = False) -> str:
    """Compile (if stale or forced) and return the path of the shared library;
    checked=True builds the MOE_CHECKED variant beside the default one."""
    lib = LIB_CHECKED if checked else LIB
    bdir = BUILD + "_checked" if checked else BUILD
    if not force and not stale(lib):
        return lib
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    flags = NVCC_FLAGS + (["-DMOE_CHECKED"] if checked else []) + list(extra_flags or [])

    def compile_one(src: str) -> str:
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [nvcc] + flags + ["-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{res.stderr}")
        if verbose and res.stderr:
            print(res.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc] + ARCH + ["-shared", "-o", tmp] + objs
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem usage")
    ap.add_argument("--checked", action="store_true",
                    help="build the MOE_CHECKED variant (libmoe_dispatch_checked.so)")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, checked=args.checked))
