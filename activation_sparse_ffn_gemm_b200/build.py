"""In-tree build of libtwell.so (the sm_100a CUDA library behind include/twell.h)
and of its bounds-checked variant libtwell_bounds.so (the same sources compiled
with -DTWELL_BOUNDS: every index a kernel reads from a buffer is checked before
the access it steers, see TWELL_STATUS_BOUNDS in twell.h).

Usage: python -m activation_sparse_ffn_gemm_b200.build [--force] [--verbose]
nvcc cross-compiles for sm_100a without a GPU, so this runs on any host with
the CUDA 12.9 toolkit. The libraries land next to this file so that they travel
with the source tree.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtwell.so")
BOUNDS_LIB = os.path.join(PKG, "libtwell_bounds.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libtwell")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def _cmd(out: str, extra: list[str], verbose: bool) -> list[str]:
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--threads", "0", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-shared", "-I", INCLUDE, "-I", CSRC, *extra, *sources(), "-o", out]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds whichever of the two libraries is missing or older than its sources
    (both nvcc runs at once); returns the path of libtwell.so."""
    jobs = []
    for lib, extra in ((LIB, []), (BOUNDS_LIB, ["-DTWELL_BOUNDS"])):
        if force or _stale(lib):
            tmp = lib + f".tmp{os.getpid()}"
            jobs.append((lib, tmp, subprocess.Popen(_cmd(tmp, extra, verbose))))
    for lib, tmp, proc in jobs:
        if proc.wait() != 0:
            raise subprocess.CalledProcessError(proc.returncode, proc.args)
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
    print(BOUNDS_LIB)
