"""Build libmoe.so (the CUDA library behind include/moe.h) in-tree for sm_100a.

    python -m sparse_mixture_experts_10_b200.build [--force] [--bounds-check]

One translation unit (csrc/moe_api.cu) compiled with nvcc for
``-gencode arch=compute_100a,code=sm_100a``; the CUDA runtime is linked
statically, the driver's tensor-map encoder is looked up at run time, so the
library needs no GPU to build and no libcuda at link time.

``--bounds-check`` builds libmoe_debug.so instead: the same source with
``-DMOE_DEBUG_BOUNDS``, whose kernels check the indices they take from other
kernels or from the caller (permuted rows inside their expert's segment, group
tables on 128-row blocks and non-decreasing, slots and z rows in range) and,
where one fails, set MOE_STATUS_BOUNDS and skip the access instead of
faulting.  The binding loads it when MOE_BOUNDS_CHECK=1 is set.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libmoe.so")
LIB_DEBUG = os.path.join(PKG, "libmoe_debug.so")
SOURCES = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")) + glob.glob(os.path.join(PKG, "csrc", "*.cuh"))
                 + [os.path.join(ROOT, "include", "moe.h")])

NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-shared", "-diag-suppress", "128"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in SOURCES)


def build(force: bool = False, verbose: bool = False, bounds_check: bool = False) -> str:
    lib = LIB_DEBUG if bounds_check else LIB
    if not force and not needs_build(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DMOE_DEBUG_BOUNDS"] if bounds_check else []), "-I",
           os.path.join(ROOT, "include"), "-o", tmp, os.path.join(PKG, "csrc", "moe_api.cu")]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, bounds_check="--bounds-check" in sys.argv))
