"""Build the CUDA library ``libmsa.so`` in-tree for sm_100a with nvcc.

    python block_sparse_long_03_b200/build.py [--force]

The library is the product: every kernel of the forward pass lives in
``csrc/*.cu`` and the C ABI is ``include/msa.h``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmsa.so")
# The checked build: device bounds checks on data-derived indices (see
# msa_bounds_failures in include/msa.h); relocatable device code so the one
# failure counter is shared by every translation unit.
LIB_CHECKED = os.path.join(HERE, "libmsa_checked.so")
CHECKED_FLAGS = ["-DMSA_CHECKED=1", "-rdc=true"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [
        os.path.join(ROOT, "include", "msa.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile every CUDA source into one shared library (skipped when fresh);
    checked=True builds the bounds-checked variant instead."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(CHECKED_FLAGS if checked else []), *sources(), "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv))
