"""Build the CUDA library ``libfp4attn.so`` in-tree for sm_100a.

    python -m nvfp4_precision_b200.build [--force] [--verbose]

Plain nvcc, one shared library, static CUDA runtime; the C ABI is declared in
include/fp4attn.h at the repository root.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfp4attn.so")
# The same library with every kernel's global stores, atomics and tile
# coordinates checked against their buffers (-DFP4ATTN_BOUNDS_CHECK): a failed
# check records FP4ATTN_ERR_RANGE instead of touching memory.  A debugging
# build; the binding loads it when FP4ATTN_BOUNDS_CHECK=1.
LIB_CHECKED = os.path.join(PKG, "libfp4attn_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    out = LIB_CHECKED if checked else LIB
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    if not force and os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    if checked:
        cmd += ["-DFP4ATTN_BOUNDS_CHECK"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [*sources(), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
