"""Build ``libfar.so`` (the C ABI of include/far.h) for sm_100a with nvcc.

The library is built in-tree, next to this file, so that it travels with the
source tree.  ``python -m reduce_residual_add_b200.build [--force] [--verbose]``
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SOURCES = [os.path.join(CSRC, f) for f in ("far_abi.cu", "far_kernels.cu")]
HEADERS = [os.path.join(CSRC, "far_internal.h"), os.path.join(INCLUDE, "far.h")]
LIB = os.path.join(PKG, "libfar.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I", INCLUDE, "-I", CSRC,
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False, out: str = LIB) -> str:
    """Compile the library unless it is up to date; return its path."""
    if not force and not stale(out):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, *SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
