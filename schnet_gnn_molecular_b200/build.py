"""Build the sm_100a shared library ``libschnet_b200.so`` in-tree with nvcc.

Usage: ``python -m schnet_gnn_molecular_b200.build [--force] [--verbose]``.
The library exports the C ABI declared in ``include/schnet.h``.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libschnet_b200.so")
SOURCES = ["api.cu", "neighbors.cu", "cfconv.cu", "atomwise.cu", "integrate.cu", "taps.cu"]
HEADERS = ["common.cuh", "internal.h", os.path.join("..", "..", "include", "schnet.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-ftz=true",
         "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", "-Xcompiler", "-fvisibility=hidden"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(extra or []), "-I", os.path.join(ROOT, "include"),
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp, "-lcuda"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else None
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv or extra is not None, extra=extra))
