"""Build libmoe_w4a8.so in-tree with nvcc for sm_100a.

    python -m bit_quantized_moe_token_b200.build [-v]

The library is one translation unit (csrc/moe_w4a8.cu includes the other sources).  No
fast-math: IEEE division and square root, no flush-to-zero, as the layer's rounding rules
need.
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
LIB = os.path.join(PKG, "libmoe_w4a8.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    p = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    if not os.path.exists(p):
        raise RuntimeError(f"nvcc not found at {p}")
    return p


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def command(extra=()):
    return [nvcc(), "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", *ARCH, "-lineinfo",
            "-I", INCLUDE, *extra, os.path.join(CSRC, "moe_w4a8.cu"), "-o", LIB]


def build(verbose: bool = False, force: bool = False) -> str:
    if force or stale():
        cmd = command()
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force="-f" in sys.argv)
