"""Build step for the CUDA library: compiles ``csrc/onebit_adam.cu`` for sm_100a into
``libonebit_adam.so`` next to this file (in-tree, so the built library travels with the repo).

Run ``python -m communication_compressed_optimizer_momentum_b200.build`` or call ``build()``.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC_DIR = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libonebit_adam.so")
SOURCES = [os.path.join(SRC_DIR, "onebit_adam.cu")]
DEPS = SOURCES + [os.path.join(SRC_DIR, "kernels.cuh"), os.path.join(SRC_DIR, "kernels_dp.cuh"),
                  os.path.join(SRC_DIR, "kernels_zero_one.cuh"),
                  os.path.join(INCLUDE, "onebit_adam.h")]

# --fmad=false: no contraction of the method's fp32 multiply-adds (every fp32 operation is one
# IEEE operation); fp64 fused multiply-adds are written out where wanted. No fast-math, so
# division and square root are the correctly rounded ones.
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17", "--fmad=false",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than its sources; return its path."""
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", SRC_DIR, "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
