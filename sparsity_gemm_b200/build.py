"""Builds the SharQ CUDA library in-tree: sparsity_gemm_b200/libsharq.so.

sm_100a only (tcgen05 tensor cores, TMA). nvcc cross-compiles without a GPU.
The library links the CUDA runtime as a shared library, so inside a PyTorch
process it shares torch's runtime (same contexts, same streams).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsharq.so")
SOURCES = ["api.cu", "prep.cu", "wquant.cu", "gemm.cu", "group.cu"]
HEADERS = ["layout.h", "sharq_dev.cuh", "sq_internal.h", os.path.join("..", "..", "include", "sharq.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xcompiler", "-Werror=return-type", "--diag-error=940",  # a missing return is an error
    "-cudart", "shared",
    "-Xlinker", "-rpath=/usr/local/cuda/lib64",
]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [NVCC, *FLAGS, *[os.path.join(CSRC, s) for s in SOURCES], "-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
