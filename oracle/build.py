"""Compiles the CPU oracle into oracle/liboracle.so (test infrastructure).

-ffp-contract=off keeps every binary32 multiply and add separately rounded;
-fno-fast-math keeps IEEE semantics (signed zeros, subnormals, exact
division and square root).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sharq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=gnu11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fexcess-precision=standard", "-Wall", "-Wextra", "-Wno-unknown-pragmas"]


LIB_OMP = os.path.join(HERE, "liboracle_omp.so")


def build(force: bool = False, omp: bool = False) -> str:
    """omp=False: the plain single-threaded oracle (its OpenMP pragmas are
    ignored). omp=True: the same source with OpenMP, which splits independent
    rows and output elements across threads without changing any result
    (the benchmark's all-cores CPU baseline)."""
    lib = LIB_OMP if omp else LIB
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    cmd = ["gcc", *CFLAGS, *(["-fopenmp"] if omp else []), SRC, "-o", lib + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build(force="--force" in sys.argv, omp=True))
