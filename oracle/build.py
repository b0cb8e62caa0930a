"""Build the CPU oracle's shared library (test infrastructure only).

``python oracle/build.py`` compiles ``bitlinear_oracle.c`` with gcc into
``liboracle.so`` beside it, and the same source with -fopenmp into
``liboracle_omp.so`` (used only for the benchmark's all-core CPU baseline).
No CUDA is involved.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitlinear_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra", "-Wno-unknown-pragmas"]


LIB_OMP = os.path.join(HERE, "liboracle_omp.so")


def _build(lib: str, extra: list, force: bool) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    cmd = ["gcc", *CFLAGS, *extra, SRC, "-o", lib + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False) -> str:
    return _build(LIB, [], force)


def build_omp(force: bool = False) -> str:
    """The same source compiled with -fopenmp: the integer contraction's
    (m, n) pairs are shared among threads; every result is the same."""
    return _build(LIB_OMP, ["-fopenmp"], force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build_omp(force="--force" in sys.argv))
