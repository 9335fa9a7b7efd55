"""Builds the CPU oracle shared library (oracle/liboracle.so).

TEST INFRASTRUCTURE ONLY: the oracle is the independent CPU statement of the
AQLM layer that the tests, the smoke check and the benchmark's CPU-baseline leg
compare against.  The product path never loads it.

Flags: -O2 without -ffast-math and with -ffp-contract=off, so every float
operation in the oracle is one IEEE-754 operation (no fused multiply-add, no
reassociation).  OpenMP parallelises over output rows only, which changes no
arithmetic order.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "aqlm_oracle.cpp")
LIBRARY = os.path.join(HERE, "liboracle.so")

FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
         "-fPIC", "-shared", "-Wall", "-Wextra"]


def needs_build() -> bool:
    return (not os.path.exists(LIBRARY)
            or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE))


def build(force: bool = False) -> str:
    """Compile the oracle if it is missing or older than its source."""
    if force or needs_build():
        tmp = LIBRARY + f".tmp{os.getpid()}"
        cmd = ["g++", *FLAGS, SOURCE, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
