"""Builds libaqlm.so in-tree with nvcc for sm_100a (B200), and libaqlm_cpu.so
(the host-CPU kernel, g++ with OpenMP).

    python -m weight_only_additive_b200.build [--force] [--verbose-ptxas]

nvcc cross-compiles without a GPU.  The GPU library links the CUDA runtime
statically so it has no dependency beyond the driver.  The CPU library is a
separate shared object: neither library calls the other.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libaqlm.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr",
              "-Xcompiler", "-fPIC,-O2,-Wall", "-shared", "-cudart", "static",
              "-Xptxas", "-warn-spills,-warn-lmem-usage"]


CPU_SRC = os.path.join(PKG, "cpu", "aqlm_cpu.cpp")
CPU_LIBRARY = os.path.join(PKG, "libaqlm_cpu.so")
# IEEE arithmetic (no -ffast-math); AVX2/FMA/F16C only inside functions that carry
# target attributes and run after a CPU feature check
CPU_FLAGS = ["-O3", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libaqlm.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def needs_build() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build_cpu(force: bool = False) -> str:
    """Compile libaqlm_cpu.so if it is missing or older than its sources."""
    inputs = [CPU_SRC, os.path.join(INCLUDE, "aqlm_cpu.h"), os.path.join(INCLUDE, "aqlm.h")]
    if not force and os.path.exists(CPU_LIBRARY) and \
            all(os.path.getmtime(f) <= os.path.getmtime(CPU_LIBRARY) for f in inputs):
        return CPU_LIBRARY
    tmp = CPU_LIBRARY + f".tmp{os.getpid()}"
    subprocess.run(["g++", *CPU_FLAGS, "-I", INCLUDE, CPU_SRC, "-o", tmp], check=True)
    os.replace(tmp, CPU_LIBRARY)
    return CPU_LIBRARY


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    build_cpu(force)
    if not (force or needs_build()):
        return LIBRARY
    tmp = LIBRARY + f".tmp{os.getpid()}"
    flags = list(NVCC_FLAGS)
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    cmd = [nvcc(), *ARCH_FLAGS, *flags, "-I", INCLUDE, "-I", CSRC, *sources(), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
