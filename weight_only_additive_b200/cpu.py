"""ctypes binding of libaqlm_cpu.so: the AQLM linear layer on the host CPU
(include/aqlm_cpu.h).  Argument marshalling only; the arithmetic is in
weight_only_additive_b200/cpu/aqlm_cpu.cpp.  This library is separate from the
GPU library: nothing here is a fallback for a GPU call."""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

from .native import Status


class AqlmCpuError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = Status(status) if status in Status._value2member_map_ else status
        name = self.status.name if isinstance(self.status, Status) else f"status {status}"
        super().__init__(f"{what}: AQLM_ERR_{name}" if what else f"AQLM_ERR_{name}")

PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(PKG, "libaqlm_cpu.so")

EXPORTS = ("aqlm_cpu_matmul", "aqlm_cpu_simd_level", "aqlm_cpu_set_max_simd_level", "aqlm_cpu_abi_version")
ABI_VERSION = 3

_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Loads libaqlm_cpu.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIBRARY):
                    raise ImportError(f"{LIBRARY} is missing: build it with python -m weight_only_additive_b200.build")
                L = ctypes.CDLL(LIBRARY)
                _vp, _i = ctypes.c_void_p, ctypes.c_int
                L.aqlm_cpu_matmul.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i]
                L.aqlm_cpu_matmul.restype = _i
                L.aqlm_cpu_simd_level.restype = _i
                L.aqlm_cpu_set_max_simd_level.argtypes = [_i]
                L.aqlm_cpu_set_max_simd_level.restype = _i
                L.aqlm_cpu_abi_version.restype = _i
                if L.aqlm_cpu_abi_version() != ABI_VERSION:
                    raise ImportError(f"libaqlm_cpu.so ABI {L.aqlm_cpu_abi_version()} != binding ABI {ABI_VERSION}")
                _lib = L
    return _lib


def simd_level() -> int:
    """0 = scalar, 1 = AVX2 + FMA + F16C, 2 = AVX-512 (F, BW, VL) as well."""
    return lib().aqlm_cpu_simd_level()


def set_max_simd_level(level: int) -> int:
    """Caps the SIMD level for the whole process (tests, comparisons); returns the
    previous cap."""
    return lib().aqlm_cpu_set_max_simd_level(int(level))


SIMD_NAMES = {0: "scalar", 1: "avx2+fma+f16c", 2: "avx512f+bw+vl"}


def _arr(a, dtype):
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype).name}, got {a.dtype}")
    if not a.flags.c_contiguous:
        raise ValueError("arrays must be C-contiguous")
    return a


def matmul(x, codes, codebooks, scales, bias, M: int, B: int, g: int, nthreads: int = 0,
           out=None) -> np.ndarray:
    """y [batch, N] fp16 = x . W^T . diag(s) + bias on the host CPU."""
    x = _arr(x, np.float16)
    codes = _arr(codes, np.uint8 if B <= 8 else np.uint16)
    cb = _arr(codebooks, np.float16)
    sc = _arr(scales, np.float16)
    bi = _arr(bias, np.float16) if bias is not None else None
    if x.ndim != 2 or codes.ndim != 3:
        raise ValueError("expected x [batch, K] and codes [N, K/g, M]")
    batch, K = x.shape
    N = codes.shape[0]
    if codes.shape != (N, K // g, M) or cb.shape != (M, 1 << B, g) or sc.shape != (N,):
        raise ValueError("expected codes [N, K/g, M], codebooks [M, 2^B, g], scales [N]")
    if bi is not None and bi.shape != (N,):
        raise ValueError(f"expected bias [N] = [{N}], got {bi.shape}")
    y = np.empty((batch, N), np.float16) if out is None else _arr(out, np.float16)
    if y.shape != (batch, N):  # the kernel writes batch x N values
        raise ValueError(f"expected out [batch, N] = [{batch}, {N}], got {y.shape}")
    st = lib().aqlm_cpu_matmul(x.ctypes.data, codes.ctypes.data, cb.ctypes.data, sc.ctypes.data,
                               bi.ctypes.data if bi is not None else None, y.ctypes.data,
                               M, B, g, K, N, batch, nthreads)
    if st != 0:
        raise AqlmCpuError(st, "aqlm_cpu_matmul")
    return y
