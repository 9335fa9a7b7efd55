"""CPU oracle for the AQLM weight-only linear layer (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and the library never imports it.

Every function follows the definition stated at the top of
``oracle/aqlm_oracle.cpp``:

* ``dequantize``    -- W16[n, j*g+t] = f16_rne(fp32(sum_m C_m[code][t]) * s_n),
                       codebooks summed in ascending m starting from C_0;
* ``linear``        -- y = x . W16^T + bias in fp64 (exact products, k ascending);
* ``linear_exact``  -- y = s . (x . (sum of codewords)^T) + bias in fp64, no fp16 W;
* ``linear_lut``    -- the lookup-table route: per group and codebook a table of
                       x . codeword for every entry, then y = s . sum of looked-up
                       values + bias (fp64);
* ``input_grad``    -- dx = dy . W16 in fp64 (n ascending): the gradient of the
                       layer with respect to its input, for fine-tuning through a
                       fixed quantised layer;
* ``half_to_float`` / ``float_to_half`` -- IEEE-754 binary16 conversions written
                       from the format's definition (round to nearest, ties to even).

Sources: the AQLM pages -- repo summary "What it does" (weights as sums of
codebook vectors; PV-Tuning fine-tuning after quantisation), "Key highlights"
(PEFT fine-tuning), inference-research record "Bits" / "Activation scheme" /
"Kernels" / "notes" (fp16 activations, lookup route, dequantise-then-GEMM
route, no group-shared scale), paper record method paragraph.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64


class OracleError(RuntimeError):
    pass


_STATUS = {1: "invalid argument or shape", 2: "code out of range for 2^B entries",
           3: "problem too large for the lookup-table form"}


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.oracle_abi_version.restype = _i
    lib.oracle_max_threads.restype = _i
    lib.oracle_half_to_float.argtypes = [_u16p, _f32p, _i64]
    lib.oracle_float_to_half.argtypes = [_f32p, _u16p, _i64]
    lib.oracle_float_bits_to_half_range.argtypes = [ctypes.c_uint32, _i64, _u16p]
    lib.oracle_dequantize.argtypes = [_vp, _u16p, _u16p, _u16p, _i, _i, _i, _i, _i, _i]
    lib.oracle_dequantize.restype = _i
    lib.oracle_linear_rows.argtypes = [_u16p, _vp, _u16p, _u16p, _u16p, _f64p,
                                       _i, _i, _i, _i, _i, _i, _i64p, _i64, _i]
    lib.oracle_linear_rows.restype = _i
    lib.oracle_input_grad_cols.argtypes = [_u16p, _vp, _u16p, _u16p, _f64p,
                                           _i, _i, _i, _i, _i, _i, _i64p, _i64, _i]
    lib.oracle_input_grad_cols.restype = _i
    for name in ("oracle_linear_exact", "oracle_linear_lut"):
        fn = getattr(lib, name)
        fn.argtypes = [_u16p, _vp, _u16p, _u16p, _u16p, _f64p, _i, _i, _i, _i, _i, _i, _i]
        fn.restype = _i
    return lib


_default_lib = None
_active_lib = None


def _load():
    global _default_lib
    if _active_lib is not None:
        return _active_lib
    if _default_lib is None:
        _default_lib = _bind(_build.build())
    return _default_lib


class use_library:
    """Context manager: route this module's functions to another build of the
    oracle source (the mutation tests use it to run the pins against copies of
    the oracle with a planted mistake)."""

    def __init__(self, path: str):
        self._lib = _bind(path)

    def __enter__(self):
        global _active_lib
        self._prev, _active_lib = _active_lib, self._lib
        return self

    def __exit__(self, *exc):
        global _active_lib
        _active_lib = self._prev
        return False


def _bits16(a) -> np.ndarray:
    """fp16 array (or raw uint16 bit patterns) -> contiguous uint16 bits."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16/uint16 data, got {a.dtype}")
    return np.ascontiguousarray(a)


def _codes(codes, B: int) -> np.ndarray:
    want = np.uint8 if B <= 8 else np.uint16
    codes = np.asarray(codes)
    if codes.dtype != want:
        raise TypeError(f"codes for B={B} must be {np.dtype(want).name}, got {codes.dtype}")
    return np.ascontiguousarray(codes)


def _p(a, t):
    return a.ctypes.data_as(t) if a is not None else None


def _check(rc: int):
    if rc != 0:
        raise OracleError(_STATUS.get(rc, f"status {rc}"))


def max_threads() -> int:
    return _load().oracle_max_threads()


def half_to_float(h) -> np.ndarray:
    h = _bits16(h)
    out = np.empty(h.shape, np.float32)
    _load().oracle_half_to_float(_p(h, _u16p), _p(out, _f32p), h.size)
    return out


def float_to_half(f) -> np.ndarray:
    """Round binary32 values to binary16 (RNE); returns uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(f, dtype=np.float32))
    out = np.empty(f.shape, np.uint16)
    _load().oracle_float_to_half(_p(f, _f32p), _p(out, _u16p), f.size)
    return out


def float_bits_to_half_range(start: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint16)
    _load().oracle_float_bits_to_half_range(start, count, _p(out, _u16p))
    return out


def _shape(codes, codebooks, M, B, g):
    N, G, Mc = codes.shape
    if Mc != M or codebooks.shape != (M, 1 << B, g):
        raise ValueError("codes must be [N, K/g, M] and codebooks [M, 2^B, g]")
    return N, G * g


def dequantize(codes, codebooks, scales, M: int, B: int, g: int, nthreads: int = 0) -> np.ndarray:
    """Returns W16 [N, K] as uint16 bit patterns."""
    codes = _codes(codes, B)
    cb, sc = _bits16(codebooks), _bits16(scales)
    N, K = _shape(codes, cb, M, B, g)
    out = np.empty((N, K), np.uint16)
    _check(_load().oracle_dequantize(codes.ctypes.data, _p(cb, _u16p), _p(sc, _u16p),
                                     _p(out, _u16p), M, B, g, K, N, nthreads))
    return out


def linear(x, codes, codebooks, scales, bias, M: int, B: int, g: int,
           rows=None, nthreads: int = 0) -> np.ndarray:
    """Reference y [batch, N] (or [batch, len(rows)]) in fp64: decode to fp16, then fp64 matmul."""
    codes = _codes(codes, B)
    x, cb, sc = _bits16(x), _bits16(codebooks), _bits16(scales)
    N, K = _shape(codes, cb, M, B, g)
    batch = x.shape[0]
    if x.shape[1] != K:
        raise ValueError("x must be [batch, K]")
    bi = _bits16(bias) if bias is not None else None
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nrows = N if r is None else r.size
    y = np.empty((batch, nrows), np.float64)
    _check(_load().oracle_linear_rows(_p(x, _u16p), codes.ctypes.data, _p(cb, _u16p),
                                      _p(sc, _u16p), _p(bi, _u16p), _p(y, _f64p),
                                      M, B, g, K, N, batch, _p(r, _i64p), nrows, nthreads))
    return y


def _linear_variant(name, x, codes, codebooks, scales, bias, M, B, g, nthreads):
    codes = _codes(codes, B)
    x, cb, sc = _bits16(x), _bits16(codebooks), _bits16(scales)
    N, K = _shape(codes, cb, M, B, g)
    batch = x.shape[0]
    bi = _bits16(bias) if bias is not None else None
    y = np.empty((batch, N), np.float64)
    _check(getattr(_load(), name)(_p(x, _u16p), codes.ctypes.data, _p(cb, _u16p), _p(sc, _u16p),
                                  _p(bi, _u16p), _p(y, _f64p), M, B, g, K, N, batch, nthreads))
    return y


def linear_exact(x, codes, codebooks, scales, bias, M: int, B: int, g: int, nthreads: int = 0):
    return _linear_variant("oracle_linear_exact", x, codes, codebooks, scales, bias, M, B, g, nthreads)


def linear_lut(x, codes, codebooks, scales, bias, M: int, B: int, g: int, nthreads: int = 0):
    return _linear_variant("oracle_linear_lut", x, codes, codebooks, scales, bias, M, B, g, nthreads)


def input_grad(dy, codes, codebooks, scales, M: int, B: int, g: int,
               cols=None, nthreads: int = 0) -> np.ndarray:
    """Reference dx [batch, K] (or [batch, len(cols)]) in fp64: dx = dy . W16, where
    W16 is dequantize()'s fp16 weight and n is summed in ascending order."""
    codes = _codes(codes, B)
    dy, cb, sc = _bits16(dy), _bits16(codebooks), _bits16(scales)
    N, K = _shape(codes, cb, M, B, g)
    batch = dy.shape[0]
    if dy.shape[1] != N:
        raise ValueError("dy must be [batch, N]")
    c = None if cols is None else np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
    ncols = K if c is None else c.size
    dx = np.empty((batch, ncols), np.float64)
    _check(_load().oracle_input_grad_cols(_p(dy, _u16p), codes.ctypes.data, _p(cb, _u16p),
                                          _p(sc, _u16p), _p(dx, _f64p), M, B, g, K, N, batch,
                                          _p(c, _i64p), ncols, nthreads))
    return dx


def library_path() -> str:
    return os.path.abspath(_build.LIBRARY)
