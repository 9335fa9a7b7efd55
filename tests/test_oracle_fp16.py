"""Pins for the oracle's IEEE-754 binary16 conversions.

The oracle writes both directions from the binary16 definition.  They are
pinned against (a) the closed form evaluated in Python integers/floats, (b)
hand-derived rounding cases (tests/golden/fp16_rounding.json) and (c) numpy's
own float16 conversion, an independent implementation.
"""
import json
import math
import os
import warnings

import numpy as np
import pytest

import oracle


def _closed_form(h: int) -> float:
    s = -1.0 if h >> 15 else 1.0
    e = (h >> 10) & 0x1F
    f = h & 0x3FF
    if e == 0:
        return s * math.ldexp(f, -24)
    if e == 31:
        return s * math.inf if f == 0 else math.nan
    return s * math.ldexp(1024 + f, e - 25)


def test_half_to_float_exhaustive_closed_form_and_numpy():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.half_to_float(h)
    ref = np.array([_closed_form(int(v)) for v in h], dtype=np.float64).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))  # signed zeros too
    ref_np = h.view(np.float16).astype(np.float32)
    assert np.array_equal(got[~nan].view(np.uint32), ref_np[~nan].view(np.uint32))


def test_float_to_half_golden_cases(golden_dir):
    with open(os.path.join(golden_dir, "fp16_rounding.json")) as fh:
        cases = json.load(fh)["cases"]
    bits = np.array([int(c["f32"], 16) for c in cases], dtype=np.uint32)
    want = np.array([int(c["f16"], 16) for c in cases], dtype=np.uint16)
    got = oracle.float_to_half(bits.view(np.float32))
    bad = [(c["why"], hex(g)) for c, g, w in zip(cases, got, want) if g != w]
    assert not bad, bad


def _numpy_f2h(u32: np.ndarray) -> np.ndarray:
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        return u32.view(np.float32).astype(np.float16).view(np.uint16)


def _is_nan32(u32):
    return ((u32 & 0x7F800000) == 0x7F800000) & ((u32 & 0x7FFFFF) != 0)


@pytest.mark.parametrize("sign", [0, 1])
def test_float_to_half_exhaustive_over_rounding_exponents(sign):
    """Every binary32 pattern whose exponent lies in [-26, 16] (all values that do
    not trivially flush to zero or overflow) against numpy's conversion.  The
    negative half runs on every 4th exponent to keep the CPU suite short."""
    exps = range(-26, 17) if sign == 0 else range(-26, 17, 4)
    chunk = 1 << 23
    for e in exps:
        start = (sign << 31) | ((e + 127) << 23)
        got = oracle.float_bits_to_half_range(start, chunk)
        u = (np.arange(chunk, dtype=np.uint32) + np.uint32(start)).astype(np.uint32)
        ref = _numpy_f2h(u)
        mism = np.nonzero(got != ref)[0]
        assert mism.size == 0, (e, hex(int(u[mism[0]])), hex(int(got[mism[0]])), hex(int(ref[mism[0]])))


def test_float_to_half_random_patterns_everywhere():
    rng = np.random.Generator(np.random.PCG64(12345))
    u = rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    got = oracle.float_to_half(u.view(np.float32))
    ref = _numpy_f2h(u)
    nan = _is_nan32(u)
    assert np.array_equal(got[~nan], ref[~nan])
    # NaN stays NaN (payloads are not part of the contract)
    assert np.all(((got[nan] & 0x7C00) == 0x7C00) & ((got[nan] & 0x3FF) != 0))


def test_round_trip_half_float_half_is_identity():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = oracle.half_to_float(h)
    back = oracle.float_to_half(f)
    finite = (h & 0x7C00) != 0x7C00
    assert np.array_equal(back[finite], h[finite])
