"""Mutation check of the oracle's pins.

Each mutant is a copy of oracle/aqlm_oracle.cpp with one plausible mistake
planted (a dropped term, a transposed layout, a wrong sign, rounding or
summation precision).  Every mutant must fail at least one pin in
tests/oracle_pins.py; a mutant that passes them all would mean the pins leave
that part of the oracle unchecked.  The mistakes are planted in copies on the
CPU only; the oracle itself is not modified.
"""
import os
import subprocess
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle
from oracle import build as oracle_build
from tests import oracle_pins

MUTANTS = {
    "decode_starts_from_plus_zero": (
        "for (int m = 1; m < s.M; ++m) {\n        a = a +",
        "a = 0.0f + a;\n      for (int m = 1; m < s.M; ++m) {\n        a = a +"),
    "decode_drops_last_codebook": (
        "for (int m = 1; m < s.M; ++m) {\n        a = a +",
        "for (int m = 1; m < s.M - 1; ++m) {\n        a = a +"),
    "decode_sums_in_fp64": (
        "float a = half_bits_to_float(codebook_at(cb, s, 0,",
        "double a = half_bits_to_float(codebook_at(cb, s, 0,"),
    "decode_rounds_sum_to_fp16_before_scale": (
        "const float w = a * scale;",
        "const float w = half_bits_to_float(float_to_half_bits_rne(a)) * scale;"),
    "decode_uses_first_row_scale": (
        "const float scale = half_bits_to_float(scales[n]);",
        "const float scale = half_bits_to_float(scales[0]);"),
    "codes_layout_m_slowest": (
        "const int64_t idx = (n * s.G + j) * s.M + m;",
        "const int64_t idx = (static_cast<int64_t>(m) * s.N + n) * s.G + j;"),
    "codebook_layout_transposed": (
        "return cb[(static_cast<int64_t>(m) * s.entries + i) * s.g + t];",
        "return cb[(static_cast<int64_t>(t) * s.entries + i) * s.M + m];"),
    "reference_shifts_weight_index": (
        "half_bits_to_float(wrow[k])", "half_bits_to_float(wrow[(k + 1) % K])"),
    "reference_drops_bias": (
        "if (bias) acc += static_cast<double>(half_bits_to_float(bias[n]));\n        y[b * nrows + r] = acc;",
        "y[b * nrows + r] = acc;"),
    "exact_form_ignores_scale": (
        "double out = static_cast<double>(half_bits_to_float(scales[n])) * acc;\n      if (bias) out += static_cast<double>(half_bits_to_float(bias[n]));\n      y[b * N + n] = out;\n    }\n  }\n  return 0;\n}\n\n// Lookup",
        "double out = acc;\n      if (bias) out += static_cast<double>(half_bits_to_float(bias[n]));\n      y[b * N + n] = out;\n    }\n  }\n  return 0;\n}\n\n// Lookup"),
    "lut_looks_up_first_codebook_code": (
        "acc += T[(j * M + m) * s.entries + code_at(codes, s, n, j, m)];",
        "acc += T[(j * M + m) * s.entries + code_at(codes, s, n, j, 0)];"),
    "lut_sign_flip": (
        "T[(j * M + m) * s.entries + i] = dot;", "T[(j * M + m) * s.entries + i] = -dot;"),
    "input_grad_reads_dy_transposed": (
        "acc += static_cast<double>(half_bits_to_float(dy[b * N + n])) *",
        "acc += static_cast<double>(half_bits_to_float(dy[n * batch + b])) *"),
    "input_grad_shifts_weight_column": (
        "static_cast<double>(half_bits_to_float(W[n * K + k]));",
        "static_cast<double>(half_bits_to_float(W[n * K + (k + 1) % K]));"),
    "input_grad_skips_first_row": (
        "for (int64_t n = 0; n < N; ++n) {\n        acc += static_cast<double>(half_bits_to_float(dy[",
        "for (int64_t n = 1; n < N; ++n) {\n        acc += static_cast<double>(half_bits_to_float(dy["),
    "input_grad_uses_row_as_column": (
        "static_cast<double>(half_bits_to_float(W[n * K + k]));",
        "static_cast<double>(half_bits_to_float(W[(k % N) * K + (n % K)]));"),
    "half_to_float_subnormal_scale": (
        "mag = std::ldexp(static_cast<float>(f), -24);", "mag = std::ldexp(static_cast<float>(f), -25);"),
    "half_to_float_drops_sign": ("return sign ? -mag : mag;", "return mag;"),
    "float_to_half_ties_away": (
        "if (rem > halfway || (rem == halfway && (q & 1u))) ++q;", "if (rem >= halfway) ++q;"),
    "float_to_half_subnormal_boundary": (
        "const int shift = (e >= -14) ? 13 : (-1 - e);", "const int shift = (e >= -15) ? 13 : (-1 - e);"),
}


@pytest.fixture(scope="module")
def mutant_libs():
    src = open(oracle_build.SOURCE).read()
    tmp = tempfile.mkdtemp(prefix="oracle_mutants_")

    def make(item):
        name, (old, new) = item
        assert src.count(old) == 1, f"{name}: planted-mistake anchor not found exactly once"
        path_cpp = os.path.join(tmp, f"{name}.cpp")
        path_so = os.path.join(tmp, f"{name}.so")
        with open(path_cpp, "w") as fh:
            fh.write(src.replace(old, new))
        subprocess.run(["g++", *oracle_build.FLAGS, "-w", path_cpp, "-o", path_so], check=True)
        return name, path_so

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as pool:
        libs = dict(pool.map(make, MUTANTS.items()))
    return libs


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(mutant_libs, name):
    failed = []
    with oracle.use_library(mutant_libs[name]):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError):
                failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
