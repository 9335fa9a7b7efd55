"""libaqlm_cpu.so (the multithreaded host-CPU kernel) against the CPU oracle.

The same bar as the GPU path: max|y - y_ref| / max|y_ref| <= 5e-3 against the
oracle's fp64 reference of the decoded fp16 weights, no NaN/Inf, for every
supported scheme on both methods (lookup tables for B = 8 at batch <= 8, decode +
dot otherwise, and the fused decode + dot with AVX-512); integer-valued layers bit
for bit; the same bits run to run for a given thread count; argument errors before any
work.  The numeric tests run at every SIMD level this CPU has (scalar, AVX2, AVX-512),
selected with the library's process-wide cap.  No GPU is involved.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from weight_only_additive_b200 import build as lib_build
from weight_only_additive_b200 import cpu, synth
from weight_only_additive_b200.native import Status

TOL = 5e-3
SCHEMES = [(m, 8, g) for m in (1, 2, 3, 4) for g in (8, 16)] + [(m, 16, g) for m in (1, 2) for g in (8, 16)]
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "aqlm_cpu.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    lib_build.build_cpu()
    cpu.lib()


@pytest.fixture(params=[0, 1, 2], ids=["scalar", "avx2", "avx512"])
def simd(request):
    """Runs the test with the SIMD level capped at the parameter (skipped where the CPU
    lacks it); the previous cap is restored afterwards."""
    prev = cpu.set_max_simd_level(request.param)
    try:
        if cpu.simd_level() != request.param:
            pytest.skip(f"this CPU has no SIMD level {request.param}")
        yield request.param
    finally:
        cpu.set_max_simd_level(prev)


def close(y, ref, what):
    assert np.isfinite(y.astype(np.float32)).all(), what
    err = float(np.abs(y.astype(np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))
    assert err <= TOL, f"{what}: rel err {err:.3e}"


def test_header_declares_the_binding_exports():
    text = open(HEADER).read()
    declared = sorted(set(re.findall(r"\b(aqlm_cpu_\w+)\s*\(", text)))
    assert declared == sorted(cpu.EXPORTS)
    for name in cpu.EXPORTS:
        assert isinstance(getattr(cpu.lib(), name), ctypes._CFuncPtr)
    assert cpu.simd_level() in (0, 1, 2)


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("batch", [1, 3, 8, 9])
def test_cpu_matmul_matches_oracle(M, B, g, batch, simd):
    N, K = 150, 16 * 37  # several table slices and a partial one; ragged rows
    ld = synth.make_layer(M, B, g, K, N, seed=80, layer=batch, with_bias=batch % 2 == 1)
    x = synth.make_x(batch, K, seed=81, layer=M)
    ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
    for nt in (1, 4):
        close(cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g, nthreads=nt), ref,
              f"{M}x{B} g{g} b={batch} threads={nt} simd={simd}")


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("batch", [1, 20])
def test_cpu_matmul_integer_layers_bit_exact(M, B, g, batch, simd):
    N, K = 70, 512
    rng = np.random.Generator(np.random.PCG64(82 + M + g + B))
    cb = rng.integers(-2, 3, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8 if B <= 8 else np.uint16)
    sc = rng.choice(np.array([1.0, 2.0]), size=N).astype(np.float16)
    bias = rng.integers(-3, 4, size=N).astype(np.float16)
    x = rng.integers(-1, 2, size=(batch, K)).astype(np.float16)
    ref = oracle.linear(x, codes, cb, sc, bias, M, B, g)
    assert np.abs(ref).max() <= 2048
    for nt in (1, 3):
        y = cpu.matmul(x, codes, cb, sc, bias, M, B, g, nthreads=nt).astype(np.float64)
        assert np.array_equal(y, ref), (nt, int((y != ref).sum()))


@pytest.mark.parametrize("M,B,g", [(2, 8, 8), (3, 8, 8), (1, 16, 8), (2, 16, 8)])
@pytest.mark.parametrize("batch", [1, 2, 5, 17])
def test_cpu_matmul_odd_group_count_and_batch_chunks(M, B, g, batch, simd):
    """K = 8 * 75 (an odd number of g = 8 groups: the last group has no partner in a
    16-weight step), N = 101 (no multiple of any row block), and batches that leave a
    partial chunk of 8."""
    N, K = 101, 8 * 75
    ld = synth.make_layer(M, B, g, K, N, seed=86, layer=batch, with_bias=True)
    x = synth.make_x(batch, K, seed=87, layer=M)
    ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
    for nt in (1, 5):
        close(cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g, nthreads=nt), ref,
              f"{M}x{B} g{g} b={batch} threads={nt} simd={simd}")


def test_cpu_fused_method_independent_of_thread_count():
    """At SIMD level 2 everything but B = 8 at batch 1 takes the fused decode + dot,
    where each output row is summed by one thread in one order: any thread count gives
    the same bits."""
    if cpu.simd_level() < 2:
        pytest.skip("this CPU has no AVX-512")
    for M, B, g, batch in ((2, 8, 8, 4), (1, 16, 8, 1), (2, 16, 16, 9)):
        ld = synth.make_layer(M, B, g, 1024, 300, seed=88)
        x = synth.make_x(batch, 1024, seed=88)
        ys = [cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, None, M, B, g, nthreads=nt).view(np.uint16)
              for nt in (1, 2, 7)]
        assert all(np.array_equal(ys[0], y) for y in ys[1:]), (M, B, g, batch)


def test_cpu_matmul_full_size_layer_sampled_rows(simd):
    """A Llama-2-7B down_proj-shaped layer (4096 x 11008), 2x8 g8, batch 1."""
    ld = synth.make_layer(2, 8, 8, 11008, 4096, seed=83)
    x = synth.make_x(1, 11008, seed=83)
    y = cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, None, 2, 8, 8)
    rows = np.random.Generator(np.random.PCG64(84)).choice(4096, size=64, replace=False)
    ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, 2, 8, 8, rows=rows)
    close(y[:, rows], ref, "4096x11008 2x8 g8")


def test_cpu_matmul_deterministic_for_a_thread_count(simd):
    ld = synth.make_layer(2, 8, 8, 4096, 512, seed=85)
    x = synth.make_x(2, 4096, seed=85)
    a = cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, None, 2, 8, 8, nthreads=4)
    b = cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, None, 2, 8, 8, nthreads=4)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_cpu_matmul_special_values():
    """fp16 rounding of the output: zero codebooks leave the bias (a +0 sum plus a
    -0 bias is +0, as in the oracle's fp64 sum), subnormal and large values pass
    through, and an overflowing sum becomes +inf."""
    M, B, g, K, N = 1, 8, 8, 64, 8
    cb = np.zeros((M, 256, g), np.float16)
    codes = np.zeros((N, K // g, M), np.uint8)
    sc = np.ones(N, np.float16)
    bias = np.array([-0.0, 0.0, 6e-8, -6e-8, 1e-5, 60000, -60000, 1], np.float16)
    x = np.ones((1, K), np.float16)
    y = cpu.matmul(x, codes, cb, sc, bias, M, B, g)
    ref = oracle.linear(x, codes, cb, sc, bias, M, B, g).astype(np.float16)
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16))
    assert y[0, 0].view(np.uint16) == 0  # +0
    cb[0, 0, :] = 60000
    y = cpu.matmul(np.ones((1, K), np.float16), codes, cb, sc, None, M, B, g)
    assert np.isinf(y).all() and (y > 0).all()


@pytest.mark.parametrize("kwargs,want", [
    (dict(M=5), Status.UNSUPPORTED),
    (dict(g=4), Status.UNSUPPORTED),
    (dict(nthreads=-1), Status.INVALID_ARG),
])
def test_cpu_matmul_argument_errors(kwargs, want):
    M, B, g = kwargs.get("M", 2), 8, kwargs.get("g", 8)
    lib = cpu.lib()
    x = np.zeros((1, 64), np.float16)
    codes = np.zeros((4, 64 // 8, 2), np.uint8)
    cb = np.zeros((2, 256, 8), np.float16)
    sc = np.ones(4, np.float16)
    y = np.zeros((1, 4), np.float16)
    st = lib.aqlm_cpu_matmul(x.ctypes.data, codes.ctypes.data, cb.ctypes.data, sc.ctypes.data, None,
                             y.ctypes.data, M, B, g, 64, 4, 1, kwargs.get("nthreads", 0))
    assert st == want
    # output overlapping an input, misaligned fp16 pointer, NULL input
    assert lib.aqlm_cpu_matmul(x.ctypes.data, codes.ctypes.data, cb.ctypes.data, sc.ctypes.data, None,
                               x.ctypes.data, 2, 8, 8, 64, 4, 1, 0) == Status.INVALID_ARG
    assert lib.aqlm_cpu_matmul(x.ctypes.data + 1, codes.ctypes.data, cb.ctypes.data, sc.ctypes.data, None,
                               y.ctypes.data, 2, 8, 8, 64, 4, 1, 0) == Status.MISALIGNED
    assert lib.aqlm_cpu_matmul(None, codes.ctypes.data, cb.ctypes.data, sc.ctypes.data, None,
                               y.ctypes.data, 2, 8, 8, 64, 4, 1, 0) == Status.INVALID_ARG


@pytest.mark.parametrize("M,B,g", SCHEMES)
def test_cpu_matmul_degenerate_shapes(M, B, g, simd):
    """One output row, one or two groups of K (for g = 8 a single group is the fused
    method's odd-group tail alone), batch 1 and 9, more threads than rows or slices."""
    for N, K, batch in ((1, g, 1), (1, g, 9), (3, 2 * g, 1), (2, g, 2)):
        ld = synth.make_layer(M, B, g, K, N, seed=89, layer=N + K, with_bias=True)
        x = synth.make_x(batch, K, seed=90, layer=M)
        ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        for nt in (1, 8):
            close(cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g, nthreads=nt), ref,
                  f"{M}x{B} g{g} N={N} K={K} b={batch} threads={nt} simd={simd}")


def test_binding_rejects_mis_sized_bias_and_output():
    """The kernel reads N bias values and writes batch x N outputs: the binding checks
    both sizes before the call."""
    ld = synth.make_layer(2, 8, 8, 64, 16, seed=91, with_bias=True)
    x = synth.make_x(2, 64, seed=91)
    with pytest.raises(ValueError):
        cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, ld.bias[:8].copy(), 2, 8, 8)
    with pytest.raises(ValueError):
        cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, ld.bias, 2, 8, 8, out=np.empty((1, 16), np.float16))
    with pytest.raises(ValueError):
        cpu.matmul(x[0], ld.codes, ld.codebooks, ld.scales, ld.bias, 2, 8, 8)
    out = np.empty((2, 16), np.float16)
    assert cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, ld.bias, 2, 8, 8, out=out) is out


try:
    import hypothesis.strategies as hst
    from hypothesis import HealthCheck, given, settings
except ImportError:  # pragma: no cover
    hst = None


if hst is not None:
    @settings(max_examples=300, deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))
    @given(scheme=hst.sampled_from(SCHEMES), N=hst.integers(1, 300), G=hst.integers(1, 40),
           batch=hst.integers(1, 20), nt=hst.integers(1, 8), level=hst.integers(0, 2),
           bias=hst.booleans(), seed=hst.integers(0, 1000))
    def test_cpu_matmul_random_shapes(scheme, N, G, batch, nt, level, bias, seed):
        """Random shapes against the oracle at a random SIMD level (capped to what the
        CPU has): partial slices, groups that straddle them, batch chunk remainders.

        At least 64 outputs per case: the bar is relative to the layer's largest output,
        and with a handful of outputs that maximum can cancel to near zero, where the
        accepted difference between weights decoded in fp32 (scale on the accumulator)
        and the reference's fp16-rounded W, about 2^-11 of sum |x w| / sqrt(K), is no
        longer small beside it (N = 1 cases with fixed seeds are in
        test_cpu_matmul_degenerate_shapes)."""
        M, B, g = scheme
        K = G * g
        N = max(N, -(-64 // batch))
        ld = synth.make_layer(M, B, g, K, N, seed=seed, layer=N, with_bias=bias)
        x = synth.make_x(batch, K, seed=seed + 1, layer=G)
        ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        prev = cpu.set_max_simd_level(level)
        try:
            y = cpu.matmul(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g, nthreads=nt)
        finally:
            cpu.set_max_simd_level(prev)
        if np.abs(ref).max() > 0:
            close(y, ref, f"{M}x{B} g{g} N={N} K={K} b={batch} threads={nt} level={level}")
