"""Checks that pin the CPU oracle to facts fixed outside itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a
hand-derived worked example, a closed form, an exact special case, an
invariant or an independent library.  ``tests/test_oracle_pins.py`` runs them
against the oracle; ``tests/test_oracle_mutants.py`` runs them against copies
of the oracle with a planted mistake and requires every copy to fail one.

Sources for what the layer computes: AQLM repo summary "What it does" (weights
are sums of codebook vectors); inference-research record "AQLM (additive /
multi-codebook quantization)" sections "Bits" (fp16 activations), "Kernels"
(lookup route), "notes" (dequantise-then-fp16-GEMM route; no group-shared
scale); paper record "Extreme Compression of Large Language Models via Additive
Quantization", method paragraph.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _f16(values):
    return np.asarray(values, dtype=np.float64).astype(np.float16)


def _hex16(values):
    return np.asarray([int(v, 16) for v in np.ravel(values)], dtype=np.uint16).reshape(np.shape(values))


def _golden_decode_cases():
    with open(os.path.join(GOLDEN, "decode_worked_examples.json")) as fh:
        return json.load(fh)["cases"]


def _case_arrays(c):
    M, B, g = c["M"], c["B"], c["g"]
    if "codebooks" in c:
        cb = _f16(c["codebooks"]).view(np.uint16)
    else:
        cb = _hex16(c["codebooks_f16_hex"])
    cb = cb.reshape(M, 1 << B, g)
    codes = np.asarray(c["codes"], dtype=np.uint8 if B <= 8 else np.uint16)
    sc = _f16(c["scales"]).view(np.uint16) if "scales" in c else _hex16(c["scales_f16_hex"])
    return M, B, g, cb, codes, sc


# ---------------------------------------------------------------------------
# worked examples (hand-derived, tests/golden/decode_worked_examples.json)
# ---------------------------------------------------------------------------
def pin_golden_decode():
    for c in _golden_decode_cases():
        M, B, g, cb, codes, sc = _case_arrays(c)
        W = oracle.dequantize(codes, cb, sc, M, B, g)
        want = _f16(c["W"]).view(np.uint16) if "W" in c else _hex16(c["W_f16_hex"])
        assert np.array_equal(W, want), (c["name"], [hex(v) for v in W.ravel()])
        if "y" in c:
            x = _f16(c["x"])
            bias = _f16(c["bias"])
            y = oracle.linear(x, codes, cb, sc, bias, M, B, g)
            assert np.array_equal(y, np.asarray(c["y"], dtype=np.float64)), (c["name"], y)
            y_ex = oracle.linear_exact(x, codes, cb, sc, bias, M, B, g)
            assert np.array_equal(y_ex, np.asarray(c["y"], dtype=np.float64)), (c["name"], y_ex)
            y_lut = oracle.linear_lut(x, codes, cb, sc, bias, M, B, g)
            assert np.array_equal(y_lut, np.asarray(c["y"], dtype=np.float64)), (c["name"], y_lut)


# ---------------------------------------------------------------------------
# closed forms and exact special cases
# ---------------------------------------------------------------------------
def pin_identity_codebook_reproduces_w(seed=1, N=48, K=256, g=8, B=16):
    """M=1 and 2^B >= N*G: codeword i is the i-th g-group of a chosen W (row-major),
    code = i, scale = 1, so dequantisation returns W bit for bit."""
    rng = np.random.Generator(np.random.PCG64(seed))
    G = K // g
    W = rng.normal(0, 0.3, size=(N, K)).astype(np.float16)
    cb = np.zeros((1, 1 << B, g), np.float16)
    cb[0, : N * G] = W.reshape(N * G, g)
    perm = rng.permutation(N * G)  # store the groups in a shuffled order
    cb_shuf = np.zeros_like(cb)
    cb_shuf[0, perm] = cb[0, : N * G]
    codes = perm.reshape(N, G, 1).astype(np.uint16 if B > 8 else np.uint8)
    sc = np.ones(N, np.float16)
    got = oracle.dequantize(codes, cb_shuf, sc, 1, B, g)
    assert np.array_equal(got, W.view(np.uint16))
    # with batch rows of one-hot x, linear() returns columns of W exactly
    x = np.zeros((4, K), np.float16)
    cols = rng.choice(K, size=4, replace=False)
    x[np.arange(4), cols] = 1
    y = oracle.linear(x, codes, cb_shuf, sc, None, 1, B, g)
    assert np.array_equal(y, W[:, cols].T.astype(np.float64))


def _integer_layer(seed, M, B, g, K, N, batch):
    rng = np.random.Generator(np.random.PCG64(seed))
    cb = rng.integers(-3, 4, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8 if B <= 8 else np.uint16)
    sc = rng.choice(np.array([0.5, 1.0, 2.0]), size=N).astype(np.float16)
    x = rng.integers(-2, 3, size=(batch, K)).astype(np.float16)
    bias = rng.integers(-4, 5, size=N).astype(np.float16)
    return cb, codes, sc, x, bias


def pin_integer_layer_exact(seed=2, M=2, B=8, g=8, K=256, N=96, batch=3):
    """Small-integer codebooks, x and power-of-two scales make every fp32/fp64
    operation exact, so the result is the exact integer arithmetic (int64 numpy)."""
    cb, codes, sc, x, bias = _integer_layer(seed, M, B, g, K, N, batch)
    cb_i = cb.astype(np.int64)
    # exact weights times 2 (scales are 0.5, 1 or 2) as integers
    s2 = (sc.astype(np.float64) * 2).astype(np.int64)
    groups = np.zeros((N, K // g, g), np.int64)
    for m in range(M):
        groups += cb_i[m][codes[:, :, m].astype(np.int64)]
    W2 = groups.reshape(N, K) * s2[:, None]
    W = oracle.dequantize(codes, cb, sc, M, B, g)
    assert np.array_equal(oracle.half_to_float(W).astype(np.float64) * 2, W2.astype(np.float64))
    y2 = x.astype(np.int64) @ W2.T + 2 * bias.astype(np.int64)[None, :]
    for fn in (oracle.linear, oracle.linear_exact, oracle.linear_lut):
        y = fn(x, codes, cb, sc, bias, M, B, g)
        assert np.array_equal(y * 2, y2.astype(np.float64)), fn.__name__
    # the input gradient of the same layer: dy . W, exact in int64 (times 2)
    dy = np.random.Generator(np.random.PCG64(seed + 100)).integers(-2, 3, size=(batch, N)).astype(np.float16)
    dx2 = dy.astype(np.int64) @ W2
    assert np.array_equal(oracle.input_grad(dy, codes, cb, sc, M, B, g) * 2, dx2.astype(np.float64))


def pin_brute_force_tiny():
    """Every code assignment of tiny layers (M in {1,2}, B in {1,2,3}, g in {1,2},
    K in {g, 2g}) against sums expanded term by term in Python floats.  Codebook
    values are multiples of 1/8 below 4, so every sum is exact."""
    rng = np.random.Generator(np.random.PCG64(3))
    for M, B, g, groups in itertools.product((1, 2), (1, 2, 3), (1, 2), (1, 2)):
        K = g * groups
        E = 1 << B
        cb = (rng.integers(-32, 33, size=(M, E, g)) / 8.0).astype(np.float16)
        x = (rng.integers(-8, 9, size=(1, K)) / 4.0).astype(np.float16)
        assignments = list(itertools.product(range(E), repeat=M * groups))
        N = len(assignments)
        codes = np.asarray(assignments, dtype=np.uint8).reshape(N, groups, M)
        sc = np.full(N, 0.5, np.float16)
        W = oracle.half_to_float(oracle.dequantize(codes, cb, sc, M, B, g)).astype(np.float64)
        y = oracle.linear(x, codes, cb, sc, None, M, B, g)
        cbf = cb.astype(np.float64)
        xf = x.astype(np.float64)[0]
        for n, a in enumerate(assignments):
            yy = 0.0
            for j in range(groups):
                for t in range(g):
                    w = 0.0
                    for m in range(M):
                        w += cbf[m, a[j * M + m], t]
                    w *= 0.5
                    assert W[n, j * g + t] == w, (M, B, g, groups, a, j, t)
                    yy += xf[j * g + t] * w
            assert y[0, n] == yy, (M, B, g, groups, a)


def pin_one_hot_codewords_closed_form(seed=4, M=2, B=8, g=8, K=512, N=64, batch=2):
    """Codeword i of codebook m is v[m,i] on coordinate (i mod g) and zero elsewhere.
    Then y[b,n] = s_n * sum_j sum_m v[m, c] * x[b, j*g + (c mod g)] with c = codes[n,j,m]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    E = 1 << B
    v = rng.normal(0, 0.5, size=(M, E)).astype(np.float16)
    cb = np.zeros((M, E, g), np.float16)
    for m in range(M):
        cb[m, np.arange(E), np.arange(E) % g] = v[m]
    codes = rng.integers(0, E, size=(N, K // g, M)).astype(np.uint8)
    sc = rng.uniform(0.5, 1.5, size=N).astype(np.float16)
    x = rng.normal(0, 1, size=(batch, K)).astype(np.float16)
    xf, vf, sf = x.astype(np.float64), v.astype(np.float64), sc.astype(np.float64)
    j_idx = np.arange(K // g)[None, :, None] * g
    pos = j_idx + (codes.astype(np.int64) % g)                      # [N, G, M]
    vals = vf[np.arange(M)[None, None, :], codes.astype(np.int64)]   # [N, G, M]
    want = np.stack([sf * (vals * xf[b][pos]).sum(axis=(1, 2)) for b in range(batch)])
    got = oracle.linear_exact(x, codes, cb, sc, None, M, B, g)
    assert np.allclose(got, want, rtol=0, atol=1e-12 * np.abs(want).max())
    got_lut = oracle.linear_lut(x, codes, cb, sc, None, M, B, g)
    assert np.allclose(got_lut, want, rtol=0, atol=1e-12 * np.abs(want).max())


def pin_reference_matches_numpy_matmul(seed=5, M=2, B=8, g=8, K=384, N=80, batch=5):
    """linear() = numpy fp64 x @ W16^T (an independent BLAS), W16 from dequantize()."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cb = rng.normal(0, 0.05, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8)
    sc = rng.uniform(0.5, 1.5, size=N).astype(np.float16)
    x = rng.normal(0, 1, size=(batch, K)).astype(np.float16)
    bias = rng.normal(0, 1, size=N).astype(np.float16)
    W = oracle.dequantize(codes, cb, sc, M, B, g)
    want = x.astype(np.float64) @ W.view(np.float16).astype(np.float64).T + bias.astype(np.float64)
    got = oracle.linear(x, codes, cb, sc, bias, M, B, g)
    assert np.allclose(got, want, rtol=0, atol=1e-13 * np.abs(want).max())


def pin_lut_route_equals_decode_route(seed=6):
    """The lookup-table route and the exact-codeword route are the same product in
    two summation orders: they agree to 1e-12 (fp64).  The fp16-rounded-W
    reference stays within the bound that rounding W to fp16 allows."""
    rng = np.random.Generator(np.random.PCG64(seed))
    for (M, B, g, K, N, batch) in ((2, 8, 8, 512, 64, 3), (1, 10, 8, 256, 40, 2), (3, 6, 4, 96, 20, 2)):
        cb = rng.normal(0, 0.05, size=(M, 1 << B, g)).astype(np.float16)
        codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8 if B <= 8 else np.uint16)
        sc = rng.uniform(0.5, 1.5, size=N).astype(np.float16)
        x = rng.normal(0, 1, size=(batch, K)).astype(np.float16)
        bias = rng.normal(0, 1, size=N).astype(np.float16)
        y_ex = oracle.linear_exact(x, codes, cb, sc, bias, M, B, g)
        y_lut = oracle.linear_lut(x, codes, cb, sc, bias, M, B, g)
        scale = np.abs(y_ex).max()
        assert np.abs(y_ex - y_lut).max() <= 1e-12 * scale, (M, B, g)
        # |y_ref - y_ex| <= sum_k |x_k| * |W_k| * 2^-11 (+ fp32 sum/scale rounding, 2^-23 each)
        y_ref = oracle.linear(x, codes, cb, sc, bias, M, B, g)
        W = oracle.half_to_float(oracle.dequantize(codes, cb, sc, M, B, g)).astype(np.float64)
        bound = np.abs(x.astype(np.float64)) @ np.abs(W).T * (2.0 ** -11 + M * 2.0 ** -22) + 1e-12
        assert np.all(np.abs(y_ref - y_ex) <= bound), (M, B, g)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
def pin_invariants(seed=7, M=2, B=8, g=8, K=256, N=64, batch=2):
    rng = np.random.Generator(np.random.PCG64(seed))
    cb = rng.normal(0, 0.05, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8)
    sc = rng.uniform(0.5, 1.5, size=N).astype(np.float16)
    x = rng.normal(0, 1, size=(batch, K)).astype(np.float16)
    bias = rng.normal(0, 1, size=N).astype(np.float16)
    y = oracle.linear(x, codes, cb, sc, bias, M, B, g)
    # zero codebooks -> y == bias
    yz = oracle.linear(x, codes, np.zeros_like(cb), sc, bias, M, B, g)
    assert np.array_equal(yz, np.broadcast_to(bias.astype(np.float64), yz.shape))
    # exact scaling by powers of two.  Doubling x is exact in fp16 and fp64, so the
    # reference doubles exactly.  Doubling s doubles the fp64 exact form exactly; the
    # fp16-W form is only exact where s*a stays out of the binary16 subnormal range.
    y_nb = oracle.linear(x, codes, cb, sc, None, M, B, g)
    y2x = oracle.linear((x.astype(np.float32) * 2).astype(np.float16), codes, cb, sc, None, M, B, g)
    assert np.array_equal(y2x, 2 * y_nb)
    s2 = (sc.astype(np.float32) * 2).astype(np.float16)
    y_ex = oracle.linear_exact(x, codes, cb, sc, None, M, B, g)
    assert np.array_equal(oracle.linear_exact(x, codes, cb, s2, None, M, B, g), 2 * y_ex)
    W1 = oracle.half_to_float(oracle.dequantize(codes, cb, sc, M, B, g))
    W2 = oracle.half_to_float(oracle.dequantize(codes, cb, s2, M, B, g))
    normal = np.abs(W1) >= 2.0 ** -14
    assert np.array_equal(W2[normal], 2 * W1[normal])
    # permuting a codebook's entries together with its codes changes nothing
    W = oracle.dequantize(codes, cb, sc, M, B, g)
    perm = rng.permutation(1 << B)
    cb_p = cb.copy()
    codes_p = codes.copy()
    cb_p[1, perm] = cb[1]
    codes_p[:, :, 1] = perm[codes[:, :, 1]]
    assert np.array_equal(oracle.dequantize(codes_p, cb_p, sc, M, B, g), W)
    # swapping the two codebooks (and their code slots) changes nothing for M=2
    assert np.array_equal(oracle.dequantize(codes[:, :, ::-1].copy(), cb[::-1].copy(), sc, M, B, g), W)
    # batch rows are independent; row subsets equal the full result
    y0 = oracle.linear(x[:1], codes, cb, sc, bias, M, B, g)
    assert np.array_equal(y0, y[:1])
    rows = np.array([N - 1, 0, 17])
    assert np.array_equal(oracle.linear(x, codes, cb, sc, bias, M, B, g, rows=rows), y[:, rows])
    # the scale multiplies the whole output row
    sc1 = np.ones_like(sc)
    y_s1 = oracle.linear_exact(x, codes, cb, sc1, None, M, B, g)
    y_s = oracle.linear_exact(x, codes, cb, sc, None, M, B, g)
    assert np.allclose(y_s, y_s1 * sc.astype(np.float64)[None, :], rtol=1e-13, atol=0)


ALL_PINS = [pin_golden_decode, pin_identity_codebook_reproduces_w, pin_integer_layer_exact,
            pin_brute_force_tiny, pin_one_hot_codewords_closed_form,
            pin_reference_matches_numpy_matmul, pin_lut_route_equals_decode_route, pin_invariants]


# ---------------------------------------------------------------------------
# binary16 conversions (fast subset; tests/test_oracle_fp16.py is exhaustive)
# ---------------------------------------------------------------------------
# ---------------------------------------------------------------------------
# input gradient dx = dy . W16 (fine-tuning through a fixed quantised layer)
# ---------------------------------------------------------------------------
def pin_golden_input_grad():
    """Hand-derived worked example, tests/golden/input_grad_worked_example.json."""
    with open(os.path.join(GOLDEN, "input_grad_worked_example.json")) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        M, B, g, cb, codes, sc = _case_arrays(c)
        W = oracle.dequantize(codes, cb, sc, M, B, g)
        assert np.array_equal(W, _f16(c["W"]).view(np.uint16)), c["name"]
        dx = oracle.input_grad(_f16(c["dy"]), codes, cb, sc, M, B, g)
        assert np.array_equal(dx, np.asarray(c["dx"], dtype=np.float64)), (c["name"], dx)
        cols = [3, 0]
        dx_cols = oracle.input_grad(_f16(c["dy"]), codes, cb, sc, M, B, g, cols=cols)
        assert np.array_equal(dx_cols, np.asarray(c["dx"], dtype=np.float64)[:, cols]), c["name"]


def pin_input_grad_matches_numpy(seed=11, M=3, B=8, g=16, K=320, N=72, batch=4):
    """input_grad() = numpy fp64 dy @ W16 (an independent BLAS), W16 from dequantize()."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cb = rng.normal(0, 0.05, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8)
    sc = rng.uniform(0.5, 1.5, size=N).astype(np.float16)
    dy = rng.normal(0, 1, size=(batch, N)).astype(np.float16)
    W = oracle.dequantize(codes, cb, sc, M, B, g).view(np.float16).astype(np.float64)
    want = dy.astype(np.float64) @ W
    got = oracle.input_grad(dy, codes, cb, sc, M, B, g)
    assert np.allclose(got, want, rtol=0, atol=1e-13 * np.abs(want).max())
    cols = rng.choice(K, size=17, replace=False)
    assert np.array_equal(oracle.input_grad(dy, codes, cb, sc, M, B, g, cols=cols), got[:, cols])


def pin_input_grad_is_the_adjoint_of_linear(seed=12, K=256, N=96, batch=3):
    """<dx, x> = <dy, y - bias> for every x: input_grad() is the transpose of the very
    operator linear() applies (same W16, same scale, same index layout), checked on
    schemes with one and two byte codes."""
    rng = np.random.Generator(np.random.PCG64(seed))
    for M, B, g in ((2, 8, 8), (1, 16, 8), (2, 16, 16)):
        cb = rng.normal(0, 0.05, size=(M, 1 << B, g)).astype(np.float16)
        codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8 if B <= 8 else np.uint16)
        sc = rng.uniform(0.5, 1.5, size=N).astype(np.float16)
        bias = rng.normal(0, 1, size=N).astype(np.float16)
        x = rng.normal(0, 1, size=(batch, K)).astype(np.float16)
        dy = rng.normal(0, 1, size=(batch, N)).astype(np.float16)
        y = oracle.linear(x, codes, cb, sc, bias, M, B, g)
        dx = oracle.input_grad(dy, codes, cb, sc, M, B, g)
        lhs = (dx * x.astype(np.float64)).sum(axis=1)
        rhs = (dy.astype(np.float64) * (y - bias.astype(np.float64))).sum(axis=1)
        scale = np.abs(dx).sum() * np.abs(x.astype(np.float64)).max()
        assert np.allclose(lhs, rhs, rtol=0, atol=1e-12 * scale), (M, B, g, lhs, rhs)


def pin_fp16_conversions():
    import math
    import warnings
    with open(os.path.join(GOLDEN, "fp16_rounding.json")) as fh:
        cases = json.load(fh)["cases"]
    bits = np.array([int(c["f32"], 16) for c in cases], dtype=np.uint32)
    want = np.array([int(c["f16"], 16) for c in cases], dtype=np.uint16)
    assert np.array_equal(oracle.float_to_half(bits.view(np.float32)), want)
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.half_to_float(h)
    finite = (h & 0x7C00) != 0x7C00
    for v in h[finite][::97]:
        e, f = (int(v) >> 10) & 31, int(v) & 1023
        mag = math.ldexp(f, -24) if e == 0 else math.ldexp(1024 + f, e - 25)
        ref = -mag if v >> 15 else mag
        assert got[v] == ref and math.copysign(1, got[v]) == math.copysign(1, ref), hex(int(v))
    rng = np.random.Generator(np.random.PCG64(8))
    u = rng.integers(0x30000000, 0x48000000, size=1 << 18, dtype=np.uint64).astype(np.uint32)
    u |= (rng.integers(0, 2, size=u.size).astype(np.uint32) << 31)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        ref16 = u.view(np.float32).astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.float_to_half(u.view(np.float32)), ref16)


ALL_PINS += [pin_fp16_conversions, pin_golden_input_grad, pin_input_grad_matches_numpy,
             pin_input_grad_is_the_adjoint_of_linear]
