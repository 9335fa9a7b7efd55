"""Every supported codebook shape (M codebooks of 2^B entries, g-wide codewords)
against the oracle, through the C ABI: B = 8 with M = 1..4 and B = 16 with
M = 1..2, each with g = 8 and 16 (the 1-, 2-, 3- and 4-bit variants the AQLM
pages list beside the 1x16 and 2x8 configurations).

* aqlm_dequantize bit for bit;
* aqlm_matmul within 5e-3 on the gather GEMV, the tensor-core path and AUTO, on
  shapes with ragged rows, a K that is not a multiple of 64 and several batch sizes;
* the lookup-table GEMV (batch 1, B = 8) on code rows from 16 bytes (one partial
  slice) to 8192 (16 CTAs x 4 slices), groups that straddle slices (M = 3) and
  ragged row counts;
* integer-valued layers bit for bit on every path.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_additive_b200 import layer as L
from weight_only_additive_b200 import native, synth
from weight_only_additive_b200.native import Path, Status

pytestmark = pytest.mark.gpu

TOL = 5e-3
SCHEMES = [(m, 8, g) for m in (1, 2, 3, 4) for g in (8, 16)] + [(m, 16, g) for m in (1, 2) for g in (8, 16)]


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    native.lib()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


def run(ld, x, dev, path):
    w = L.AqlmWeights.from_numpy(ld, dev)
    y = L.matmul(torch.from_numpy(x).to(dev), w, path=path)
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))
    return y.cpu().numpy()


def close(y, y_ref, what):
    assert np.isfinite(y.astype(np.float32)).all(), what
    err = float(np.abs(y.astype(np.float64) - y_ref).max() / max(np.abs(y_ref).max(), 1e-30))
    assert err <= TOL, f"{what}: rel err {err:.3e}"


@pytest.mark.parametrize("M,B,g", SCHEMES)
def test_dequantize_bit_exact(dev, M, B, g):
    for N, K in ((37, 16 * 17), (300, 1024)):
        ld = synth.make_layer(M, B, g, K, N, seed=70, layer=N)
        w = L.AqlmWeights.from_numpy(ld, dev)
        got = L.dequantize(w).cpu().numpy().view(np.uint16)
        want = oracle.dequantize(ld.codes, ld.codebooks, ld.scales, M, B, g)
        assert np.array_equal(got, want), (N, K, int((got != want).sum()))


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("N,K", [(129, 1024), (300, 16 * 17)])
@pytest.mark.parametrize("path,batch", [(Path.GEMV, 1), (Path.GEMV, 5), (Path.TENSOR_CORE, 1),
                                        (Path.TENSOR_CORE, 16), (Path.TENSOR_CORE, 70), (Path.AUTO, 1),
                                        (Path.AUTO, 8)])
def test_matmul_parity(dev, M, B, g, N, K, path, batch):
    ld = synth.make_layer(M, B, g, K, N, seed=71, layer=N + batch, with_bias=(batch % 2 == 1))
    x = synth.make_x(batch, K, seed=71, layer=N)
    y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
    close(run(ld, x, dev, path), y_ref, f"{M}x{B} g{g} N={N} K={K} {path.name} b={batch}")


# (M, g, K, N): code rows of K / g x M bytes, cut into 128-byte slices
LUT_CASES = [(1, 8, 128, 5),            # one 16-byte partial slice
             (4, 8, 256, 64),           # one full slice
             (1, 8, 4096, 1),           # a single row
             (3, 8, 5504, 37),          # 2064-byte rows: 16 slices + 16 bytes, groups straddle slices
             (3, 8, 5504, 300),
             (3, 16, 11008, 129),
             (2, 16, 14336, 200),
             (4, 16, 4096, 4100),       # many row blocks
             (4, 8, 11008, 1000),       # 5504-byte rows: 43 slices
             (4, 8, 11008, 4096),       # code tiles of a CTA do not all fit: slots reloaded
             (3, 8, 11008, 4096),
             (1, 16, 16 * 8192, 70)]    # 8192-byte rows: the longest (16 CTAs x 4 slices)


@pytest.mark.parametrize("M,g,K,N", LUT_CASES)
def test_lut_parity(dev, M, g, K, N):
    ld = synth.make_layer(M, 8, g, K, N, seed=73, layer=N, with_bias=(N % 2 == 1))
    x = synth.make_x(1, K, seed=73, layer=N)
    assert native.aqlm_select_path(M, 8, g, K, N, 1) == Path.GEMV_LUT
    y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, 8, g)
    close(run(ld, x, dev, Path.GEMV_LUT), y_ref, f"lut {M}x8 g{g} N={N} K={K}")


@pytest.mark.parametrize("M,g", [(1, 8), (3, 8), (4, 16)])
def test_lut_deterministic(dev, M, g):
    ld = synth.make_layer(M, 8, g, 4096, 1000, seed=74)
    x = synth.make_x(1, 4096, seed=74)
    a = run(ld, x, dev, Path.GEMV_LUT)
    b = run(ld, x, dev, Path.GEMV_LUT)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("path,batch", [(Path.GEMV, 1), (Path.GEMV, 4), (Path.TENSOR_CORE, 1),
                                        (Path.TENSOR_CORE, 33), (Path.GEMV_LUT, 1)])
def test_integer_layers_bit_exact(dev, M, B, g, path, batch):
    """Small-integer codebooks and x, scales in {1, 2}: every operation is exact in
    fp16/fp32 whatever the order, so y must equal the oracle bit for bit."""
    if path == Path.GEMV_LUT and B != 8:
        pytest.skip("the lookup-table GEMV needs 256-entry codebooks")
    N, K = 200, 512
    rng = np.random.Generator(np.random.PCG64(72 + M))
    cb = rng.integers(-2, 3, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8 if B <= 8 else np.uint16)
    sc = rng.choice(np.array([1.0, 2.0]), size=N).astype(np.float16)
    bias = rng.integers(-3, 4, size=N).astype(np.float16)
    x = rng.integers(-1, 2, size=(batch, K)).astype(np.float16)
    ld = synth.LayerData(M, B, g, K, N, codes, cb, sc, bias)
    y_ref = oracle.linear(x, codes, cb, sc, bias, M, B, g)
    assert np.abs(y_ref).max() <= 2048 and np.array_equal(y_ref, np.round(y_ref))
    y = run(ld, x, dev, path).astype(np.float64)
    assert np.array_equal(y, y_ref), int((y != y_ref).sum())
