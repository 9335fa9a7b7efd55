"""Every supported codebook shape (M codebooks of 2^B entries, g-wide codewords)
against the oracle, through the C ABI: B = 8 with M = 1..4 and B = 16 with
M = 1..2, each with g = 8 and 16 (the 1-, 2-, 3- and 4-bit variants the AQLM
pages list beside the 1x16 and 2x8 configurations).

* aqlm_dequantize bit for bit;
* aqlm_matmul within 5e-3 on the gather GEMV, the tensor-core path and AUTO, on
  shapes with ragged rows, a K that is not a multiple of 64 and several batch sizes;
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


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("path,batch", [(Path.GEMV, 1), (Path.GEMV, 4), (Path.TENSOR_CORE, 1),
                                        (Path.TENSOR_CORE, 33)])
def test_integer_layers_bit_exact(dev, M, B, g, path, batch):
    """Small-integer codebooks and x, scales in {1, 2}: every operation is exact in
    fp16/fp32 whatever the order, so y must equal the oracle bit for bit."""
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
