"""aqlm_input_grad (dx = dy . diag(s) . W, the layer's input gradient) against the
CPU oracle, through the C ABI.

The bar is aqlm_matmul's: max|dx - dx_ref| / max|dx_ref| <= 5e-3 against the
oracle's fp64 dy . W16, no NaN/Inf; bit for bit on integer-valued layers;
run-to-run bitwise identical.  Every supported scheme, on shapes whose output rows
end in a partial 64-row stage, whose features end in a partial 128-feature tile
where the scheme's code rows allow it, and batch sizes that leave partial and
several batch tiles; full-size published layer shapes on sampled columns.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_additive_b200 import layer as L
from weight_only_additive_b200 import native, synth, workloads
from weight_only_additive_b200.native import Status

pytestmark = pytest.mark.gpu

TOL = 5e-3
SCHEMES = [(m, 8, g) for m in (1, 2, 3, 4) for g in (8, 16)] + [(m, 16, g) for m in (1, 2) for g in (8, 16)]


def supported(M, B, g, K, N):
    row_bytes = K // g * M * (1 if B <= 8 else 2)
    return N % 8 == 0 and row_bytes % 16 == 0


def ragged_k(M, B, g):
    """A K ending in a partial 128-feature tile if the scheme's code rows allow one."""
    for K in (1088, 1216, 1280):
        if supported(M, B, g, K, 8):
            return K
    raise AssertionError


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    native.lib()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


def run(ld, dy, dev):
    w = L.AqlmWeights.from_numpy(ld, dev)
    dx = L.input_grad(torch.from_numpy(dy).to(dev), w)
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))
    return dx.cpu().numpy()


def close(dx, ref, what):
    assert np.isfinite(dx.astype(np.float32)).all(), what
    err = float(np.abs(dx.astype(np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))
    assert err <= TOL, f"{what}: rel err {err:.3e}"


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("batch", [1, 16, 70, 300])
def test_input_grad_matches_oracle(dev, M, B, g, batch):
    for N, K in ((200, 768), (136, ragged_k(M, B, g))):
        ld = synth.make_layer(M, B, g, K, N, seed=90, layer=N + batch)
        dy = synth.make_x(batch, N, seed=91, layer=K)
        ref = oracle.input_grad(dy, ld.codes, ld.codebooks, ld.scales, M, B, g)
        close(run(ld, dy, dev), ref, f"{M}x{B} g{g} N={N} K={K} b={batch}")


@pytest.mark.parametrize("M,B,g", SCHEMES)
def test_input_grad_integer_layers_bit_exact(dev, M, B, g):
    """Small-integer codebooks and dy, scales in {1, 2}: every product and partial
    sum is an exact integer, so dx must equal the oracle bit for bit."""
    N, K, batch = 264, 512, 33
    rng = np.random.Generator(np.random.PCG64(92 + M + g))
    cb = rng.integers(-2, 3, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8 if B <= 8 else np.uint16)
    sc = rng.choice(np.array([1.0, 2.0]), size=N).astype(np.float16)
    dy = rng.integers(-1, 2, size=(batch, N)).astype(np.float16)
    ld = synth.LayerData(M, B, g, K, N, codes, cb, sc, None)
    ref = oracle.input_grad(dy, codes, cb, sc, M, B, g)
    assert np.abs(ref).max() <= 2048 and np.array_equal(ref, np.round(ref))
    dx = run(ld, dy, dev).astype(np.float64)
    assert np.array_equal(dx, ref), int((dx != ref).sum())


def test_input_grad_deterministic(dev):
    ld = synth.make_layer(2, 8, 8, 4096, 1024, seed=93)
    dy = synth.make_x(40, 1024, seed=93)
    a, b = run(ld, dy, dev), run(ld, dy, dev)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_input_grad_zero_codebooks_give_zero(dev):
    ld = synth.make_layer(1, 16, 8, 1024, 256, seed=94)
    ld.codebooks[:] = 0
    dx = run(ld, synth.make_x(5, 256, seed=94), dev)
    assert not np.any(dx.astype(np.float32))


@pytest.mark.parametrize("wname", ["llama2_7b_layer_set_2x8g8", "single_4096x4096_1x16g8",
                                   "mixtral_8x7b_experts_1x16g16"])
def test_input_grad_published_shapes_sampled_columns(dev, wname):
    """Full-size layer shapes of the published workloads (each distinct shape once)
    at a fine-tuning micro-batch of 64 rows; the oracle computes sampled columns."""
    w = workloads.get(wname)
    seen = set()
    rng = np.random.Generator(np.random.PCG64(95))
    for li, lay in enumerate(w.layers):
        if (lay.N, lay.K) in seen:
            continue
        seen.add((lay.N, lay.K))
        s = lay.scheme
        ld = synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=0, workload=w.index, layer=li)
        dy = synth.make_x(64, lay.N, seed=1, workload=w.index, layer=li)
        dx = run(ld, dy, dev)
        cols = np.unique(np.concatenate([rng.choice(lay.K, size=40, replace=False),
                                         [0, 127, 128, lay.K - 1]]))
        ref = oracle.input_grad(dy, ld.codes, ld.codebooks, ld.scales, s.M, s.B, s.g, cols=cols)
        close(dx[:, cols], ref, f"{wname}/{lay.name}")
