"""CUDA path vs the CPU oracle, through the C ABI (libaqlm.so).

* aqlm_dequantize must equal the oracle's decode bit for bit.
* aqlm_matmul must satisfy max|y - y_ref| / max|y_ref| <= 5e-3 (fp16 output)
  against the oracle's fp64 reference of the decoded weights, with no NaN/Inf,
  on every kernel family, on small shapes spanning several tiles with ragged
  tails, on every published layer shape (sampled rows computed one by one by
  the oracle), and bit for bit on integer-valued layers where every operation
  is exact whatever the summation order.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_additive_b200 import layer as L
from weight_only_additive_b200 import native, synth, workloads
from weight_only_additive_b200.native import Path, Status

pytestmark = pytest.mark.gpu

TOL = 5e-3
SCHEMES = [(1, 16, 8), (2, 8, 8), (1, 16, 16)]


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    native.lib()  # raises if the CUDA library is missing: there is no fallback
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


def rel_err(y_gpu, y_ref):
    return float(np.abs(y_gpu.astype(np.float64) - y_ref).max() / max(np.abs(y_ref).max(), 1e-30))


def gpu_matmul(ld, x, dev, path=Path.AUTO):
    w = L.AqlmWeights.from_numpy(ld, dev)
    xt = torch.from_numpy(x).to(dev)
    y = L.matmul(xt, w, path=path)
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))
    return y.cpu().numpy()


def gpu_dequant(ld, dev):
    w = L.AqlmWeights.from_numpy(ld, dev)
    W = L.dequantize(w)
    torch.cuda.synchronize()
    return W.cpu().numpy().view(np.uint16)


def assert_close(y_gpu, y_ref, what):
    assert np.isfinite(y_gpu.astype(np.float32)).all(), f"{what}: non-finite output"
    err = rel_err(y_gpu, y_ref)
    assert err <= TOL, f"{what}: rel err {err:.3e} > {TOL}"
    return err


# ---------------------------------------------------------------------------
# dequantisation: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("N,K", [(1, 16), (37, 16 * 17), (200, 192), (129, 1024), (300, 2064)])
def test_dequantize_bit_exact_small(dev, M, B, g, N, K):
    ld = synth.make_layer(M, B, g, K, N, seed=11, layer=N)
    got = gpu_dequant(ld, dev)
    want = oracle.dequantize(ld.codes, ld.codebooks, ld.scales, M, B, g)
    assert np.array_equal(got, want), int((got != want).sum())


@pytest.mark.parametrize("M,B,g,N,K", [(1, 16, 8, 4096, 4096), (2, 8, 8, 11008, 4096),
                                       (1, 16, 16, 14336, 4096), (2, 8, 8, 4096, 11008)])
def test_dequantize_bit_exact_full_layers(dev, M, B, g, N, K):
    ld = synth.make_layer(M, B, g, K, N, seed=0, workload=99)
    got = gpu_dequant(ld, dev)
    want = oracle.dequantize(ld.codes, ld.codebooks, ld.scales, M, B, g)
    mism = int((got != want).sum())
    assert mism == 0, f"{mism} mismatching weights"


def test_dequantize_golden_edge_values(dev):
    """Signed zeros, overflow to infinity and fp32 double rounding survive on the GPU."""
    # 1x16 g8 layer whose codebook holds the special values
    cb = np.zeros((1, 1 << 16, 8), np.uint16)
    cb[0, 0] = [0x8000, 0x8000, 0x7B53, 0xFB53, 0x3C00, 0x0001, 0x03FF, 0x1000]
    codes = np.zeros((2, 1, 1), np.uint16)
    sc = np.array([0x3C00, 0x4000], np.uint16)  # 1.0, 2.0
    ld = synth.LayerData(1, 16, 8, 8, 2, codes, cb.view(np.float16), sc.view(np.float16), None)
    got = gpu_dequant(ld, dev)
    want = oracle.dequantize(codes, cb, sc, 1, 16, 8)
    assert np.array_equal(got, want), (got, want)
    # 2x8: sum -0 + -0, -0 + +0, ties at fp16 after the fp32 sum
    cb2 = np.zeros((2, 256, 8), np.uint16)
    cb2[0, 1] = [0x8000, 0x8000, 0x3C00, 0x3C00, 0x3C00, 0x7B53, 0x0001, 0x0400]
    cb2[1, 2] = [0x8000, 0x0000, 0x1000, 0x1400, 0x0000, 0x7B53, 0x8001, 0x8400]
    codes2 = np.array([[[1, 2]]], np.uint8)
    sc2 = np.array([0x3C01], np.uint16)
    ld2 = synth.LayerData(2, 8, 8, 8, 1, codes2, cb2.view(np.float16), sc2.view(np.float16), None)
    got2 = gpu_dequant(ld2, dev)
    want2 = oracle.dequantize(codes2, cb2, sc2, 2, 8, 8)
    assert np.array_equal(got2, want2), ([hex(v) for v in got2.ravel()], [hex(v) for v in want2.ravel()])


# ---------------------------------------------------------------------------
# matmul: every kernel family, several tiles with ragged tails
# ---------------------------------------------------------------------------
SMALL_SHAPES = [(1, 16), (37, 16 * 17), (200, 192), (300, 1024), (129, 2064)]


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8])
def test_gemv_parity(dev, M, B, g, N, K, batch):
    ld = synth.make_layer(M, B, g, K, N, seed=12, layer=N + batch, with_bias=(batch % 2 == 1))
    x = synth.make_x(batch, K, seed=12, layer=N)
    y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
    assert_close(gpu_matmul(ld, x, dev, Path.GEMV), y_ref, f"gemv {M}x{B}g{g} N={N} K={K} b={batch}")


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("N,K", SMALL_SHAPES)
@pytest.mark.parametrize("batch", [1, 7, 16, 17, 64, 200, 256, 300])
def test_tensor_core_parity(dev, M, B, g, N, K, batch):
    ld = synth.make_layer(M, B, g, K, N, seed=13, layer=N + batch, with_bias=(batch % 2 == 0))
    x = synth.make_x(batch, K, seed=13, layer=N)
    y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
    assert_close(gpu_matmul(ld, x, dev, Path.TENSOR_CORE), y_ref,
                 f"tc {M}x{B}g{g} N={N} K={K} b={batch}")


@pytest.mark.parametrize("N,K", [(1, 64), (37, 128), (200, 512), (300, 4096), (129, 64 * 23),
                                 (1000, 11008), (700, 14336), (4100, 4096), (2048, 32768)])
def test_gemv_lut_parity(dev, N, K):
    """Lookup-table GEMV (2x8, batch 1): ragged row counts, K from one pass to
    several passes per CTA, cluster sizes from 1 to 16; 2048 x 32768 (the longest rows,
    four passes per CTA) does not keep every code tile resident and recycles slots."""
    ld = synth.make_layer(2, 8, 8, K, N, seed=17, layer=N, with_bias=(N % 2 == 1))
    x = synth.make_x(1, K, seed=17, layer=N)
    y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, 2, 8, 8)
    assert_close(gpu_matmul(ld, x, dev, Path.GEMV_LUT), y_ref, f"lut N={N} K={K}")


@pytest.mark.parametrize("M,B,g", SCHEMES)
@pytest.mark.parametrize("path,batch", [(Path.GEMV, 1), (Path.GEMV, 4), (Path.GEMV, 8),
                                        (Path.GEMV_LUT, 1),
                                        (Path.TENSOR_CORE, 16), (Path.TENSOR_CORE, 100)])
def test_integer_layers_bit_exact(dev, M, B, g, path, batch):
    """Small-integer codebooks and x, scales in {1, 2}: every product and partial sum
    is an exact small integer in fp16/fp32, so any summation order gives the exact
    value and y must equal the oracle bit for bit."""
    if path == Path.GEMV_LUT and B != 8:
        pytest.skip("the lookup-table GEMV needs 256-entry codebooks")
    N, K = 260, 512
    rng = np.random.Generator(np.random.PCG64(14))
    cb = rng.integers(-2, 3, size=(M, 1 << B, g)).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(N, K // g, M)).astype(np.uint8 if B <= 8 else np.uint16)
    sc = rng.choice(np.array([1.0, 2.0]), size=N).astype(np.float16)
    bias = rng.integers(-3, 4, size=N).astype(np.float16)
    x = rng.integers(-1, 2, size=(batch, K)).astype(np.float16)
    ld = synth.LayerData(M, B, g, K, N, codes, cb, sc, bias)
    y_ref = oracle.linear(x, codes, cb, sc, bias, M, B, g)
    assert np.abs(y_ref).max() <= 2048 and np.array_equal(y_ref, np.round(y_ref))
    y = gpu_matmul(ld, x, dev, path).astype(np.float64)
    assert np.array_equal(y, y_ref), int((y != y_ref).sum())


def test_zero_codebooks_give_bias(dev):
    for path, batch in ((Path.GEMV, 3), (Path.TENSOR_CORE, 33)):
        ld = synth.make_layer(2, 8, 8, 256, 70, seed=15, with_bias=True)
        ld.codebooks[:] = 0
        x = synth.make_x(batch, 256, seed=15)
        y = gpu_matmul(ld, x, dev, path)
        assert np.array_equal(y, np.broadcast_to(ld.bias, y.shape))


def test_runs_are_deterministic(dev):
    for (M, B, g), batch, path in (((1, 16, 8), 1, Path.GEMV), ((1, 16, 8), 64, Path.TENSOR_CORE),
                                   ((2, 8, 8), 1, Path.GEMV_LUT)):
        ld = synth.make_layer(M, B, g, 4096, 1000, seed=16)
        x = synth.make_x(batch, 4096, seed=16)
        a = gpu_matmul(ld, x, dev, path)
        b = gpu_matmul(ld, x, dev, path)
        assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


# ---------------------------------------------------------------------------
# every published layer shape, batch sizes as published, AUTO dispatch;
# the oracle computes a sample of rows one by one
# ---------------------------------------------------------------------------
def _sample_rows(N, rng, count=48):
    rows = set(rng.choice(N, size=min(count, N), replace=False).tolist())
    rows.update({0, N - 1, min(127, N - 1), min(128, N - 1)})
    return np.array(sorted(rows), dtype=np.int64)


def _published_cases():
    cases = []
    for w in workloads.WORKLOADS:
        seen = set()
        for li, lay in enumerate(w.layers):
            key = (lay.N, lay.K, lay.scheme)
            if key in seen:
                continue
            seen.add(key)
            for batch in w.batches:
                cases.append(pytest.param(w.name, li, batch, id=f"{w.name}-{lay.name}-b{batch}"))
    return cases


@pytest.mark.parametrize("wname,li,batch", _published_cases())
def test_published_layers_sampled_rows(dev, wname, li, batch):
    w = workloads.get(wname)
    lay = w.layers[li]
    s = lay.scheme
    ld = synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=0, workload=w.index, layer=li)
    x = synth.make_x(batch, lay.K, seed=0, workload=w.index, layer=li)
    y = gpu_matmul(ld, x, dev)
    assert np.isfinite(y.astype(np.float32)).all()
    rows = _sample_rows(lay.N, np.random.Generator(np.random.PCG64(li + 100 * batch)))
    y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, s.M, s.B, s.g, rows=rows)
    assert_close(y[:, rows], y_ref, f"{wname}/{lay.name} b={batch}")


def test_device_status_clean_after_all(dev):
    st, detail = L.check_device_status()
    assert st == Status.OK, hex(detail)


@pytest.mark.parametrize("M,B,g,path,batch", [(2, 8, 8, Path.GEMV_LUT, 1), (2, 8, 8, Path.GEMV, 3),
                                              (1, 16, 8, Path.GEMV, 1), (1, 16, 16, Path.GEMV, 4),
                                              (1, 16, 8, Path.TENSOR_CORE, 64), (2, 8, 8, Path.TENSOR_CORE, 32),
                                              (3, 8, 16, Path.GEMV_LUT, 1), (4, 8, 8, Path.GEMV_LUT, 1)])
def test_chained_layers_read_the_previous_output(dev, M, B, g, path, batch):
    """Kernels start their weight-only set-up while the previous kernel on the stream
    is still running (programmatic dependent launch); x must still be read only after
    that kernel has written it.  Layer 2 consumes layer 1's output, back to back on one
    stream with no synchronisation in between."""
    K = N = 1024
    ld1 = synth.make_layer(M, B, g, K, N, seed=18, layer=1)
    ld2 = synth.make_layer(M, B, g, K, N, seed=18, layer=2)
    x = synth.make_x(batch, K, seed=18)
    w1, w2 = L.AqlmWeights.from_numpy(ld1, dev), L.AqlmWeights.from_numpy(ld2, dev)
    xt = torch.from_numpy(x).to(dev)
    outs = []
    for _ in range(3):  # repeat to give overlapping launches a chance to race
        y1 = L.matmul(xt, w1, path=path)
        y2 = L.matmul(y1, w2, path=path)
        outs.append((y1, y2))
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, hex(detail)
    for y1, y2 in outs:
        y1h = y1.cpu().numpy()
        ref2 = oracle.linear(y1h, ld2.codes, ld2.codebooks, ld2.scales, None, M, B, g)
        assert_close(y2.cpu().numpy(), ref2, f"chained {M}x{B}g{g} {path.name}")
