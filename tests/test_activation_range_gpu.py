"""Every kernel family against the CPU oracle on activations with the spread of a
real fp16 layer input, through the C ABI.

The pages fix the activations as fp16 (w2a16 / w3a16: inference-research record
"AQLM (additive / multi-codebook quantization)", sections "Bits" and "Activation
scheme").  Inputs of trained LLM layers are not N(0, 1): they carry a wide spread
and a few outlier channels hundreds to thousands of times larger.  Here
x ~ N(0, sigma), sigma in {1, 8, 32}, alone or with 4 outlier channels of
magnitude 500..2000, and every path must still meet the layer's bar,
max|y - y_ref| / max|y_ref| <= 5e-3 with no NaN/Inf, element by element against
the oracle's fp64 reference of the decoded weights.  The lookup-table kernels
round x . codeword table entries to fp16 and accumulate them in fp32; the
tensor-core kernels take x itself as an fp16 MMA operand.

Each test prints its error ("range-err ..." lines, visible with pytest -s).
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
RANGES = [(1.0, 0), (8.0, 0), (32.0, 0), (1.0, 4), (8.0, 4), (32.0, 4)]
RANGE_IDS = [f"sigma{int(s)}-out{o}" for s, o in RANGES]


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    native.lib()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


def rel_err(y_gpu, y_ref):
    return float(np.abs(y_gpu.astype(np.float64) - y_ref).max() / max(np.abs(y_ref).max(), 1e-30))


def check(y_gpu, y_ref, what):
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))
    assert np.isfinite(y_gpu.astype(np.float32)).all(), f"{what}: non-finite output"
    err = rel_err(y_gpu, y_ref)
    print(f"range-err {what} {err:.3e} (max|y_ref| {np.abs(y_ref).max():.1f})")
    assert err <= TOL, f"{what}: rel err {err:.3e} > {TOL}"


def x_for(batch, K, sigma, n_out, seed, layer=0):
    return synth.make_x_outliers(batch, K, sigma=sigma, n_outliers=n_out, seed=seed, layer=layer)


# single-layer calls: (M, B, g, K, N, batch, path); the lookup-table kernel takes every
# B = 8 scheme at batch 1 (2x8 g8 its tuned build, 4x8 g8 and 1x8 g16 the stacked one),
# the tensor-core kernel every scheme and batch, the gather GEMV batches up to 8
LAYER_CASES = [
    (2, 8, 8, 4096, 1000, 1, Path.GEMV_LUT),
    (4, 8, 8, 4096, 1000, 1, Path.GEMV_LUT),
    (1, 8, 16, 4096, 1000, 1, Path.GEMV_LUT),
    (2, 8, 8, 4096, 1000, 1, Path.TENSOR_CORE),
    (2, 8, 8, 4096, 1000, 70, Path.TENSOR_CORE),
    (1, 16, 8, 4096, 1000, 1, Path.TENSOR_CORE),
    (1, 16, 8, 4096, 1000, 16, Path.TENSOR_CORE),
    (1, 16, 16, 4096, 1000, 5, Path.TENSOR_CORE),
    (1, 16, 8, 4096, 1000, 4, Path.GEMV),
    (2, 8, 8, 4096, 300, 3, Path.GEMV),
]
LAYER_IDS = [f"{M}x{B}g{g}-{path.name}-b{b}" for (M, B, g, K, N, b, path) in LAYER_CASES]


@pytest.mark.parametrize("sigma,n_out", RANGES, ids=RANGE_IDS)
@pytest.mark.parametrize("M,B,g,K,N,batch,path", LAYER_CASES, ids=LAYER_IDS)
def test_layer_activation_range(dev, M, B, g, K, N, batch, path, sigma, n_out):
    ld = synth.make_layer(M, B, g, K, N, seed=70, layer=M * 100 + g, with_bias=True)
    x = x_for(batch, K, sigma, n_out, seed=71, layer=batch)
    w = L.AqlmWeights.from_numpy(ld, dev)
    y = L.matmul(torch.from_numpy(x).to(dev), w, path=path).cpu().numpy()
    y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
    check(y, y_ref, f"{M}x{B}g{g} {path.name} b={batch} sigma={sigma} outliers={n_out}")


# grouped lookup-table kernel: a 2x8 g8 set (tuned build) and a generic set
GROUPS = {
    "2x8g8": [(2, 8, 8, 4096, 1000), (2, 8, 8, 11008, 300)],
    "generic": [(3, 8, 8, 4096, 500), (2, 8, 16, 4096, 700), (4, 8, 8, 2048, 200)],
}


@pytest.mark.parametrize("sigma,n_out", RANGES, ids=RANGE_IDS)
@pytest.mark.parametrize("name", sorted(GROUPS))
def test_group_activation_range(dev, name, sigma, n_out):
    specs = GROUPS[name]
    items, refs = [], []
    for i, (M, B, g, K, N) in enumerate(specs):
        ld = synth.make_layer(M, B, g, K, N, seed=72, layer=i, with_bias=(i == 0))
        x = x_for(1, K, sigma, n_out, seed=73, layer=i)
        out = torch.full((1, N), float("nan"), dtype=torch.float16, device=dev)
        items.append((L.AqlmWeights.from_numpy(ld, dev), torch.from_numpy(x).to(dev), out))
        refs.append(oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g))
    L.LayerGroup(items).run()
    for (_, _, out), y_ref, (M, B, g, K, N) in zip(items, refs, specs):
        check(out.cpu().numpy(), y_ref, f"group[{name}] {M}x{B}g{g} {N}x{K} sigma={sigma} outliers={n_out}")


@pytest.mark.parametrize("sigma,n_out", RANGES, ids=RANGE_IDS)
@pytest.mark.parametrize("M,B,g", [(2, 8, 8), (1, 16, 8)])
def test_input_grad_activation_range(dev, M, B, g, sigma, n_out):
    K, N, batch = 1024, 512, 32
    ld = synth.make_layer(M, B, g, K, N, seed=74, layer=M)
    dy = x_for(batch, N, sigma, n_out, seed=75)
    dx = L.input_grad(torch.from_numpy(dy).to(dev), L.AqlmWeights.from_numpy(ld, dev)).cpu().numpy()
    dx_ref = oracle.input_grad(dy, ld.codes, ld.codebooks, ld.scales, M, B, g)
    check(dx, dx_ref, f"input-grad {M}x{B}g{g} sigma={sigma} outliers={n_out}")
