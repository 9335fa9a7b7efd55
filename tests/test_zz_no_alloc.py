"""aqlm_matmul_group_static (the group call on the library's static scratch
buffer) against aqlm_matmul_group (caller workspace) and the oracle.

Collected last on purpose: it must hold both alone and after every other test
has used the library on this device.  Two calls in a row on one stream, with no
synchronisation between them, reuse the static buffer; each must give exactly
the caller-workspace result for its inputs.
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


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    native.lib()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


def _layer_set(dev, seed):
    """Llama-2-7B decoder linears (2x8 g8, batch 1) plus one non-grouped 1x16 layer."""
    w = workloads.get("llama2_7b_layer_set_2x8g8")
    shapes = [(lay.scheme.M, lay.scheme.B, lay.scheme.g, lay.K, lay.N) for lay in w.layers] + [(1, 16, 8, 1024, 300)]
    layers, xs = [], []
    for i, (M, B, g, K, N) in enumerate(shapes):
        ld = synth.make_layer(M, B, g, K, N, seed=seed, layer=i, with_bias=(i % 2 == 1))
        layers.append((ld, L.AqlmWeights.from_numpy(ld, dev)))
        xs.append(synth.make_x(1, K, seed=seed, layer=i))
    return layers, xs


def _problems(layers, xts, outs):
    return native.problem_array([(x.data_ptr(), w.codes.data_ptr(), w.codebooks.data_ptr(), w.scales.data_ptr(),
                                  None if w.bias is None else w.bias.data_ptr(), y.data_ptr(), w.M, w.B, w.g, w.K,
                                  w.N, 1) for (_, w), x, y in zip(layers, xts, outs)])


def test_static_scratch_matches_caller_workspace_on_two_calls_in_a_row(dev):
    layers, xs = _layer_set(dev, seed=50)
    n = len(layers)
    stream = torch.cuda.current_stream(dev).cuda_stream
    inputs = [[torch.from_numpy(x).to(dev) for x in xs], [torch.from_numpy(-2 * x).to(dev) for x in xs]]
    outs_static = [[torch.empty((1, lay[1].N), dtype=torch.float16, device=dev) for lay in layers] for _ in range(2)]
    outs_ws = [[torch.empty((1, lay[1].N), dtype=torch.float16, device=dev) for lay in layers] for _ in range(2)]
    probs_static = [_problems(layers, inputs[c], outs_static[c]) for c in range(2)]
    probs_ws = [_problems(layers, inputs[c], outs_ws[c]) for c in range(2)]
    need = native.aqlm_group_workspace_size(probs_ws[0], n)
    assert 0 < need <= native.STATIC_GROUP_SCRATCH_BYTES
    # two calls in a row on the static buffer, no synchronisation in between
    native.aqlm_matmul_group_static(probs_static[0], stream, count=n)
    native.aqlm_matmul_group_static(probs_static[1], stream, count=n)
    ws = torch.zeros((need,), dtype=torch.uint8, device=dev)
    for c in range(2):
        native.aqlm_matmul_group(probs_ws[c], ws.data_ptr(), need, stream, count=n)
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, hex(detail)
    for c in range(2):
        for i, ((ld, w), a, b) in enumerate(zip(layers, outs_static[c], outs_ws[c])):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"call {c} layer {i}"
    # and both are right: sampled rows against the oracle
    rng = np.random.Generator(np.random.PCG64(51))
    for c, scale in ((0, 1.0), (1, -2.0)):
        for (ld, w), x, y in zip(layers, xs, outs_static[c]):
            rows = np.unique(np.concatenate([rng.choice(w.N, size=16, replace=False), [0, w.N - 1]]))
            xin = (scale * x.astype(np.float32)).astype(np.float16)
            y_ref = oracle.linear(xin, ld.codes, ld.codebooks, ld.scales, ld.bias, w.M, w.B, w.g, rows=rows)
            got = y.cpu().numpy()[:, rows].astype(np.float64)
            err = np.abs(got - y_ref).max() / max(np.abs(y_ref).max(), 1e-30)
            assert np.isfinite(got).all() and err <= TOL, (c, w.N, w.K, err)


def test_static_scratch_rejects_groups_over_its_size(dev):
    """10 grouped 28672 x 8192 layers need 10 x 1835008 bytes of partials > 16 MiB:
    rejected before anything is launched (the fake pointers are never touched)."""
    A = 1 << 40
    step = 1 << 32
    probs = [(A + i * step, A + i * step + (1 << 28), A + i * step + (2 << 28), A + i * step + (3 << 28), None,
              A + i * step + (4 << 28), 2, 8, 8, 8192, 28672, 1) for i in range(10)]
    arr = native.problem_array(probs)
    assert native.aqlm_group_workspace_size(arr, 10) > native.STATIC_GROUP_SCRATCH_BYTES
    assert native.lib().aqlm_static_group_scratch_bytes() == native.STATIC_GROUP_SCRATCH_BYTES
    assert native.lib().aqlm_matmul_group_static(arr, 10, None) == Status.INVALID_ARG


def test_static_scratch_holds_the_mixtral_expert_set(dev):
    """The 24 expert linears of a Mixtral-8x7B layer (2x8 g8, batch 1) need 11 MB of
    partials: one launch on the static buffer, bitwise equal to the caller-workspace
    call and within tolerance of the oracle on sampled rows."""
    w = workloads.get("mixtral_8x7b_experts_2x8g8")
    layers, xs = [], []
    for i, lay in enumerate(w.layers):
        s = lay.scheme
        ld = synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=52, layer=i)
        layers.append((ld, L.AqlmWeights.from_numpy(ld, dev)))
        xs.append(synth.make_x(1, lay.K, seed=52, layer=i))
    xts = [torch.from_numpy(x).to(dev) for x in xs]
    outs_static = [torch.empty((1, lay.N), dtype=torch.float16, device=dev) for lay in w.layers]
    outs_ws = [torch.empty((1, lay.N), dtype=torch.float16, device=dev) for lay in w.layers]
    n = len(layers)
    probs_static = _problems(layers, xts, outs_static)
    probs_ws = _problems(layers, xts, outs_ws)
    need = native.aqlm_group_workspace_size(probs_ws, n)
    assert 8 << 20 < need <= native.STATIC_GROUP_SCRATCH_BYTES
    stream = torch.cuda.current_stream(dev).cuda_stream
    native.aqlm_matmul_group_static(probs_static, stream, count=n)
    ws = torch.zeros((need,), dtype=torch.uint8, device=dev)
    native.aqlm_matmul_group(probs_ws, ws.data_ptr(), need, stream, count=n)
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, hex(detail)
    rng = np.random.Generator(np.random.PCG64(53))
    for i, ((ld, wt), x, a, b) in enumerate(zip(layers, xs, outs_static, outs_ws)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"layer {i}"
        if i % 3 == 0 or i % 3 == 2:  # a w1 and the w2 of every expert
            rows = np.unique(np.concatenate([rng.choice(wt.N, size=12, replace=False), [0, wt.N - 1]]))
            y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, wt.M, wt.B, wt.g, rows=rows)
            got = a.cpu().numpy()[:, rows].astype(np.float64)
            err = np.abs(got - y_ref).max() / max(np.abs(y_ref).max(), 1e-30)
            assert np.isfinite(got).all() and err <= TOL, (i, err)
