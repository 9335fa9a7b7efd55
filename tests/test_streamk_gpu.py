"""The tensor-core kernel on its stream-K schedule (aqlm_matmul_ws, aqlm_input_grad_ws
with a workspace), against the CPU oracle, through the C ABI.

Every SM takes an equal share of the (row tile, batch tile, K stage) space, so a
tile can be cut into pieces done by different CTAs and finished from fp32 partials
in the workspace.  The bar is the layer's own: max|y - y_ref| / max|y_ref| <= 5e-3
against the oracle's fp64 result, no NaN/Inf.  On top of that: the workspace
counters are zero again after every call (the contract that lets calls reuse it),
results are bitwise identical run to run (the pieces are summed in K order whoever
finishes), and the shapes cut tiles into up to 16 pieces, with ragged row tiles,
several batch tiles and a ragged last batch tile.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_additive_b200 import layer as L
from weight_only_additive_b200 import native, synth
from weight_only_additive_b200.native import Path, Schedule, Status

pytestmark = pytest.mark.gpu

TOL = 5e-3


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    native.lib()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


# the counters at the start of every workspace (AQLM_WORKSPACE_COUNTER_BYTES)
CB = native.WORKSPACE_COUNTER_BYTES


def rel_err(y, ref):
    return float(np.abs(y.astype(np.float64) - ref).max() / max(np.abs(ref).max(), 1e-30))


def run_matmul(ld, x, dev, ws, schedule=Schedule.STREAMK):
    """The tensor-core kernel on a forced stream-K schedule (the tile plan when ws is False)."""
    w = L.AqlmWeights.from_numpy(ld, dev)
    sched = Schedule.TILES if ws is False else schedule
    y = L.matmul(torch.from_numpy(x).to(dev), w, path=Path.TENSOR_CORE, workspace=ws, schedule=sched)
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))
    return y.cpu().numpy()


# (M, B, g, N, K, batch, cut): every case runs the forced stream-K schedule; cut = its
# partition certainly cuts tiles (so pieces store partials)
CASES = [
    (2, 8, 8, 256, 4096, 256, True),     # 2 row tiles x 16 units: 16 pieces per tile
    (2, 8, 8, 1000, 2048, 300, True),    # ragged row tile, two batch tiles (the second of 44)
    (2, 8, 8, 11008, 4096, 256, True),   # the published FFN shape: 86 tiles on the SMs
    (2, 8, 8, 300, 1024, 129, True),     # 12 units on 12 CTAs: 4 pieces per tile
    (1, 16, 8, 4096, 4096, 1, True),     # 1x16 g8 at batch 1: 32 tiles of 16 units on the SMs
    (1, 16, 8, 512, 4096, 64, False),
    (3, 8, 8, 600, 2048, 200, False),    # 48-byte code tiles of 2 stages
    (4, 8, 8, 384, 4096, 256, False),    # one decoder group
    (1, 16, 16, 640, 4096, 256, False),  # register-staged B = 16 decode
]


@pytest.mark.parametrize("M,B,g,N,K,batch,cut", CASES)
def test_streamk_matmul_matches_oracle(dev, M, B, g, N, K, batch, cut):
    need = native.aqlm_matmul_workspace_size(M, B, g, K, N, batch)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    ld = synth.make_layer(M, B, g, K, N, seed=140, layer=N + batch, with_bias=True)
    x = synth.make_x(batch, K, seed=141, layer=N)
    y = run_matmul(ld, x, dev, ws)
    assert np.isfinite(y.astype(np.float32)).all()
    if N * batch <= 300 * 1000:
        rows = None
        ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        got = y
    else:  # the oracle computes a sample of rows, tile edges included
        rng = np.random.Generator(np.random.PCG64(N))
        rows = np.unique(np.concatenate([rng.choice(N, 40, replace=False), [0, 127, 128, N - 1]]))
        ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g, rows=rows)
        got = y[:, rows]
    err = rel_err(got, ref)
    assert err <= TOL, f"{M}x{B} g{g} N={N} K={K} b={batch}: rel err {err:.3e}"
    cb = CB
    assert not ws[:cb].any().item(), "tile counters must be zero after the call"
    if cut:
        assert ws[cb:].any().item(), "expected stream-K pieces to have stored partials"


def test_streamk_matches_the_tile_plan_and_is_deterministic(dev):
    """Same layer through the tile plan (no workspace) and twice through stream-K with
    one reused workspace: every result within the tolerance of the oracle, stream-K
    bit-identical run to run."""
    M, B, g, N, K, batch = 2, 8, 8, 640, 4096, 256
    ld = synth.make_layer(M, B, g, K, N, seed=142)
    x = synth.make_x(batch, K, seed=143)
    ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, M, B, g)
    ws = torch.zeros(native.aqlm_matmul_workspace_size(M, B, g, K, N, batch), dtype=torch.uint8, device=dev)
    a = run_matmul(ld, x, dev, ws)
    b = run_matmul(ld, x, dev, ws)
    c = run_matmul(ld, x, dev, False)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    for y, what in ((a, "stream-K"), (c, "tile plan")):
        assert rel_err(y, ref) <= TOL, what


def test_streamk_chained_calls_share_one_workspace(dev):
    """Back-to-back calls on one stream reuse one workspace; the second consumes the
    first's output while the first may still be finishing (programmatic dependent
    launch): the second's epilogue must wait for it before touching the workspace."""
    M, B, g, K, N, batch = 2, 8, 8, 1024, 1024, 256
    ld1 = synth.make_layer(M, B, g, K, N, seed=144, layer=1)
    ld2 = synth.make_layer(M, B, g, K, N, seed=144, layer=2)
    x = synth.make_x(batch, K, seed=145)
    w1, w2 = L.AqlmWeights.from_numpy(ld1, dev), L.AqlmWeights.from_numpy(ld2, dev)
    ws = torch.zeros(native.aqlm_matmul_workspace_size(M, B, g, K, N, batch), dtype=torch.uint8, device=dev)
    xt = torch.from_numpy(x).to(dev)
    outs = []
    for _ in range(3):
        y1 = L.matmul(xt, w1, path=Path.TENSOR_CORE, workspace=ws, schedule=Schedule.STREAMK)
        y2 = L.matmul(y1, w2, path=Path.TENSOR_CORE, workspace=ws, schedule=Schedule.STREAMK)
        outs.append((y1, y2))
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, hex(detail)
    assert not ws[:CB].any().item()
    for y1, y2 in outs:
        ref1 = oracle.linear(x, ld1.codes, ld1.codebooks, ld1.scales, None, M, B, g)
        assert rel_err(y1.cpu().numpy(), ref1) <= TOL
        ref2 = oracle.linear(y1.cpu().numpy(), ld2.codes, ld2.codebooks, ld2.scales, None, M, B, g)
        assert rel_err(y2.cpu().numpy(), ref2) <= TOL


def test_streamk_one_workspace_serves_every_shape(dev):
    """One workspace, zero-filled once, shared by calls of different shapes (tile counts
    and batch tiles differ, so their partial slots cover different bytes): every
    result stays within the tolerance and the counters stay zero.  Partials of one
    shape must never land where another shape keeps its counters."""
    shapes = [(2, 8, 8, 11008, 4096, 256), (2, 8, 8, 256, 4096, 256), (2, 8, 8, 1000, 2048, 300),
              (1, 16, 8, 4096, 4096, 1), (2, 8, 8, 256, 4096, 256), (2, 8, 8, 11008, 4096, 256)]
    need = max(native.aqlm_matmul_workspace_size(M, B, g, K, N, b) for M, B, g, N, K, b in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    for i, (M, B, g, N, K, batch) in enumerate(shapes):
        ld = synth.make_layer(M, B, g, K, N, seed=150, layer=i)
        x = synth.make_x(batch, K, seed=151, layer=i)
        y = run_matmul(ld, x, dev, ws)
        rows = np.unique(np.concatenate([np.random.Generator(np.random.PCG64(i)).choice(N, 24, replace=False),
                                         [0, min(127, N - 1), N - 1]]))
        ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, M, B, g, rows=rows)
        assert rel_err(y[:, rows], ref) <= TOL, (i, M, B, g, N, K, batch)
        assert not ws[:CB].any().item(), i
    # the gradient kernels in the same workspace, after the layer calls
    for i, (M, B, g, K, N, batch) in enumerate([(2, 8, 8, 1024, 4096, 1024), (2, 8, 8, 4096, 4096, 64)]):
        gneed = native.aqlm_input_grad_workspace_size(M, B, g, K, N, batch)
        wsg = ws if gneed <= ws.numel() else torch.zeros(gneed, dtype=torch.uint8, device=dev)
        ld = synth.make_layer(M, B, g, K, N, seed=152, layer=i)
        dy = synth.make_x(batch, N, seed=153, layer=i)
        dx = L.input_grad(torch.from_numpy(dy).to(dev), L.AqlmWeights.from_numpy(ld, dev), workspace=wsg,
                          schedule=Schedule.STREAMK)
        torch.cuda.synchronize()
        cols = np.array([0, 1, 127, 128, 1000 % K, K - 1])
        ref = oracle.input_grad(dy, ld.codes, ld.codebooks, ld.scales, M, B, g, cols=cols)
        assert rel_err(dx.cpu().numpy()[:, cols], ref) <= TOL, ("grad", i)
        assert not wsg[:CB].any().item()


GRAD_CASES = [
    (2, 8, 8, 1024, 4096, 1024, True),   # 8 feature tiles x 4 batch tiles, pieces of ~14 stages
    (2, 8, 8, 1088, 1000, 300, True),    # ragged feature tile, partial last stage, 2 batch tiles
    (1, 8, 16, 2048, 4096, 256, False),
    (4, 8, 8, 1024, 2048, 64, False),
]


@pytest.mark.parametrize("M,B,g,K,N,batch,cut", GRAD_CASES)
def test_streamk_input_grad_matches_oracle(dev, M, B, g, K, N, batch, cut):
    need = native.aqlm_input_grad_workspace_size(M, B, g, K, N, batch)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    ld = synth.make_layer(M, B, g, K, N, seed=146, layer=K + batch)
    dy = synth.make_x(batch, N, seed=147, layer=K)
    w = L.AqlmWeights.from_numpy(ld, dev)
    dx = L.input_grad(torch.from_numpy(dy).to(dev), w, workspace=ws, schedule=Schedule.STREAMK)
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))
    dx = dx.cpu().numpy()
    assert np.isfinite(dx.astype(np.float32)).all()
    rng = np.random.Generator(np.random.PCG64(K))
    cols = np.unique(np.concatenate([rng.choice(K, 48, replace=False), [0, 127, 128, K - 1]]))
    ref = oracle.input_grad(dy, ld.codes, ld.codebooks, ld.scales, M, B, g, cols=cols)
    err = rel_err(dx[:, cols], ref)
    assert err <= TOL, f"grad {M}x{B} g{g} K={K} N={N} b={batch}: rel err {err:.3e}"
    cb = CB
    assert not ws[:cb].any().item()
    if cut:
        assert ws[cb:].any().item()


def test_device_status_clean_after_streamk(dev):
    st, detail = L.check_device_status()
    assert st == Status.OK, hex(detail)


def test_per_stream_workspaces_are_kept_apart_and_bounded(dev):
    """layer.matmul's default workspace is one per (device, stream): calls on 20
    streams at once (a layer whose call needs a workspace: the grouped-kernel route)
    give one result bit for bit, meet the oracle, and the cache keeps at most 16."""
    M, B, g, K, N = 2, 8, 8, 11008, 4096
    assert native.aqlm_matmul_workspace_size(M, B, g, K, N, 1) > 0
    ld = synth.make_layer(M, B, g, K, N, seed=170)
    x = synth.make_x(1, K, seed=171)
    w = L.AqlmWeights.from_numpy(ld, dev)
    xt = torch.from_numpy(x).to(dev)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(dev) for _ in range(20)]
    outs = [L.matmul(xt, w, stream=s) for s in streams]
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, hex(detail)
    first = outs[0].cpu().numpy()
    for y in outs[1:]:
        assert np.array_equal(y.cpu().numpy().view(np.uint16), first.view(np.uint16))
    rows = np.array([0, 1, 127, 128, 2047, N - 1])
    ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, M, B, g, rows=rows)
    assert rel_err(first[:, rows], ref) <= TOL
    assert len(L._workspaces) <= 16
