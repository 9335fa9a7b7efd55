"""aqlm_matmul_group (grouped lookup-table kernel + reduction) vs the CPU oracle,
through the C ABI.

Every layer of a group must meet the aqlm_matmul bar: max|y - y_ref| / max|y_ref|
<= 5e-3 against the oracle's fp64 reference of the decoded weights, no NaN/Inf;
bit for bit on integer-valued layers; run-to-run bitwise identical; correct when
the workspace is reused by back-to-back calls; and correct for groups that mix
grouped and non-grouped problems or exceed one launch's 32 layers.
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


def rel_err(y_gpu, y_ref):
    return float(np.abs(y_gpu.astype(np.float64) - y_ref).max() / max(np.abs(y_ref).max(), 1e-30))


def assert_close(y_gpu, y_ref, what):
    assert np.isfinite(y_gpu.astype(np.float32)).all(), f"{what}: non-finite output"
    err = rel_err(y_gpu, y_ref)
    assert err <= TOL, f"{what}: rel err {err:.3e} > {TOL}"


def build_group(specs, dev, seed):
    """specs: (M, B, g, K, N, batch, with_bias) per layer -> (LayerGroup, layer data, x, out)."""
    lds, xs, items = [], [], []
    for i, (M, B, g, K, N, batch, bias) in enumerate(specs):
        ld = synth.make_layer(M, B, g, K, N, seed=seed, layer=i, with_bias=bias)
        x = synth.make_x(batch, K, seed=seed, layer=i)
        w = L.AqlmWeights.from_numpy(ld, dev)
        xt = torch.from_numpy(x).to(dev)
        out = torch.full((batch, N), float("nan"), dtype=torch.float16, device=dev)
        lds.append(ld)
        xs.append(x)
        items.append((w, xt, out))
    return L.LayerGroup(items), lds, xs, [it[2] for it in items]


def check_status():
    torch.cuda.synchronize()
    st, detail = L.check_device_status()
    assert st == Status.OK, (st, hex(detail))


MIXED = [
    (2, 8, 8, 4096, 4096, 1, False),   # q_proj-sized
    (2, 8, 8, 11008, 200, 1, True),    # G = 1376: a half-filled last 64-group slice; ragged rows
    (2, 8, 8, 64, 1, 1, True),         # one slice, one row
    (2, 8, 8, 512, 1000, 1, False),    # ragged last 64-row tile
    (1, 16, 8, 1024, 300, 1, True),    # not grouped: tensor-core path
    (2, 8, 8, 1024, 130, 4, False),    # not grouped: batch 4
    (2, 8, 8, 1032, 77, 1, False),     # not grouped: K % 64 != 0
    (2, 8, 8, 2048, 129, 1, True),
]


def test_group_mixed_layers_match_oracle(dev):
    grp, lds, xs, outs = build_group(MIXED, dev, seed=40)
    assert grp.workspace_bytes == native.aqlm_group_workspace_size(grp.problems, grp.count) > 0
    grp.run()
    check_status()
    for (M, B, g, K, N, batch, _), ld, x, out in zip(MIXED, lds, xs, outs):
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        assert_close(out.cpu().numpy(), y_ref, f"group layer {M}x{B}g{g} K={K} N={N} b={batch}")


def test_group_is_deterministic_and_reuses_its_workspace(dev):
    """Two calls back to back on one stream, no synchronisation between them: the
    second call's partial-sum kernel must not overwrite the workspace before the
    first call's reduction has read it.  Different x per call, same weights."""
    specs = [(2, 8, 8, 4096, 1024, 1, False), (2, 8, 8, 11008, 512, 1, True), (2, 8, 8, 1024, 4096, 1, False)]
    grp, lds, xs, outs = build_group(specs, dev, seed=41)
    first = []
    for rep in range(3):
        for (w, xt, out), x in zip(grp._keep, xs):
            xt.copy_(torch.from_numpy(x if rep % 2 == 0 else -x))
        grp.run()
        first.append([o.clone() for o in outs])
    check_status()
    for rep, ys in enumerate(first):
        sign = 1 if rep % 2 == 0 else -1
        for (M, B, g, K, N, batch, _), ld, x, y in zip(specs, lds, xs, ys):
            y_ref = oracle.linear((sign * x.astype(np.float32)).astype(np.float16), ld.codes, ld.codebooks,
                                  ld.scales, ld.bias, M, B, g)
            assert_close(y.cpu().numpy(), y_ref, f"rep {rep} K={K} N={N}")
    for a, b in zip(first[0], first[2]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), "grouped runs differ"


def test_group_larger_than_one_launch(dev):
    """40 grouped layers: two launch pairs (32 + 8 layers) sharing one workspace."""
    specs = [(2, 8, 8, 64 * (1 + i % 5), 50 + 37 * i, 1, i % 3 == 0) for i in range(40)]
    grp, lds, xs, outs = build_group(specs, dev, seed=42)
    grp.run()
    check_status()
    for (M, B, g, K, N, batch, _), ld, x, out in zip(specs, lds, xs, outs):
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        assert_close(out.cpu().numpy(), y_ref, f"K={K} N={N}")


def test_group_integer_layers_bit_exact(dev):
    """Small-integer codebooks and x: every lookup, half2 pair sum and fp32 partial
    is an exact integer, so y must equal the oracle bit for bit."""
    rng = np.random.Generator(np.random.PCG64(43))
    items, refs = [], []
    for N, K in ((260, 512), (70, 1024), (129, 64)):
        cb = rng.integers(-2, 3, size=(2, 256, 8)).astype(np.float16)
        codes = rng.integers(0, 256, size=(N, K // 8, 2)).astype(np.uint8)
        sc = rng.choice(np.array([1.0, 2.0]), size=N).astype(np.float16)
        bias = rng.integers(-3, 4, size=N).astype(np.float16)
        x = rng.integers(-1, 2, size=(1, K)).astype(np.float16)
        y_ref = oracle.linear(x, codes, cb, sc, bias, 2, 8, 8)
        assert np.abs(y_ref).max() <= 2048 and np.array_equal(y_ref, np.round(y_ref))
        w = L.AqlmWeights.from_numpy(synth.LayerData(2, 8, 8, K, N, codes, cb, sc, bias), dev)
        items.append((w, torch.from_numpy(x).to(dev), torch.empty((1, N), dtype=torch.float16, device=dev)))
        refs.append(y_ref)
    L.LayerGroup(items).run()
    check_status()
    for (_, _, out), y_ref in zip(items, refs):
        y = out.cpu().numpy().astype(np.float64)
        assert np.array_equal(y, y_ref), int((y != y_ref).sum())


def test_group_zero_codebooks_give_bias(dev):
    ld = synth.make_layer(2, 8, 8, 1024, 300, seed=44, with_bias=True)
    ld.codebooks[:] = 0
    w = L.AqlmWeights.from_numpy(ld, dev)
    x = torch.from_numpy(synth.make_x(1, 1024, seed=44)).to(dev)
    out = torch.empty((1, 300), dtype=torch.float16, device=dev)
    L.LayerGroup([(w, x, out)]).run()
    check_status()
    assert np.array_equal(out.cpu().numpy()[0], ld.bias)


@pytest.mark.parametrize("wname", ["llama2_7b_layer_set_2x8g8", "mixtral_8x7b_experts_2x8g8"])
def test_group_published_layer_sets_sampled_rows(dev, wname):
    """A published layer set as one group call; the oracle computes sampled rows."""
    w = workloads.get(wname)
    items, lds, xs = [], [], []
    for li, lay in enumerate(w.layers):
        s = lay.scheme
        ld = synth.make_layer(s.M, s.B, s.g, lay.K, lay.N, seed=0, workload=w.index, layer=li)
        x = synth.make_x(1, lay.K, seed=0, workload=w.index, layer=li)
        items.append((L.AqlmWeights.from_numpy(ld, dev), torch.from_numpy(x).to(dev),
                      torch.empty((1, lay.N), dtype=torch.float16, device=dev)))
        lds.append(ld)
        xs.append(x)
    L.LayerGroup(items).run()
    check_status()
    rng = np.random.Generator(np.random.PCG64(45))
    for li, (lay, ld, x, item) in enumerate(zip(w.layers, lds, xs, items)):
        rows = np.unique(np.concatenate([rng.choice(lay.N, size=24, replace=False), [0, lay.N - 1, 63, 64]]))
        s = lay.scheme
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, s.M, s.B, s.g, rows=rows)
        y = item[2].cpu().numpy()
        assert np.isfinite(y.astype(np.float32)).all()
        assert_close(y[:, rows], y_ref, f"{wname}/{lay.name}")


@pytest.mark.parametrize("packed,pinned", [(True, True), (False, True), (True, False)])
def test_group_from_host_buffers(dev, packed, pinned):
    """aqlm_matmul_group_host: x copied from one packed host buffer, y copied back into
    one; with packed device buffers (one copy each way) and with separate ones (one
    copy per problem); page-locked and pageable host buffers."""
    # packed offsets stay 16-byte aligned: every batch * K and batch * N is a multiple of 8
    specs = [(2, 8, 8, 4096, 1024, 1, False), (2, 8, 8, 11008, 512, 1, True), (1, 16, 8, 1024, 304, 1, False),
             (2, 8, 8, 1024, 130, 4, False)]
    lds, xs = [], []
    for i, (M, B, g, K, N, batch, bias) in enumerate(specs):
        lds.append(synth.make_layer(M, B, g, K, N, seed=46, layer=i, with_bias=bias))
        xs.append(synth.make_x(batch, K, seed=46, layer=i))
    nx = sum(x.size for x in xs)
    ny = sum(batch * N for (_, _, _, _, N, batch, _) in specs)
    if packed:
        dxf = torch.empty(nx, dtype=torch.float16, device=dev)
        dyf = torch.full((ny,), float("nan"), dtype=torch.float16, device=dev)
        xo = np.cumsum([0] + [x.size for x in xs])
        yo = np.cumsum([0] + [batch * N for (_, _, _, _, N, batch, _) in specs])
        dx = [dxf[xo[i]:xo[i + 1]].view(xs[i].shape) for i in range(len(specs))]
        dy = [dyf[yo[i]:yo[i + 1]].view(specs[i][5], specs[i][4]) for i in range(len(specs))]
    else:
        dx = [torch.empty(x.shape, dtype=torch.float16, device=dev) for x in xs]
        dy = [torch.full((s[5], s[4]), float("nan"), dtype=torch.float16, device=dev) for s in specs]
    items = [(L.AqlmWeights.from_numpy(ld, dev), dx[i], dy[i]) for i, ld in enumerate(lds)]
    grp = L.LayerGroup(items)
    hx = torch.from_numpy(np.concatenate([x.reshape(-1) for x in xs]))
    hy = torch.full((ny,), float("nan"), dtype=torch.float16)
    if pinned:
        hx, hy = hx.pin_memory(), hy.pin_memory()
    s = torch.cuda.Stream(dev)
    for rep in range(3):  # back to back on one stream
        grp.run_host(hx, hy, stream=s)
    s.synchronize()
    check_status()
    off = 0
    for (M, B, g, K, N, batch, _), ld, x in zip(specs, lds, xs):
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        assert_close(hy[off:off + batch * N].numpy().reshape(batch, N), y_ref, f"host group K={K} N={N} b={batch}")
        off += batch * N


GENERIC = [
    (1, 8, 8, 4096, 1000, 1, False),    # 1 bit: 512-byte code rows, 4 slices
    (1, 8, 16, 4096, 520, 1, True),     # 0.5 bit: 256-byte rows, 2 slices
    (2, 8, 16, 2048, 300, 1, False),    # 1 bit
    (3, 8, 8, 1024, 257, 1, True),      # 3 bit: groups straddle the 128-byte slices
    (3, 8, 16, 2048, 130, 1, False),    # 1.5 bit
    (4, 8, 8, 1024, 64, 1, True),       # 4 bit: two K steps in the stacked table build
    (4, 8, 16, 4096, 200, 1, False),
    (2, 8, 8, 1024, 129, 1, True),      # the tuned 2x8 g8 path in the same launch
]


def test_group_generic_schemes_match_oracle(dev):
    """Every B = 8 scheme as grouped lookup-table layers, several in one launch (with
    layers of M g > 32 present the launch uses the four-K-step layout)."""
    grp, lds, xs, outs = build_group(GENERIC, dev, seed=47)
    grp.run()
    check_status()
    for (M, B, g, K, N, batch, _), ld, x, out in zip(GENERIC, lds, xs, outs):
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        assert_close(out.cpu().numpy(), y_ref, f"group {M}x{B}g{g} K={K} N={N}")


@pytest.mark.parametrize("M,g", [(1, 8), (1, 16), (2, 16), (3, 8), (3, 16), (4, 8), (4, 16)])
def test_group_generic_scheme_alone(dev, M, g):
    """One scheme per launch (the two-K-step layout for M g <= 32, else four), ragged
    rows."""
    spec = [(M, 8, g, 2048, 333, 1, True), (M, 8, g, 1024, 64, 1, False)]
    grp, lds, xs, outs = build_group(spec, dev, seed=48 + M + g)
    grp.run()
    check_status()
    for (M_, B, g_, K, N, batch, _), ld, x, out in zip(spec, lds, xs, outs):
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M_, B, g_)
        assert_close(out.cpu().numpy(), y_ref, f"{M_}x{B}g{g_} K={K} N={N}")


def test_group_two_step_layout_mixed_schemes(dev):
    """Schemes of one and two K steps (M g <= 32) sharing the two-K-step layout, the
    codebooks reloaded with a different step count at every layer change."""
    spec = [(4, 8, 8, 2048, 300, 1, True), (1, 8, 16, 4096, 130, 1, False), (3, 8, 8, 1024, 200, 1, False),
            (2, 8, 16, 2048, 64, 1, True), (2, 8, 8, 1024, 100, 1, False), (4, 8, 8, 1024, 70, 1, False)]
    grp, lds, xs, outs = build_group(spec, dev, seed=46)
    grp.run()
    check_status()
    for (M, B, g, K, N, batch, _), ld, x, out in zip(spec, lds, xs, outs):
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, B, g)
        assert_close(out.cpu().numpy(), y_ref, f"group {M}x{B}g{g} K={K} N={N}")


@pytest.mark.parametrize("M,g", [(1, 8), (3, 8), (4, 16)])
def test_group_generic_integer_layers_bit_exact(dev, M, g):
    """Small-integer codebooks and x: every table entry, half2 sum and fp32 partial is
    an exact integer, so y equals the oracle bit for bit."""
    rng = np.random.Generator(np.random.PCG64(49 + M + g))
    items, refs = [], []
    for N, K in ((260, 1024), (70, 2048)):
        cb = rng.integers(-2, 3, size=(M, 256, g)).astype(np.float16)
        codes = rng.integers(0, 256, size=(N, K // g, M)).astype(np.uint8)
        sc = rng.choice(np.array([1.0, 2.0]), size=N).astype(np.float16)
        bias = rng.integers(-3, 4, size=N).astype(np.float16)
        x = rng.integers(-1, 2, size=(1, K)).astype(np.float16)
        y_ref = oracle.linear(x, codes, cb, sc, bias, M, 8, g)
        assert np.abs(y_ref).max() <= 2048 and np.array_equal(y_ref, np.round(y_ref))
        w = L.AqlmWeights.from_numpy(synth.LayerData(M, 8, g, K, N, codes, cb, sc, bias), dev)
        items.append((w, torch.from_numpy(x).to(dev), torch.empty((1, N), dtype=torch.float16, device=dev)))
        refs.append(y_ref)
    L.LayerGroup(items).run()
    check_status()
    for (_, _, out), y_ref in zip(items, refs):
        y = out.cpu().numpy().astype(np.float64)
        assert np.array_equal(y, y_ref), int((y != y_ref).sum())


@pytest.mark.parametrize("scheme", ["4x8g8", "1x8g16", "3x8g8"])
def test_group_llama_set_other_schemes_sampled_rows(dev, scheme):
    """The Llama-2-7B layer set with another B = 8 scheme, one group call, sampled rows."""
    M, g = int(scheme[0]), int(scheme.split("g")[1])
    w = workloads.get("llama2_7b_layer_set_2x8g8")
    items, lds, xs = [], [], []
    for li, lay in enumerate(w.layers):
        ld = synth.make_layer(M, 8, g, lay.K, lay.N, seed=3, layer=li)
        x = synth.make_x(1, lay.K, seed=3, layer=li)
        items.append((L.AqlmWeights.from_numpy(ld, dev), torch.from_numpy(x).to(dev),
                      torch.empty((1, lay.N), dtype=torch.float16, device=dev)))
        lds.append(ld)
        xs.append(x)
    L.LayerGroup(items).run()
    check_status()
    rng = np.random.Generator(np.random.PCG64(50))
    for lay, ld, x, item in zip(w.layers, lds, xs, items):
        rows = np.unique(np.concatenate([rng.choice(lay.N, size=24, replace=False), [0, lay.N - 1]]))
        y_ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, None, M, 8, g, rows=rows)
        assert_close(item[2].cpu().numpy()[:, rows], y_ref, f"{scheme}/{lay.name}")


@pytest.mark.parametrize("M,g,K,N", [(3, 8, 4096, 11008), (2, 8, 11008, 4096), (4, 8, 14336, 4096),
                                     (4, 16, 11008, 4096)])
def test_single_layer_call_takes_the_grouped_kernel_where_it_pays(dev, M, g, K, N):
    """aqlm_matmul_ws at batch 1 (AUTO, with a workspace) runs the grouped lookup kernel
    on long-row B = 8 layers with at least 10 MiB of codes: its result equals a
    one-element group call's bit for bit (the same kernel and sum order), and the oracle
    within the layer tolerance.  Without a workspace the single-layer kernel runs."""
    assert native.aqlm_matmul_workspace_size(M, 8, g, K, N, 1) > 0
    ld = synth.make_layer(M, 8, g, K, N, seed=77, with_bias=True)
    x = synth.make_x(1, K, seed=78)
    w = L.AqlmWeights.from_numpy(ld, dev)
    xt = torch.from_numpy(x).to(dev)
    out = torch.empty((1, N), dtype=torch.float16, device=dev)
    L.LayerGroup([(w, xt, out)]).run()
    y_route = L.matmul(xt, w)             # the per-stream workspace: routed
    y_single = L.matmul(xt, w, workspace=False)
    check_status()
    assert np.array_equal(y_route.cpu().numpy().view(np.uint16), out.cpu().numpy().view(np.uint16))
    rows = np.unique(np.concatenate([np.random.Generator(np.random.PCG64(N)).choice(N, 48, replace=False),
                                     [0, 127, N - 1]]))
    ref = oracle.linear(x, ld.codes, ld.codebooks, ld.scales, ld.bias, M, 8, g, rows=rows)
    assert_close(y_route.cpu().numpy()[:, rows], ref, f"routed {M}x8 g{g} {N}x{K}")
    assert_close(y_single.cpu().numpy()[:, rows], ref, f"single-layer {M}x8 g{g} {N}x{K}")
