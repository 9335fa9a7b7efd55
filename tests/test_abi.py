"""The C-ABI library on a machine without a GPU: it loads, exports every symbol
include/aqlm.h declares, and its host-side validation and path selection work
without touching the device (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from weight_only_additive_b200 import build, native
from weight_only_additive_b200.native import Path, Schedule, Status

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "aqlm.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return native.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(aqlm_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(native.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_abi_version_and_status_strings(lib):
    assert lib.aqlm_abi_version() == native.ABI_VERSION
    for st in Status:
        assert native.status_string(st).startswith("AQLM_")
    assert "unknown" in native.status_string(99)


A = 1 << 20  # a 16-byte aligned fake address: validation never dereferences it


SUPPORTED = [(m, 8, g) for m in (1, 2, 3, 4) for g in (8, 16)] + [(m, 16, g) for m in (1, 2) for g in (8, 16)]


# disjoint 16-byte aligned fake buffers (x, codes, codebooks, scales, bias, y), 64 MiB apart
D = tuple(A + i * (1 << 26) for i in range(6))


@pytest.mark.parametrize("M,B,g", SUPPORTED)
def test_supported_schemes_validate(lib, M, B, g):
    x, codes, cb, sc, bias, y = D
    assert native.aqlm_validate(x, codes, cb, sc, None, y, M, B, g, 4096, 4096, 1) == Status.OK
    assert native.aqlm_validate(x, codes, cb, sc, bias, y, M, B, g, 4096, 11008, 256) == Status.OK


def test_output_overlapping_an_input_is_rejected(lib):
    x, codes, cb, sc, bias, y = D
    K, N, batch = 4096, 4096, 4
    ok = (x, codes, cb, sc, bias, y, 2, 8, 8, K, N, batch)
    assert native.aqlm_validate(*ok) == Status.OK
    for i, name in enumerate(("x", "codes", "codebooks", "scales", "bias")):
        args = list(ok)
        args[5] = ok[i] + 16  # y starts inside that input
        assert native.aqlm_validate(*args) == Status.INVALID_ARG, name
    # y ending exactly where x starts touches nothing
    args = list(ok)
    args[5] = x - batch * N * 2
    assert native.aqlm_validate(*args) == Status.OK
    # an absent bias overlaps nothing
    args = list(ok)
    args[4], args[5] = None, bias
    assert native.aqlm_validate(*args) == Status.OK
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_matmul(x, codes, cb, sc, None, x, 2, 8, 8, K, N, batch)  # in place: rejected before launch
    assert e.value.status == Status.INVALID_ARG
    # the dequantised weight must not land on the codes, codebooks or scales either
    for target in (codes + 16, cb, sc - 16):
        with pytest.raises(native.AqlmError) as e:
            native.aqlm_dequantize(codes, cb, sc, target, 2, 8, 8, K, N)
        assert e.value.status == Status.INVALID_ARG


@pytest.mark.parametrize("args,want", [
    ((None, A, A, A, None, A, 1, 16, 8, 64, 64, 1), Status.INVALID_ARG),   # null x
    ((A, None, A, A, None, A, 1, 16, 8, 64, 64, 1), Status.INVALID_ARG),   # null codes
    ((A, A, A, A, None, None, 1, 16, 8, 64, 64, 1), Status.INVALID_ARG),   # null y
    ((A, A, A, A, None, A, 1, 16, 8, 60, 64, 1), Status.INVALID_ARG),      # K % g != 0
    ((A, A, A, A, None, A, 1, 16, 8, 64, 0, 1), Status.INVALID_ARG),       # N = 0
    ((A, A, A, A, None, A, 1, 16, 8, 64, 64, 0), Status.INVALID_ARG),      # batch = 0
    ((A, A, A, A, None, A, 1, 16, 8, 64, 64, 70000), Status.INVALID_ARG),  # batch too large
    ((A, A, A, A, None, A, 5, 8, 8, 64, 64, 1), Status.UNSUPPORTED),       # 5x8 not built
    ((A, A, A, A, None, A, 3, 16, 8, 64, 64, 1), Status.UNSUPPORTED),      # 3x16
    ((A, A, A, A, None, A, 1, 12, 8, 64, 64, 1), Status.UNSUPPORTED),      # B = 12
    ((A, A, A, A, None, A, 1, 8, 4, 64, 64, 1), Status.UNSUPPORTED),       # g = 4
    ((A + 8, A, A, A, None, A, 1, 16, 8, 64, 64, 1), Status.MISALIGNED),
    ((A, A + 2, A, A, None, A, 1, 16, 8, 64, 64, 1), Status.MISALIGNED),
    ((A, A, A, A, A + 4, A, 1, 16, 8, 64, 64, 1), Status.MISALIGNED),       # bias
])
def test_validation_errors_need_no_gpu(lib, args, want):
    assert native.aqlm_validate(*args) == want


def test_compute_entry_points_reject_bad_arguments_before_any_cuda_call(lib):
    # these return before touching the device, so they are safe without a GPU
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_matmul(None, A, A, A, None, A, 1, 16, 8, 64, 64, 1)
    assert e.value.status == Status.INVALID_ARG
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_dequantize(A, A, A, A + 2, 1, 16, 8, 64, 64)
    assert e.value.status == Status.MISALIGNED
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_matmul_path(A, A, A, A, None, A, 1, 16, 8, 64, 64, 16, Path.GEMV)
    assert e.value.status == Status.UNSUPPORTED  # the GEMV family stops at batch 8
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_matmul_path(A, A, A, A, None, A, 1, 16, 8, 64, 64, 1, Path.GEMV_LUT)
    assert e.value.status == Status.UNSUPPORTED  # the lookup table needs 256-entry codebooks
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_matmul_path(A, A, A, A, None, A, 3, 8, 8, 64, 64, 1, Path.GEMV_LUT)
    assert e.value.status == Status.UNSUPPORTED  # code rows of 24 bytes: not whole 16-byte units
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_matmul_path(A, A, A, A, None, A, 1, 8, 8, 8 * 8200, 64, 1, Path.GEMV_LUT)
    assert e.value.status == Status.UNSUPPORTED  # code rows above 16 x 4 x 128 bytes
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_matmul_path(A, A, A, A, None, A, 2, 8, 8, 64, 64, 2, Path.GEMV_LUT)
    assert e.value.status == Status.UNSUPPORTED  # batch 1 only


def test_path_selection(lib):
    sel = native.aqlm_select_path
    assert sel(2, 8, 8, 4096, 4096, 1) == Path.GEMV_LUT
    # K % 64 == 0 (and 16-byte code rows): the pipelined tensor-core kernel from batch 1
    assert sel(1, 16, 8, 4096, 4096, 1) == Path.TENSOR_CORE
    assert sel(1, 16, 16, 4096, 4096, 1) == Path.TENSOR_CORE
    for M, B, g in ((1, 16, 8), (2, 8, 8), (1, 16, 16)):
        for batch in (2, 3, 8, 9, 16, 64, 256, 1000):
            assert sel(M, B, g, 4096, 4096, batch) == Path.TENSOR_CORE
    # other K: the GEMV up to batch 8, the single-stage tensor-core kernel above
    assert sel(2, 8, 8, 4096 + 8, 4096, 1) == Path.GEMV
    assert sel(1, 16, 16, 4096 + 64, 4096, 1) == Path.GEMV  # g = 16 code rows of 520 bytes
    for M, B, g in ((1, 16, 8), (2, 8, 8)):
        for batch in (1, 4, 8):
            assert sel(M, B, g, 4096 + 8, 4096, batch) == Path.GEMV
        for batch in (9, 16, 256):
            assert sel(M, B, g, 4096 + 8, 4096, batch) == Path.TENSOR_CORE
    assert sel(5, 8, 8, 4096, 4096, 1) == -1
    # f2 schemes with B = 8: the lookup table at batch 1 (16-byte code rows of at most
    # 8 KB), the tensor-core kernel above
    for M in (1, 2, 3, 4):
        for g in (8, 16):
            assert sel(M, 8, g, 4096, 4096, 1) == Path.GEMV_LUT, (M, g)
            assert sel(M, 8, g, 4096, 4096, 2) == Path.TENSOR_CORE, (M, g)
    assert sel(1, 8, 8, 8 * 8192, 4096, 1) == Path.GEMV_LUT  # 8192-byte rows: the longest
    assert sel(1, 8, 8, 8 * 8208, 4096, 1) != Path.GEMV_LUT
    assert sel(3, 8, 16, 16 * 1000, 4096, 1) != Path.GEMV_LUT  # 3000-byte rows
    assert sel(4, 8, 16, 16 * 1000, 4096, 1) == Path.GEMV_LUT  # 4000-byte rows
    assert sel(1, 16, 8, 4095, 4096, 1) == -1


# ---------------------------------------------------------------------------
# group call: host-side sizing and validation (returns before any CUDA call)
# ---------------------------------------------------------------------------
def _prob(base, M=2, B=8, g=8, K=4096, N=4096, batch=1, bias=False):
    """Disjoint fake buffers for one problem, laid out from `base` (never dereferenced)."""
    step = 1 << 26
    return (base, base + step, base + 2 * step, base + 3 * step, base + 4 * step if bias else None,
            base + 5 * step, M, B, g, K, N, batch)


def _ws_bytes(K, N):
    return ((K // 8 + 63) // 64 * N * 4 + 255) // 256 * 256


def test_group_workspace_size(lib):
    # layout: the counters region, then the grouped partial sums; the 1x16 layer is
    # launched on its own and needs nothing
    P = [_prob(1 << 32), _prob(1 << 33, K=11008, N=200), _prob(1 << 34, M=1, B=16)]
    grouped = _ws_bytes(4096, 4096) + _ws_bytes(11008, 200)
    assert native.aqlm_group_workspace_size(P) == COUNTERS + grouped
    assert native.aqlm_group_workspace_size(P[:2]) == COUNTERS + grouped
    assert native.aqlm_group_workspace_size([]) == 0
    assert native.aqlm_group_workspace_size([_prob(1 << 32, M=1, B=16)]) == 0       # nothing grouped
    # batch 256: nothing grouped, the layers run the tile plans
    big = [_prob(1 << 32, batch=256, N=11008), _prob(1 << 33, batch=256, N=1000, K=2048)]
    assert native.aqlm_group_workspace_size(big) == 0
    assert native.aqlm_group_workspace_size([_prob(1 << 32, batch=2)]) == 0         # batch 2: not grouped
    assert native.aqlm_group_workspace_size([_prob(1 << 32, K=4104)]) == 0          # K % 64 != 0
    assert native.aqlm_group_workspace_size([_prob(1 << 32, K=4095)]) == 0          # invalid shape
    # 40 grouped problems: runs of 32 and 8; the workspace is the larger run
    R = native.MAX_GROUP_LAYERS
    many = [_prob((i + 1) << 32, K=64 * (i + 1), N=100) for i in range(R + 8)]
    run1 = sum(_ws_bytes(64 * (i + 1), 100) for i in range(R))
    run2 = sum(_ws_bytes(64 * (i + 1), 100) for i in range(R, R + 8))
    assert native.aqlm_group_workspace_size(many) == COUNTERS + max(run1, run2) == COUNTERS + run1


def test_group_validation_needs_no_gpu(lib):
    L_ = native.lib()
    P = [_prob(1 << 32), _prob(1 << 33, K=11008, N=200)]
    need = native.aqlm_group_workspace_size(P)
    arr = native.problem_array(P)
    assert L_.aqlm_matmul_group(arr, 0, None, 0, None) == Status.OK              # no-op
    assert L_.aqlm_matmul_group(arr, -1, None, 0, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_group(None, 2, None, 0, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_group(arr, 2, None, need, None) == Status.INVALID_ARG  # no workspace
    assert L_.aqlm_matmul_group(arr, 2, 1 << 40, need - 4, None) == Status.INVALID_ARG  # too small
    assert L_.aqlm_matmul_group(arr, 2, (1 << 40) + 16, need, None) == Status.MISALIGNED
    bad = native.problem_array([P[0], _prob(1 << 35, M=5)])
    assert L_.aqlm_matmul_group(bad, 2, 1 << 40, need, None) == Status.UNSUPPORTED
    bad = native.problem_array([P[0], _prob(1 << 35, N=0)])
    assert L_.aqlm_matmul_group(bad, 2, 1 << 40, need, None) == Status.INVALID_ARG
    # y of problem 1 overlaps x of problem 0 / y of problem 0: not independent
    q = list(_prob(1 << 33))
    q[5] = P[0][0] + 4096
    assert L_.aqlm_matmul_group(native.problem_array([P[0], tuple(q)]), 2, 1 << 40, need, None) == \
        Status.INVALID_ARG
    q[5] = P[0][5]
    assert L_.aqlm_matmul_group(native.problem_array([P[0], tuple(q)]), 2, 1 << 40, need, None) == \
        Status.INVALID_ARG


def test_group_static_validation_needs_no_gpu(lib):
    L_ = native.lib()
    assert L_.aqlm_matmul_group_static(native.problem_array([_prob(1 << 32)]), 0, None) == Status.OK
    assert L_.aqlm_matmul_group_static(None, 1, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_group_static(native.problem_array([_prob(1 << 32)]), -3, None) == Status.INVALID_ARG
    # 10 grouped 28672 x 8192 layers need 10 x 16 x 28672 x 4 bytes > 16 MiB
    big = [_prob((i + 1) << 34, K=8192, N=28672) for i in range(10)]
    assert native.aqlm_group_workspace_size(big) == COUNTERS + 10 * _ws_bytes(8192, 28672) > \
        native.STATIC_GROUP_SCRATCH_BYTES
    assert L_.aqlm_matmul_group_static(native.problem_array(big), 10, None) == Status.INVALID_ARG
    # the 24 Mixtral-8x7B expert linears of a layer (w1, w3 14336 x 4096, w2 4096 x 14336) fit
    mixtral = [_prob((i + 1) << 34, K=14336, N=4096) if i % 3 == 2 else _prob((i + 1) << 34, K=4096, N=14336)
               for i in range(24)]
    assert native.aqlm_group_workspace_size(mixtral) == \
        COUNTERS + 8 * (_ws_bytes(14336, 4096) + 2 * _ws_bytes(4096, 14336)) <= native.STATIC_GROUP_SCRATCH_BYTES
    bad = [_prob(1 << 32, M=5)]
    assert L_.aqlm_matmul_group_static(native.problem_array(bad), 1, None) == Status.UNSUPPORTED


def test_static_scratch_size_agrees_everywhere(lib):
    """The #define in include/aqlm.h, the library's own report and the binding's
    constant are one number."""
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "aqlm.h")).read()
    m = re.search(r"#define AQLM_STATIC_GROUP_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m, "AQLM_STATIC_GROUP_SCRATCH_BYTES not found in include/aqlm.h"
    from_header = int(m.group(1)) << int(m.group(2))
    assert from_header == native.lib().aqlm_static_group_scratch_bytes() == native.STATIC_GROUP_SCRATCH_BYTES


def test_selftest_rejects_bad_limits_without_a_gpu(lib):
    assert native.lib().aqlm_selftest_bounded_wait(0, None) == Status.INVALID_ARG
    assert native.lib().aqlm_selftest_bounded_wait(1000001, None) == Status.INVALID_ARG


@pytest.mark.parametrize("M,B,g", SUPPORTED)
def test_input_grad_supported_schemes_validate(lib, M, B, g):
    v = native.aqlm_validate_input_grad
    dx = 1 << 34  # far from every input range
    assert v(A, A, A, A, dx, M, B, g, 4096, 4096, 1) == Status.OK
    assert v(A, A, A, A, dx, M, B, g, 4096, 11008, 512) == Status.OK


@pytest.mark.parametrize("args,want", [
    ((None, A, A, A, 1 << 34, 2, 8, 8, 1024, 64, 1), Status.INVALID_ARG),      # null dy
    ((A, A, A, A, None, 2, 8, 8, 1024, 64, 1), Status.INVALID_ARG),            # null dx
    ((A, A, A, A, 1 << 34, 2, 8, 8, 1020, 64, 1), Status.INVALID_ARG),         # K % g != 0
    ((A, A, A, A, 1 << 34, 2, 8, 8, 1024, 64, 0), Status.INVALID_ARG),         # batch = 0
    ((A, A, A, A, 1 << 34, 5, 8, 8, 1024, 64, 1), Status.UNSUPPORTED),         # 5x8
    ((A, A, A, A, 1 << 34, 2, 8, 8, 1024, 60, 1), Status.UNSUPPORTED),         # N % 8 != 0
    ((A, A, A, A, 1 << 34, 1, 8, 16, 1088, 64, 1), Status.UNSUPPORTED),        # 68-byte code rows
    ((A, A, A, A + 8, 1 << 34, 2, 8, 8, 1024, 64, 1), Status.MISALIGNED),      # scales
    ((A, A, A, A, (1 << 34) + 2, 2, 8, 8, 1024, 64, 1), Status.MISALIGNED),    # dx
    ((A, A, 1 << 30, A, A + 64, 2, 8, 8, 1024, 64, 1), Status.INVALID_ARG),     # dx overlaps dy
    ((A, 1 << 30, A, A, (1 << 30) + 4096, 2, 8, 8, 1024, 64, 1), Status.INVALID_ARG),  # dx inside codes
])
def test_input_grad_validation_needs_no_gpu(lib, args, want):
    assert native.aqlm_validate_input_grad(*args) == want


def test_input_grad_rejects_bad_arguments_before_any_cuda_call(lib):
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_input_grad(A, A, A, A, 1 << 34, 2, 8, 8, 1024, 60, 1)
    assert e.value.status == Status.UNSUPPORTED
    with pytest.raises(native.AqlmError) as e:
        native.aqlm_input_grad(None, A, A, A, 1 << 34, 2, 8, 8, 1024, 64, 1)
    assert e.value.status == Status.INVALID_ARG


def test_group_host_rejects_missing_host_buffers_without_a_gpu(lib):
    L_ = native.lib()
    probs = native.problem_array([_prob(1 << 32)])
    assert L_.aqlm_matmul_group_host(probs, 1, None, A, A, 1 << 20, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_group_host(probs, 1, A, None, A, 1 << 20, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_group_host(probs, 0, None, None, None, 0, None) == Status.OK
    # every check of the group call comes before the first host-to-device copy: a
    # missing, short or misaligned workspace is reported as such, not as a failed copy
    need = native.aqlm_group_workspace_size(native.problem_array([_prob(1 << 32)]), 1)
    hx, hy = 1 << 45, 1 << 46
    assert L_.aqlm_matmul_group_host(probs, 1, hx, hy, None, 0, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_group_host(probs, 1, hx, hy, 1 << 40, need - 256, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_group_host(probs, 1, hx, hy, (1 << 40) + 16, need, None) == Status.MISALIGNED


def test_group_workspace_must_not_overlap_a_problem(lib):
    L_ = native.lib()
    P = [_prob(1 << 32), _prob(1 << 33, K=11008, N=200)]
    arr = native.problem_array(P)
    need = native.aqlm_group_workspace_size(arr, 2)
    for i, k in ((0, 0), (0, 5), (1, 1), (1, 3)):  # x / y of problem 0, codes / scales of problem 1
        assert L_.aqlm_matmul_group(arr, 2, P[i][k], need, None) == Status.INVALID_ARG, (i, k)
        assert L_.aqlm_matmul_group_host(arr, 2, 1 << 45, 1 << 46, P[i][k], need, None) == Status.INVALID_ARG


@pytest.mark.parametrize("M,g,K", [(1, 8, 4096), (3, 8, 1024), (4, 16, 4096), (1, 16, 4096)])
def test_group_workspace_size_generic_schemes(lib, M, g, K):
    """Grouped B = 8 layers of any scheme: one fp32 partial per row and 128-code-byte
    slice, rounded up to 256 bytes."""
    N = 300
    probs = native.problem_array([_prob(1 << 32, M=M, B=8, g=g, K=K, N=N)])
    slices = (K // g * M + 127) // 128
    assert native.aqlm_group_workspace_size(probs, 1) == COUNTERS + (slices * N * 4 + 255) // 256 * 256


# ---------------------------------------------------------------------------
# workspace of the tensor-core kernel's stream-K schedule (pure host logic)
# ---------------------------------------------------------------------------
COUNTERS = 2560  # AQLM_WORKSPACE_COUNTER_BYTES: a uint32 per (CTA, lane quadrant), 160 CTAs


def _streamk_parts(units, BN):
    """Stream-K partial slots: 2 of 128 x BN fp32 per CTA, at most 160 CTAs."""
    return 2 * min(units, 160) * 128 * BN * 4


def _streamk_bytes(tiles, units, BN):
    """The size the header documents: the fixed counters, then the partial slots
    (the tile count does not enter)."""
    return COUNTERS + _streamk_parts(units, BN)


def test_workspace_counter_bytes_agree_everywhere(lib):
    text = open(HEADER).read()
    m = re.search(r"#define AQLM_WORKSPACE_COUNTER_BYTES (\d+)u", text)
    assert m and int(m.group(1)) == COUNTERS == native.WORKSPACE_COUNTER_BYTES == 160 * 4 * 4


def test_matmul_workspace_size(lib):
    # 2x8 g8 11008 x 4096 at batch 256: 86 row tiles, units of 4 stages (one code tile)
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 4096, 11008, 256) == _streamk_bytes(86, 86 * 16, 256)
    # batch 300: two batch tiles of 256
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 4096, 1000, 300) == _streamk_bytes(16, 16 * 16, 256)
    # 1x16 g8 keeps its A stages in shared memory at every batch: batch 1, tile 16
    assert native.aqlm_matmul_workspace_size(1, 16, 8, 4096, 4096, 1) == _streamk_bytes(32, 32 * 16, 16)
    # a few units only: as many CTAs as units
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 256, 128, 200) == _streamk_bytes(1, 1, 208)
    # A in tensor memory (batch tile <= 128), K not a whole number of code tiles, or
    # no pipelined kernel: no workspace
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 4096, 11008, 16) == 0
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 4096 + 64, 11008, 256) == 0
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 2064, 300, 256) == 0
    # invalid arguments
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 4100, 11008, 256) == 0
    assert native.aqlm_matmul_workspace_size(5, 8, 8, 4096, 11008, 256) == 0


def test_matmul_workspace_size_for_the_grouped_route(lib):
    """Batch-1 B = 8 layers with >= 10 MiB of codes in code rows of >= 1536 bytes get
    the counters plus the grouped kernel's partial sums (one fp32 per row and 128 code
    bytes); the others, at batch 1 with A in tensor memory, none."""
    def grouped(M, g, K, N):
        slices = (K // g * M + 127) // 128
        return COUNTERS + (slices * N * 4 + 255) // 256 * 256
    assert native.aqlm_matmul_workspace_size(3, 8, 8, 4096, 11008, 1) == grouped(3, 8, 4096, 11008)
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 11008, 4096, 1) == grouped(2, 8, 11008, 4096)
    assert native.aqlm_matmul_workspace_size(4, 8, 16, 11008, 4096, 1) == grouped(4, 16, 11008, 4096)
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 4096, 11008, 1) == 0   # 1024-byte rows
    assert native.aqlm_matmul_workspace_size(4, 8, 8, 4096, 4096, 1) == 0    # 8 MiB of codes
    assert native.aqlm_matmul_workspace_size(3, 8, 16, 11008, 4096, 1) == 0  # 8.1 MiB of codes
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 11008, 4096, 2) == 0   # batch 2


def test_input_grad_workspace_size(lib):
    # Mixtral expert down-projection at batch 1024: 32 feature tiles x 4 batch tiles,
    # 224 single-stage units each
    assert native.aqlm_input_grad_workspace_size(2, 8, 8, 4096, 14336, 1024) == _streamk_bytes(128, 128 * 224, 256)
    assert native.aqlm_input_grad_workspace_size(2, 8, 8, 1088, 1000, 16) == _streamk_bytes(9, 9 * 16, 16)
    # B = 16 gradient kernels have no stream-K schedule
    assert native.aqlm_input_grad_workspace_size(1, 16, 8, 4096, 4096, 1024) == 0
    assert native.aqlm_input_grad_workspace_size(2, 8, 8, 4100, 4096, 1024) == 0


def test_workspace_validation_needs_no_gpu(lib):
    ws_need = native.aqlm_matmul_workspace_size(2, 8, 8, 4096, 11008, 256)
    x, y, W = 1 << 32, 1 << 34, 1 << 40  # disjoint fake buffers, never dereferenced
    args = (x, x + (1 << 30), x + (1 << 31), x + (1 << 31) + (1 << 20), None, y, 2, 8, 8, 4096, 11008, 256,
            Path.TENSOR_CORE, Schedule.AUTO)
    L_ = native.lib()
    # misaligned, too small, bytes without a pointer, overlapping y
    assert L_.aqlm_matmul_ws(*args, W + 128, ws_need, None) == Status.MISALIGNED
    assert L_.aqlm_matmul_ws(*args, W, ws_need - 256, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_ws(*args, None, 256, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_ws(*args, y - 256, ws_need, None) == Status.INVALID_ARG
    # argument errors come first, as for aqlm_matmul_path
    bad = (None,) + args[1:]
    assert L_.aqlm_matmul_ws(*bad, W, ws_need, None) == Status.INVALID_ARG
    # schedules: unknown; stream-K without a workspace, on a shape without one, on
    # another kernel family
    assert L_.aqlm_matmul_ws(*args[:-1], 7, W, ws_need, None) == Status.INVALID_ARG
    assert L_.aqlm_matmul_ws(*args[:-1], Schedule.STREAMK, None, 0, None) == Status.INVALID_ARG
    small = args[:6] + (2, 8, 8, 4096, 11008, 16, Path.TENSOR_CORE, Schedule.STREAMK)
    assert native.aqlm_matmul_workspace_size(2, 8, 8, 4096, 11008, 16) == 0
    assert L_.aqlm_matmul_ws(*small, W, 1 << 20, None) == Status.UNSUPPORTED
    gemv = args[:6] + (1, 16, 8, 4096, 4096, 1, Path.GEMV, Schedule.STREAMK)
    assert L_.aqlm_matmul_ws(*gemv, W, 1 << 24, None) == Status.UNSUPPORTED
    # a shape whose workspace serves only the grouped lookup route: stream-K stays
    # unsupported there, before any CUDA call
    routed = args[:6] + (2, 8, 8, 14336, 4096, 1, Path.AUTO, Schedule.STREAMK)
    rneed = native.aqlm_matmul_workspace_size(2, 8, 8, 14336, 4096, 1)
    assert rneed > 0
    assert L_.aqlm_matmul_ws(*routed, W, rneed, None) == Status.UNSUPPORTED
    gneed = native.aqlm_input_grad_workspace_size(2, 8, 8, 4096, 14336, 1024)
    gargs = (x, x + (1 << 31), x + (1 << 31) + (1 << 28), x + (1 << 31) + (1 << 29), y, 2, 8, 8, 4096, 14336, 1024,
             Schedule.AUTO)
    assert L_.aqlm_input_grad_ws(*gargs, W + 16, gneed, None) == Status.MISALIGNED
    assert L_.aqlm_input_grad_ws(*gargs, W, gneed - 1, None) == Status.INVALID_ARG
    assert L_.aqlm_input_grad_ws(*gargs, x, gneed, None) == Status.INVALID_ARG  # overlaps dy
    assert L_.aqlm_input_grad_ws(*gargs[:-1], Schedule.STREAMK, None, 0, None) == Status.INVALID_ARG
    g16 = gargs[:5] + (1, 16, 8, 4096, 4096, 1024, Schedule.STREAMK)  # B = 16 gradient: no stream-K
    assert L_.aqlm_input_grad_ws(*g16, W, 1 << 24, None) == Status.UNSUPPORTED


def _header_enum(prefix):
    """{NAME: value} of the enumerators of include/aqlm.h whose names start with prefix."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return {m.group(1)[len(prefix):]: int(m.group(2))
            for m in re.finditer(r"\b(" + prefix + r"[A-Z_]+)\s*=\s*(\d+)", text)}


def test_binding_enums_agree_with_the_header():
    """The ctypes enums carry the header's values (status codes, paths, schedules)."""
    assert _header_enum("AQLM_ERR_") == {s.name: int(s) for s in Status if s.name != "OK"}
    assert _header_enum("AQLM_PATH_") == {p.name: int(p) for p in Path}
    assert _header_enum("AQLM_SCHEDULE_") == {s.name: int(s) for s in Schedule}
