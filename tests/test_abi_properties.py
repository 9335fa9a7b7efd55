"""Property test of the C ABI's argument checks (no GPU): aqlm_validate against a
plain restatement of the rules include/aqlm.h gives, on random shapes, paths and
pointer layouts (buffers share address slots often enough that outputs overlap
inputs, and offsets break alignment).  Checks the order of the errors too: null
pointers and shapes first, then alignment, then the path, then overlaps."""
import hypothesis.strategies as st
from hypothesis import HealthCheck, event, given, settings

from weight_only_additive_b200 import build, native
from weight_only_additive_b200.native import Path, Status

SUPPORTED = {(m, 8, g) for m in (1, 2, 3, 4) for g in (8, 16)} | {(m, 16, g) for m in (1, 2) for g in (8, 16)}
SLOT = 1 << 36  # slots far apart: buffers in different slots never overlap


def model(ptrs, M, B, g, K, N, batch, path):
    """(expected status of aqlm_validate, the rule that decides it), written from the
    header's contract."""
    x, codes, cb, sc, bias, y = ptrs
    if not all(p for p in (x, codes, cb, sc, y)):
        return Status.INVALID_ARG, "null"
    if min(M, B, g, K, N, batch) < 1 or K % g or batch > 65535:
        return Status.INVALID_ARG, "shape"
    if (M, B, g) not in SUPPORTED:
        return Status.UNSUPPORTED, "scheme"
    if any(p % 16 for p in (x, codes, cb, sc, y)) or (bias and bias % 16):
        return Status.MISALIGNED, "alignment"
    if path != Path.AUTO:
        if path not in (Path.GEMV, Path.GEMV_LUT, Path.TENSOR_CORE):
            return Status.INVALID_ARG, "path value"
        row_bytes = K // g * M
        ok = {Path.GEMV: batch <= 8,
              Path.GEMV_LUT: B == 8 and batch == 1 and row_bytes % 16 == 0 and row_bytes <= 8192,
              Path.TENSOR_CORE: True}[path]
        if not ok:
            return Status.UNSUPPORTED, "path"
    sizes = (2 * batch * K, N * (K // g) * M * (1 if B <= 8 else 2), M * (1 << B) * g * 2, 2 * N,
             2 * N if bias else 0)
    y0, y1 = y, y + 2 * batch * N
    for p, n in zip((x, codes, cb, sc, bias), sizes):
        if p and n and y0 < p + n and p < y1:
            return Status.INVALID_ARG, "overlap"
    return Status.OK, "ok"


@st.composite
def layouts(draw):
    """Six buffers (x, codes, codebooks, scales, bias, y), each in its own address slot
    by default; sometimes one shares another's slot (an overlap, or a disjoint
    neighbour), sits at an offset that breaks 16-byte alignment, or is NULL."""
    ptrs = []
    for i in range(6):
        # y (i = 5) shares a slot more often: an overlap needs it in an input's slot
        kind = draw(st.sampled_from(["own"] * (4 if i == 5 else 14) + ["shared"] * 3 + ["null"]))
        if kind == "null":
            ptrs.append(0)
            continue
        slot = i + 1 if kind == "own" else draw(st.integers(1, 6))
        off = draw(st.sampled_from([0] * 10 + [2, 8, 16, 4096, 1 << 20, 1 << 26]))
        ptrs.append(slot * SLOT + off)
    return tuple(ptrs)


SCHEMES = sorted(SUPPORTED) + [(5, 8, 8), (3, 16, 8), (1, 12, 8), (1, 8, 4), (0, 8, 8)]


@st.composite
def shapes(draw):
    """Mostly valid shapes of every supported scheme, some with K not a whole number of
    groups, an unsupported scheme, or a size out of range."""
    M, B, g = draw(st.sampled_from(SCHEMES))
    K = draw(st.sampled_from([1, 2, 7, 64, 512, 513, 1792, 8192, 8208])) * max(g, 1)
    K += draw(st.sampled_from([0] * 8 + [1, -1]))
    N = draw(st.sampled_from([1, 3, 64, 4096, 14336, 14336, 0]))
    batch = draw(st.sampled_from([1, 1, 1, 2, 8, 9, 16, 256, 65535, 65536, 0]))
    return M, B, g, K, N, batch


@settings(max_examples=4000, deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))
@given(ptrs=layouts(), shape=shapes(), path=st.sampled_from([0, 0, 0, 1, 2, 3, -1, 4]))
def test_validate_matches_the_contract(ptrs, shape, path):
    build.build()
    M, B, g, K, N, batch = shape
    want, rule = model(ptrs, M, B, g, K, N, batch, path)
    event(rule)
    got = native.aqlm_validate(*ptrs, M, B, g, K, N, batch, path)
    assert got == want, (ptrs, M, B, g, K, N, batch, path)
