"""ctypes binding to libaqlm.so (include/aqlm.h), names as in the C ABI.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  There is no CPU or PyTorch fallback -- if libaqlm.so is missing or
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import enum
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(PKG, "libaqlm.so")

# Every exported symbol of include/aqlm.h.
EXPORTS = ("aqlm_matmul", "aqlm_matmul_path", "aqlm_dequantize", "aqlm_select_path",
           "aqlm_validate", "aqlm_status_string", "aqlm_check_device_status",
           "aqlm_last_cuda_error", "aqlm_abi_version", "aqlm_matmul_group",
           "aqlm_group_workspace_size", "aqlm_matmul_group_static", "aqlm_selftest_bounded_wait",
           "aqlm_input_grad", "aqlm_validate_input_grad", "aqlm_matmul_group_host",
           "aqlm_static_group_scratch_bytes", "aqlm_matmul_workspace_size", "aqlm_matmul_ws",
           "aqlm_input_grad_workspace_size", "aqlm_input_grad_ws")

ABI_VERSION = 8

# Site code aqlm_selftest_bounded_wait records in the device status word.
SITE_SELFTEST = 0x501

# Size of the library's static scratch buffer behind aqlm_matmul_group_static
# (AQLM_STATIC_GROUP_SCRATCH_BYTES; the library reports its own value through
# aqlm_static_group_scratch_bytes, which a CPU test compares with this one).
STATIC_GROUP_SCRATCH_BYTES = 16 << 20

# Counters at the start of a workspace that can carry the tensor-core kernel's
# stream-K schedule (AQLM_WORKSPACE_COUNTER_BYTES; a CPU test compares the two).
WORKSPACE_COUNTER_BYTES = 2560

# Grouped problems one launch pair of aqlm_matmul_group computes together.
MAX_GROUP_LAYERS = 32


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    UNSUPPORTED = 2
    MISALIGNED = 3
    CUDA = 4
    TIMEOUT = 5


class Schedule(enum.IntEnum):
    AUTO = 0
    TILES = 1
    STREAMK = 2


class Path(enum.IntEnum):
    AUTO = 0
    GEMV = 1
    GEMV_LUT = 2
    TENSOR_CORE = 3


class AqlmProblem(ctypes.Structure):
    """aqlm_problem: one layer of a group call (raw device pointers and sizes)."""
    _fields_ = [("x", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("codebooks", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("M", ctypes.c_int), ("B", ctypes.c_int), ("g", ctypes.c_int), ("K", ctypes.c_int),
                ("N", ctypes.c_int), ("batch", ctypes.c_int)]


class AqlmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = Status(status) if status in Status._value2member_map_ else status
        msg = status_string(status)
        if what:
            msg = f"{what}: {msg}"
        if status == Status.CUDA:
            msg += f" (cudaError {lib().aqlm_last_cuda_error()})"
        super().__init__(msg)


_lib = None
_lock = threading.Lock()

_vp = ctypes.c_void_p
_i = ctypes.c_int


def lib() -> ctypes.CDLL:
    """Load libaqlm.so (raises if it is missing: the product has no fallback)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIBRARY):
                    raise ImportError(
                        f"{LIBRARY} is missing: build it with `python -m weight_only_additive_b200.build`")
                L = ctypes.CDLL(LIBRARY)
                L.aqlm_matmul.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
                L.aqlm_matmul.restype = _i
                L.aqlm_matmul_path.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
                L.aqlm_matmul_path.restype = _i
                L.aqlm_dequantize.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
                L.aqlm_dequantize.restype = _i
                L.aqlm_select_path.argtypes = [_i] * 6
                L.aqlm_select_path.restype = _i
                L.aqlm_validate.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i]
                L.aqlm_validate.restype = _i
                L.aqlm_input_grad.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
                L.aqlm_input_grad.restype = _i
                L.aqlm_matmul_workspace_size.argtypes = [_i] * 6
                L.aqlm_matmul_workspace_size.restype = ctypes.c_size_t
                L.aqlm_matmul_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                                             ctypes.c_size_t, _vp]
                L.aqlm_matmul_ws.restype = _i
                L.aqlm_input_grad_workspace_size.argtypes = [_i] * 6
                L.aqlm_input_grad_workspace_size.restype = ctypes.c_size_t
                L.aqlm_input_grad_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp,
                                                 ctypes.c_size_t, _vp]
                L.aqlm_input_grad_ws.restype = _i
                L.aqlm_validate_input_grad.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i]
                L.aqlm_validate_input_grad.restype = _i
                L.aqlm_status_string.argtypes = [_i]
                L.aqlm_status_string.restype = ctypes.c_char_p
                L.aqlm_check_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32)]
                L.aqlm_check_device_status.restype = _i
                L.aqlm_last_cuda_error.restype = _i
                L.aqlm_abi_version.restype = _i
                L.aqlm_matmul_group.argtypes = [ctypes.POINTER(AqlmProblem), _i, _vp, ctypes.c_size_t, _vp]
                L.aqlm_matmul_group.restype = _i
                L.aqlm_group_workspace_size.argtypes = [ctypes.POINTER(AqlmProblem), _i]
                L.aqlm_group_workspace_size.restype = ctypes.c_size_t
                L.aqlm_matmul_group_static.argtypes = [ctypes.POINTER(AqlmProblem), _i, _vp]
                L.aqlm_matmul_group_host.argtypes = [ctypes.POINTER(AqlmProblem), _i, _vp, _vp, _vp,
                                                     ctypes.c_size_t, _vp]
                L.aqlm_matmul_group_host.restype = _i
                L.aqlm_matmul_group_static.restype = _i
                L.aqlm_static_group_scratch_bytes.argtypes = []
                L.aqlm_static_group_scratch_bytes.restype = ctypes.c_size_t
                L.aqlm_selftest_bounded_wait.argtypes = [ctypes.c_uint, _vp]
                L.aqlm_selftest_bounded_wait.restype = _i
                if L.aqlm_abi_version() != ABI_VERSION:
                    raise ImportError(f"libaqlm.so ABI {L.aqlm_abi_version()} != binding ABI {ABI_VERSION}")
                _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().aqlm_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != Status.OK:
        raise AqlmError(status, what)


# --------------------------------------------------------------------------
# raw-pointer entry points (same names and argument order as the C ABI)
# --------------------------------------------------------------------------
def aqlm_matmul(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, stream=None):
    _check(lib().aqlm_matmul(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, stream),
           "aqlm_matmul")


def aqlm_matmul_path(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, path, stream=None):
    _check(lib().aqlm_matmul_path(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch,
                                  int(path), stream), "aqlm_matmul_path")


def aqlm_matmul_workspace_size(M, B, g, K, N, batch) -> int:
    return lib().aqlm_matmul_workspace_size(M, B, g, K, N, batch)


def aqlm_matmul_ws(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, path, schedule, workspace,
                   workspace_bytes, stream=None):
    _check(lib().aqlm_matmul_ws(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, int(path),
                                int(schedule), workspace, workspace_bytes, stream), "aqlm_matmul_ws")


def aqlm_input_grad_workspace_size(M, B, g, K, N, batch) -> int:
    return lib().aqlm_input_grad_workspace_size(M, B, g, K, N, batch)


def aqlm_input_grad_ws(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch, schedule, workspace,
                       workspace_bytes, stream=None):
    _check(lib().aqlm_input_grad_ws(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch, int(schedule),
                                    workspace, workspace_bytes, stream), "aqlm_input_grad_ws")


def aqlm_dequantize(codes, codebooks, scales, W_out, M, B, g, K, N, stream=None):
    _check(lib().aqlm_dequantize(codes, codebooks, scales, W_out, M, B, g, K, N, stream),
           "aqlm_dequantize")


def aqlm_select_path(M, B, g, K, N, batch) -> int:
    return lib().aqlm_select_path(M, B, g, K, N, batch)


def aqlm_validate(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, path=Path.AUTO) -> int:
    return lib().aqlm_validate(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, int(path))


def aqlm_input_grad(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch, stream=None):
    _check(lib().aqlm_input_grad(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch, stream),
           "aqlm_input_grad")


def aqlm_validate_input_grad(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch) -> int:
    return lib().aqlm_validate_input_grad(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch)


def aqlm_check_device_status(stream=None):
    """Returns (status, detail) after synchronising `stream`."""
    detail = ctypes.c_uint32(0)
    st = lib().aqlm_check_device_status(stream, ctypes.byref(detail))
    return Status(st), detail.value


def problem_array(problems) -> ctypes.Array:
    """An aqlm_problem[] from AqlmProblem instances or 12-tuples in C argument order."""
    arr = (AqlmProblem * max(1, len(problems)))()
    for i, q in enumerate(problems):
        arr[i] = q if isinstance(q, AqlmProblem) else AqlmProblem(*q)
    return arr


def aqlm_matmul_group(problems, workspace, workspace_bytes, stream=None, count=None):
    """`problems`: a ctypes aqlm_problem array (see problem_array) or a sequence."""
    arr = problems if isinstance(problems, ctypes.Array) else problem_array(problems)
    n = len(problems) if count is None else count
    _check(lib().aqlm_matmul_group(arr, n, workspace, workspace_bytes, stream), "aqlm_matmul_group")


def aqlm_group_workspace_size(problems, count=None) -> int:
    arr = problems if isinstance(problems, ctypes.Array) else problem_array(problems)
    n = len(problems) if count is None else count
    return lib().aqlm_group_workspace_size(arr, n)


def aqlm_matmul_group_static(problems, stream=None, count=None):
    """Group call on the library's static scratch buffer (allocates nothing; calls
    that overlap in time race on that buffer)."""
    arr = problems if isinstance(problems, ctypes.Array) else problem_array(problems)
    n = len(problems) if count is None else count
    _check(lib().aqlm_matmul_group_static(arr, n, stream), "aqlm_matmul_group_static")


def aqlm_matmul_group_host(problems, x_host, y_host, workspace, workspace_bytes, stream=None, count=None):
    """Group call from packed host x to packed host y (pointers; pinned for async copies)."""
    arr = problems if isinstance(problems, ctypes.Array) else problem_array(problems)
    n = len(problems) if count is None else count
    _check(lib().aqlm_matmul_group_host(arr, n, x_host, y_host, workspace, workspace_bytes, stream),
           "aqlm_matmul_group_host")


def aqlm_selftest_bounded_wait(timeout_us: int, stream=None):
    """Launch the bounded-wait self-test kernel (see include/aqlm.h)."""
    _check(lib().aqlm_selftest_bounded_wait(int(timeout_us), stream), "aqlm_selftest_bounded_wait")
