"""PyTorch-facing wrappers over the C ABI: pass `data_ptr()`s and the current
CUDA stream to libaqlm.so.  Torch provides device memory and streams only; the
arithmetic happens in the library's kernels.
"""
from __future__ import annotations

from collections import OrderedDict
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import native
from .native import Path, Schedule


def _stream_handle(stream: Optional[torch.cuda.Stream], device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


# Workspaces of aqlm_matmul_ws / aqlm_input_grad_ws, one per (device, stream): calls on
# one stream may share one (the library leaves its counters zero), calls on different
# streams must not.  The 16 most recently used are kept; a dropped one was allocated on
# its own stream, so the caching allocator reuses its memory only in that stream's order.
_workspaces: "OrderedDict" = OrderedDict()
_MAX_WORKSPACES = 16


def stream_workspace(nbytes: int, device, stream: Optional[torch.cuda.Stream] = None) -> Optional[torch.Tensor]:
    """A zero-filled uint8 workspace of at least `nbytes` for calls on `stream` (the
    device's current stream if None), kept and grown per (device, stream); None for 0."""
    if nbytes <= 0:
        return None
    dev = torch.device(device)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    key = (dev.index, s.cuda_stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        # filled on the stream that uses it, so the fill is ordered before every call
        with torch.cuda.stream(s):
            ws = torch.zeros((nbytes,), dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    _workspaces.move_to_end(key)
    while len(_workspaces) > _MAX_WORKSPACES:
        _workspaces.popitem(last=False)
    return ws


def _resolve_workspace(workspace, nbytes: int, dev, stream):
    """(pointer, bytes) for the C call: the caller's tensor, none (False), or the
    per-stream workspace (None)."""
    if workspace is False or nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = stream_workspace(nbytes, dev, stream)
    _check_tensor(workspace, "workspace", torch.uint8, dev)
    return workspace.data_ptr(), workspace.numel()


@dataclass
class AqlmWeights:
    """One AQLM linear layer resident on a CUDA device."""
    codes: torch.Tensor       # [N, K/g, M] uint8 (B=8) or int16 holding uint16 bits (B=16)
    codebooks: torch.Tensor   # [M, 2^B, g] float16
    scales: torch.Tensor      # [N] float16
    bias: Optional[torch.Tensor]
    M: int
    B: int
    g: int

    def __post_init__(self):
        # the kernels read exactly the sizes (M, B, g, K, N) imply: check them once here
        code_dtypes = (torch.uint8,) if self.B <= 8 else (torch.int16, torch.uint16)
        if self.codes.dtype not in code_dtypes:
            raise TypeError(f"codes must be {' or '.join(map(str, code_dtypes))} for B={self.B}, "
                            f"got {self.codes.dtype}")
        if self.codes.dim() != 3 or self.codes.shape[2] != self.M or not self.codes.is_contiguous():
            raise ValueError(f"codes must be a contiguous [N, K/g, {self.M}] tensor, got shape {tuple(self.codes.shape)}")
        dev = self.codes.device
        _check_tensor(self.codebooks, "codebooks", torch.float16, dev, (self.M, 1 << self.B, self.g))
        _check_tensor(self.scales, "scales", torch.float16, dev, (self.N,))
        if self.bias is not None:
            _check_tensor(self.bias, "bias", torch.float16, dev, (self.N,))

    @property
    def N(self) -> int:
        return self.codes.shape[0]

    @property
    def K(self) -> int:
        return self.codes.shape[1] * self.g

    @classmethod
    def from_numpy(cls, layer, device="cuda") -> "AqlmWeights":
        """From a synth.LayerData (numpy host arrays)."""
        # 16-bit codes travel as int16 (same bytes): torch has few uint16 kernels.
        raw = layer.codes.view(np.int16) if layer.codes.dtype == np.uint16 else layer.codes
        codes = torch.from_numpy(np.ascontiguousarray(raw))
        return cls(codes=codes.to(device), codebooks=torch.from_numpy(layer.codebooks).to(device),
                   scales=torch.from_numpy(layer.scales).to(device),
                   bias=None if layer.bias is None else torch.from_numpy(layer.bias).to(device),
                   M=layer.M, B=layer.B, g=layer.g)


def _check_tensor(t: torch.Tensor, name: str, dtype, device, shape=None):
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        # the kernels write exactly this many values: a smaller buffer would be overrun
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def matmul(x: torch.Tensor, w: AqlmWeights, out: Optional[torch.Tensor] = None,
           path: Path = Path.AUTO, stream: Optional[torch.cuda.Stream] = None, workspace=None,
           schedule: Schedule = Schedule.AUTO) -> torch.Tensor:
    """y = x . W^T . diag(s) + bias for x [batch, K] fp16 on the weights' device.

    workspace: None for this stream's cached workspace (stream_workspace), False for
    none, or a zero-filled uint8 tensor of at least aqlm_matmul_workspace_size bytes.
    schedule: the tensor-core kernel's work schedule (aqlm_schedule)."""
    dev = w.codes.device
    if dev.type != "cuda":
        raise ValueError("AQLM weights must live on a CUDA device")
    _check_tensor(x, "x", torch.float16, dev)
    if x.dim() != 2:
        raise ValueError(f"x must be [batch, K], got shape {tuple(x.shape)}")
    batch, K = x.shape
    if K != w.K:
        raise ValueError(f"x has K={K}, weights have K={w.K}")
    if out is None:
        out = torch.empty((batch, w.N), dtype=torch.float16, device=dev)
    _check_tensor(out, "out", torch.float16, dev, (batch, w.N))
    ws, ws_bytes = _resolve_workspace(workspace, native.aqlm_matmul_workspace_size(w.M, w.B, w.g, K, w.N, batch),
                                      dev, stream)
    native.aqlm_matmul_ws(x.data_ptr(), w.codes.data_ptr(), w.codebooks.data_ptr(),
                          w.scales.data_ptr(), _ptr(w.bias), out.data_ptr(),
                          w.M, w.B, w.g, K, w.N, batch, path, schedule, ws, ws_bytes, _stream_handle(stream, dev))
    return out


def input_grad(dy: torch.Tensor, w: AqlmWeights, out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None, workspace=None,
               schedule: Schedule = Schedule.AUTO) -> torch.Tensor:
    """dx = dy . diag(s) . W [batch, K] for dy [batch, N] fp16: the gradient of
    matmul() with respect to its input (the weights are fixed).  workspace and
    schedule as for matmul (aqlm_input_grad_workspace_size bytes)."""
    dev = w.codes.device
    if dev.type != "cuda":
        raise ValueError("AQLM weights must live on a CUDA device")
    _check_tensor(dy, "dy", torch.float16, dev)
    if dy.dim() != 2:
        raise ValueError(f"dy must be [batch, N], got shape {tuple(dy.shape)}")
    batch, N = dy.shape
    if N != w.N:
        raise ValueError(f"dy has N={N}, weights have N={w.N}")
    if out is None:
        out = torch.empty((batch, w.K), dtype=torch.float16, device=dev)
    _check_tensor(out, "out", torch.float16, dev, (batch, w.K))
    ws, ws_bytes = _resolve_workspace(
        workspace, native.aqlm_input_grad_workspace_size(w.M, w.B, w.g, w.K, N, batch), dev, stream)
    native.aqlm_input_grad_ws(dy.data_ptr(), w.codes.data_ptr(), w.codebooks.data_ptr(), w.scales.data_ptr(),
                              out.data_ptr(), w.M, w.B, w.g, w.K, N, batch, schedule, ws, ws_bytes,
                              _stream_handle(stream, dev))
    return out


def dequantize(w: AqlmWeights, out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """W [N, K] fp16, bit-exact decode of the AQLM weights."""
    dev = w.codes.device
    if out is None:
        out = torch.empty((w.N, w.K), dtype=torch.float16, device=dev)
    _check_tensor(out, "out", torch.float16, dev, (w.N, w.K))
    native.aqlm_dequantize(w.codes.data_ptr(), w.codebooks.data_ptr(), w.scales.data_ptr(),
                           out.data_ptr(), w.M, w.B, w.g, w.K, w.N, _stream_handle(stream, dev))
    return out


def check_device_status(stream: Optional[torch.cuda.Stream] = None, device=None):
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return native.aqlm_check_device_status(_stream_handle(stream, dev))


class LayerGroup:
    """A set of independent layers computed by one aqlm_matmul_group call.

    `items` is a sequence of (weights, x, out) with x [batch, K] and out [batch, N]
    fp16 tensors on the weights' device.  The problem table and the workspace are
    built once; run() enqueues the whole set on a stream (and may be captured in
    a CUDA graph).
    """

    def __init__(self, items, device=None):
        if not items:
            raise ValueError("a layer group needs at least one layer")
        dev = items[0][0].codes.device if device is None else torch.device(device)
        probs = []
        self._keep = []
        for w, x, out in items:
            _check_tensor(x, "x", torch.float16, dev)
            _check_tensor(out, "out", torch.float16, dev)
            batch, K = x.shape
            if K != w.K or tuple(out.shape) != (batch, w.N):
                raise ValueError(f"shapes: x {tuple(x.shape)}, out {tuple(out.shape)}, weights N={w.N} K={w.K}")
            probs.append((x.data_ptr(), w.codes.data_ptr(), w.codebooks.data_ptr(), w.scales.data_ptr(),
                          _ptr(w.bias), out.data_ptr(), w.M, w.B, w.g, K, w.N, batch))
            self._keep.append((w, x, out))
        self.device = dev
        self.problems = native.problem_array(probs)
        self.count = len(probs)
        self.workspace_bytes = native.aqlm_group_workspace_size(self.problems, self.count)
        # 256-byte aligned: torch's caching allocator hands out 512-byte aligned blocks;
        # zero-filled once, so the buffer could also serve aqlm_matmul_ws calls
        self.workspace = torch.zeros((max(self.workspace_bytes, 1),), dtype=torch.uint8, device=dev)

    def run(self, stream: Optional[torch.cuda.Stream] = None):
        native.aqlm_matmul_group(self.problems, self.workspace.data_ptr(), self.workspace_bytes,
                                 _stream_handle(stream, self.device), count=self.count)

    def run_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream: Optional[torch.cuda.Stream] = None):
        """One step from host activations to host outputs: x_host holds every layer's x
        one after another (fp16, CPU, ideally pinned), y_host receives every y; the
        copies and the group run on `stream` (aqlm_matmul_group_host).  Synchronise the
        stream before reading y_host."""
        nx = sum(int(x.numel()) for _, x, _ in self._keep)
        ny = sum(int(o.numel()) for _, _, o in self._keep)
        for t, n, name in ((x_host, nx, "x_host"), (y_host, ny, "y_host")):
            if t.device.type != "cpu" or t.dtype != torch.float16 or not t.is_contiguous() or t.numel() != n:
                raise ValueError(f"{name} must be a contiguous CPU fp16 tensor of {n} values")
        native.aqlm_matmul_group_host(self.problems, x_host.data_ptr(), y_host.data_ptr(), self.workspace.data_ptr(),
                                      self.workspace_bytes, _stream_handle(stream, self.device), count=self.count)
