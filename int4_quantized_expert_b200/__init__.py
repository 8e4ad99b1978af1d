"""Python binding of libmoe_int4: an int4 / FP8 mixture-of-experts FFN layer
for NVIDIA B200 (sm_100a).

Every function here only marshals arguments into the C ABI declared in
``include/moe_int4.h``; all arithmetic runs in the library's CUDA kernels.
PyTorch is used for device memory, dtypes and the current stream.  There is no
CPU fallback: without the built library (``python -m
int4_quantized_expert_b200.build``) or without a CUDA device the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = [
    "LIB_PATH", "lib", "MoEError", "Status", "LayerDesc", "quantize_int4", "quantize_fp8_rows", "rmsnorm",
    "route", "MoELayer", "DenseDesc", "DenseLayer", "FMT_INT4", "FMT_FP8", "PATH_AUTO", "PATH_DECODE",
    "PATH_PREFILL", "noalloc_device_status", "set_wait_limit",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libmoe_int4.so")

FMT_INT4, FMT_FP8 = 0, 1
PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2
DTYPE_BF16, DTYPE_FP32 = 0, 1


class Status:
    OK, INVALID_ARG, UNSUPPORTED_SHAPE, WORKSPACE_TOO_SMALL, CUDA, TIMEOUT = range(6)


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (fn, _status_string(status), status))


class LayerDesc(ctypes.Structure):
    """Mirror of ``moe_layer_desc``."""
    _fields_ = [
        ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("D", ctypes.c_int32), ("F", ctypes.c_int32),
        ("F_shared", ctypes.c_int32), ("format", ctypes.c_int32), ("group_size", ctypes.c_int32),
        ("path", ctypes.c_int32),
        ("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
        ("w_gate", ctypes.c_void_p), ("s_gate", ctypes.c_void_p),
        ("w_up", ctypes.c_void_p), ("s_up", ctypes.c_void_p),
        ("w_down", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
        ("act_scale_ub", ctypes.c_float),
        ("ws_gate", ctypes.c_void_p), ("ws_up", ctypes.c_void_p), ("ws_down", ctypes.c_void_p),
        ("rms_weight", ctypes.c_void_p), ("rms_eps", ctypes.c_float),
    ]


class DenseDesc(ctypes.Structure):
    """Mirror of ``moe_dense_desc``."""
    _fields_ = [
        ("D", ctypes.c_int32), ("F", ctypes.c_int32), ("path", ctypes.c_int32),
        ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
        ("rms_weight", ctypes.c_void_p), ("rms_eps", ctypes.c_float),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmoe_int4.so is not built (%s); run "
                               "`python -m int4_quantized_expert_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_abi_version.argtypes = []
        L.moe_abi_version.restype = i32
        L.moe_quantize_int4.argtypes = [vp, i64, i64, i32, vp, vp, vp]
        L.moe_quantize_int4.restype = ctypes.c_int
        L.moe_quantize_fp8_rows.argtypes = [vp, i32, i64, i64, i64, f32, vp, vp, vp]
        L.moe_quantize_fp8_rows.restype = ctypes.c_int
        L.moe_route.argtypes = [vp, i32, i32, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp]
        L.moe_route.restype = ctypes.c_int
        L.moe_ffn_workspace_size.argtypes = [ctypes.POINTER(LayerDesc), i32]
        L.moe_ffn_workspace_size.restype = ctypes.c_size_t
        L.moe_ffn_forward.argtypes = [ctypes.POINTER(LayerDesc), vp, i32, vp, vp, ctypes.c_size_t, vp]
        L.moe_ffn_forward.restype = ctypes.c_int
        L.moe_ffn_forward_host.argtypes = [ctypes.POINTER(LayerDesc), vp, i32, vp, vp, ctypes.c_size_t, vp]
        L.moe_ffn_forward_host.restype = ctypes.c_int
        L.moe_ffn_forward_timed.argtypes = [ctypes.POINTER(LayerDesc), vp, i32, vp, vp, ctypes.c_size_t, vp,
                                            ctypes.POINTER(ctypes.c_void_p), i32]
        L.moe_ffn_forward_timed.restype = ctypes.c_int
        L.moe_ffn_launch_names.argtypes = [ctypes.POINTER(LayerDesc), i32, ctypes.POINTER(ctypes.c_char_p), i32]
        L.moe_ffn_launch_names.restype = i32
        L.moe_ffn_forward_noalloc.argtypes = [ctypes.POINTER(LayerDesc), vp, i32, vp, vp]
        L.moe_ffn_forward_noalloc.restype = ctypes.c_int
        L.moe_ffn_noalloc_device_status.argtypes = [vp]
        L.moe_ffn_noalloc_device_status.restype = ctypes.c_int
        L.moe_expert_ffn_workspace_size.argtypes = [ctypes.POINTER(LayerDesc), i32]
        L.moe_expert_ffn_workspace_size.restype = ctypes.c_size_t
        L.moe_expert_ffn_forward.argtypes = [ctypes.POINTER(LayerDesc), vp, i32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_expert_ffn_forward.restype = ctypes.c_int
        L.moe_shared_ffn_workspace_size.argtypes = [ctypes.POINTER(LayerDesc), i32]
        L.moe_shared_ffn_workspace_size.restype = ctypes.c_size_t
        L.moe_shared_ffn_combine.argtypes = [ctypes.POINTER(LayerDesc), vp, i32, vp, vp, vp, ctypes.c_size_t, vp]
        L.moe_shared_ffn_combine.restype = ctypes.c_int
        L.moe_set_wait_limit.argtypes = [i64]
        L.moe_set_wait_limit.restype = ctypes.c_int
        L.moe_dense_ffn_workspace_size.argtypes = [ctypes.POINTER(DenseDesc), i32]
        L.moe_dense_ffn_workspace_size.restype = ctypes.c_size_t
        L.moe_dense_ffn_forward.argtypes = [ctypes.POINTER(DenseDesc), vp, i32, vp, vp, ctypes.c_size_t, vp]
        L.moe_dense_ffn_forward.restype = ctypes.c_int
        L.moe_rmsnorm.argtypes = [vp, i32, i32, vp, f32, vp, vp]
        L.moe_rmsnorm.restype = ctypes.c_int
        L.moe_ffn_device_status.argtypes = [vp, vp]
        L.moe_ffn_device_status.restype = ctypes.c_int
        _lib = L
    return _lib


def _status_string(status: int) -> str:
    try:
        return lib().moe_status_string(status).decode()
    except Exception:  # pragma: no cover - only for messages
        return "status %d" % status


def _check(fn: str, status: int) -> None:
    if status != Status.OK:
        raise MoEError(fn, status)


def _stream(stream: Optional[torch.cuda.Stream] = None) -> int:
    return (stream or torch.cuda.current_stream()).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def quantize_int4(w: torch.Tensor, group_size: int = 128, stream=None, out=None):
    """int4_row_quantize of fp32 ``w[rows, cols]`` -> (codes uint8 [rows, cols/2],
    scales fp32 [rows, cols/group_size]); ``out`` = optional (codes, scales)."""
    if w.dtype != torch.float32 or w.dim() != 2:
        raise ValueError("w must be a 2-D float32 tensor")
    rows, cols = w.shape
    if out is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=w.device)
        scales = torch.empty(rows, max(cols // group_size, 1), dtype=torch.float32, device=w.device)
    else:
        codes, scales = out
        if codes.numel() * 2 != rows * cols or scales.numel() * group_size != rows * cols:
            raise ValueError("output tensors have the wrong size")
    _check("moe_quantize_int4", lib().moe_quantize_int4(
        _ptr(w), rows, cols, group_size, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def quantize_fp8_rows(x: torch.Tensor, num_valid_rows: Optional[int] = None,
                      scale_ub: float = math.inf, stream=None, out=None):
    """Per-row e4m3 quantization of bf16/fp32 ``x[rows, cols]`` -> (q uint8, s fp32 [rows]);
    ``out`` = optional (q, s)."""
    if x.dim() != 2 or x.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("x must be a 2-D bf16 or fp32 tensor")
    rows, cols = x.shape
    nv = rows if num_valid_rows is None else int(num_valid_rows)
    if out is None:
        q = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
        s = torch.empty(rows, dtype=torch.float32, device=x.device)
    else:
        q, s = out
        if q.numel() != rows * cols or s.numel() != rows:
            raise ValueError("output tensors have the wrong size")
    dt = DTYPE_BF16 if x.dtype == torch.bfloat16 else DTYPE_FP32
    _check("moe_quantize_fp8_rows", lib().moe_quantize_fp8_rows(
        _ptr(x), dt, rows, cols, nv, ctypes.c_float(scale_ub), _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def rmsnorm(x: torch.Tensor, gamma: torch.Tensor, eps: float, stream=None, out=None) -> torch.Tensor:
    """RMSNorm of bf16 ``x[T, D]`` with bf16 ``gamma[D]`` (see ``moe_rmsnorm``)."""
    if x.dtype != torch.bfloat16 or gamma.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bf16 tensor and gamma bf16")
    T, D = x.shape
    out = torch.empty_like(x) if out is None else out
    _check("moe_rmsnorm", lib().moe_rmsnorm(_ptr(x), T, D, _ptr(gamma), ctypes.c_float(eps), _ptr(out),
                                            _stream(stream)))
    return out


def route(x: torch.Tensor, w_router: torch.Tensor, bias: Optional[torch.Tensor], k: int, stream=None) -> dict:
    """Router + top-k + gate + bucketing (see ``moe_route``)."""
    T, D = x.shape
    E = w_router.shape[0]
    dev = x.device
    out = dict(ids=torch.empty(T, k, dtype=torch.int32, device=dev),
               gates=torch.empty(T, k, dtype=torch.float32, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               perm=torch.empty(T * k, dtype=torch.int32, device=dev))
    _check("moe_route", lib().moe_route(
        _ptr(x), T, D, _ptr(w_router), _ptr(bias), E, k, _ptr(out["ids"]), _ptr(out["gates"]),
        _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["perm"]), _stream(stream)))
    return out


class MoELayer:
    """One MoE FFN layer on the GPU: holds the (already quantized) weights,
    a workspace for up to ``T_max`` tokens, and the ``moe_layer_desc``.

    Routed weights: int4 -- (codes uint8 [E, N, K/2], scales fp32 [E, N, K/group_size])
    per projection, group_size 128, 64 or 32; fp8 -- (codes uint8 [E, N, K],
    scales fp32 [E, N]).
    """

    def __init__(self, *, E: int, k: int, D: int, F: int, F_shared: int, w_router: torch.Tensor,
                 router_bias: Optional[torch.Tensor], gate, up, down, shared, fmt: int = FMT_INT4,
                 act_scale_ub: float = math.inf, T_max: int = 16, path: int = PATH_AUTO,
                 group_size: int = 128, rms_weight: Optional[torch.Tensor] = None, rms_eps: float = 1e-5):
        self.tensors = [w_router, router_bias, *gate, *up, *down, *shared, rms_weight]   # keep alive
        d = LayerDesc()
        d.E, d.k, d.D, d.F, d.F_shared = E, k, D, F, F_shared
        d.format, d.group_size, d.path = fmt, group_size, path
        d.w_router, d.router_bias = _ptr(w_router), _ptr(router_bias)
        d.w_gate, d.s_gate = _ptr(gate[0]), _ptr(gate[1])
        d.w_up, d.s_up = _ptr(up[0]), _ptr(up[1])
        d.w_down, d.s_down = _ptr(down[0]), _ptr(down[1])
        d.act_scale_ub = act_scale_ub
        d.ws_gate, d.ws_up, d.ws_down = (_ptr(t) for t in shared)
        d.rms_weight, d.rms_eps = _ptr(rms_weight), rms_eps
        self.desc = d
        self.D = D
        self.device = w_router.device
        self.T_max = 0
        self.workspace = None
        self.reserve(T_max)

    def workspace_bytes(self, T: int) -> int:
        n = lib().moe_ffn_workspace_size(ctypes.byref(self.desc), T)
        if n == 0:
            raise MoEError("moe_ffn_workspace_size", Status.UNSUPPORTED_SHAPE)
        return n

    def reserve(self, T_max: int) -> None:
        """Make the workspace large enough for up to ``T_max`` tokens with the
        current path setting (its size depends on the path)."""
        if T_max <= self.T_max:
            return
        n = self.workspace_bytes(T_max)
        if self.workspace is None or self.workspace.numel() < n:
            self.workspace = torch.empty(n, dtype=torch.uint8, device=self.device)
        self.T_max = T_max

    def set_path(self, path: int) -> None:
        if path != self.desc.path:
            self.desc.path = path
            T_max, self.T_max = self.T_max, 0
            self.reserve(T_max)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        self.reserve(T)
        if out is None:
            out = torch.empty(T, self.D, dtype=torch.bfloat16, device=x.device)
        _check("moe_ffn_forward", lib().moe_ffn_forward(
            ctypes.byref(self.desc), _ptr(x), T, _ptr(out), _ptr(self.workspace), self.workspace.numel(),
            _stream(stream)))
        return out

    __call__ = forward

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor, stream=None) -> None:
        """Host buffers in and out (pinned memory recommended); asynchronous."""
        T = x_host.shape[0]
        self.reserve(T)
        _check("moe_ffn_forward_host", lib().moe_ffn_forward_host(
            ctypes.byref(self.desc), x_host.data_ptr(), T, out_host.data_ptr(), _ptr(self.workspace),
            self.workspace.numel(), _stream(stream)))

    def launch_names(self, T: int) -> list:
        """Names of the kernels one forward launches, in order."""
        n = lib().moe_ffn_launch_names(ctypes.byref(self.desc), T, None, 0)
        arr = (ctypes.c_char_p * max(n, 1))()
        lib().moe_ffn_launch_names(ctypes.byref(self.desc), T, arr, n)
        return [arr[i].decode() for i in range(n)]

    def forward_timed(self, x: torch.Tensor, out: torch.Tensor, events: list, stream=None) -> None:
        """forward() that records ``events`` (torch.cuda.Event, already
        created) before each kernel launch and after the last one."""
        T = x.shape[0]
        self.reserve(T)
        handles = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        _check("moe_ffn_forward_timed", lib().moe_ffn_forward_timed(
            ctypes.byref(self.desc), _ptr(x), T, _ptr(out), _ptr(self.workspace), self.workspace.numel(),
            _stream(stream), handles, len(events)))

    def device_status(self, stream=None) -> int:
        """Synchronizes the stream; the device status of the last forward."""
        return lib().moe_ffn_device_status(_ptr(self.workspace), _stream(stream))

    def forward_noalloc(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """forward() without the workspace: the library's own fixed scratch
        (``moe_ffn_forward_noalloc``; decode-sized batches only)."""
        if out is None:
            out = torch.empty(x.shape[0], self.D, dtype=torch.bfloat16, device=x.device)
        _check("moe_ffn_forward_noalloc", lib().moe_ffn_forward_noalloc(
            ctypes.byref(self.desc), _ptr(x), x.shape[0], _ptr(out), _stream(stream)))
        return out


    # ---- the compute steps of an expert-parallel layer (see moe_expert_ffn_forward) ----
    def _scratch(self, attr: str, n: int) -> torch.Tensor:
        ws = getattr(self, attr, None)
        if ws is None or ws.numel() < n:
            ws = torch.empty(n, dtype=torch.uint8, device=self.device)
            setattr(self, attr, ws)
        return ws

    def expert_forward(self, x: torch.Tensor, expert_ids: torch.Tensor, gates: torch.Tensor,
                       stream=None) -> torch.Tensor:
        """y[r] = gates[r] * expert_{ids[r]}(x[r]), fp32 [n, D]."""
        n = x.shape[0]
        y = torch.empty(n, self.D, dtype=torch.float32, device=x.device)
        if n == 0:
            return y
        need = lib().moe_expert_ffn_workspace_size(ctypes.byref(self.desc), n)
        if need == 0:
            raise MoEError("moe_expert_ffn_workspace_size", Status.UNSUPPORTED_SHAPE)
        ws = self._scratch("_expert_ws", need)
        _check("moe_expert_ffn_forward", lib().moe_expert_ffn_forward(
            ctypes.byref(self.desc), _ptr(x), n, _ptr(expert_ids), _ptr(gates), _ptr(y), _ptr(ws), ws.numel(),
            _stream(stream)))
        self._last_ws = ws
        return y

    def shared_combine(self, x: torch.Tensor, y_slots: torch.Tensor, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
        """out[t] = bf16(shared(x[t]) + sum_j y_slots[t, j]), y_slots fp32 [T, k, D]."""
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, self.D, dtype=torch.bfloat16, device=x.device)
        need = lib().moe_shared_ffn_workspace_size(ctypes.byref(self.desc), T)
        if need == 0:
            raise MoEError("moe_shared_ffn_workspace_size", Status.UNSUPPORTED_SHAPE)
        ws = self._scratch("_shared_ws", need)
        _check("moe_shared_ffn_combine", lib().moe_shared_ffn_combine(
            ctypes.byref(self.desc), _ptr(x), T, _ptr(y_slots), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
        self._last_ws = ws
        return out

    def last_call_status(self, stream=None) -> int:
        """Synchronizes; the device status of the last expert_forward / shared_combine."""
        return lib().moe_ffn_device_status(_ptr(self._last_ws), _stream(stream))


def noalloc_device_status(stream=None) -> int:
    """Synchronizes the stream; the device status of the last no-alloc forward."""
    return lib().moe_ffn_noalloc_device_status(_stream(stream))


def set_wait_limit(cycles: int) -> None:
    """Limit of the kernels' bounded waits in SM cycles (<= 0: the default);
    lowering it makes the next forward time out, to test that path."""
    _check("moe_set_wait_limit", lib().moe_set_wait_limit(int(cycles)))


class DenseLayer:
    """A dense SwiGLU FFN layer (``moe_dense_ffn_forward``): bf16 weights
    w_gate, w_up [F, D] and w_down [D, F], an optional RMSNorm of x first,
    and a workspace for up to ``T_max`` tokens."""

    def __init__(self, *, D: int, F: int, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                 path: int = PATH_AUTO, T_max: int = 16, rms_weight: Optional[torch.Tensor] = None,
                 rms_eps: float = 1e-5):
        self.tensors = [w_gate, w_up, w_down, rms_weight]   # keep alive
        d = DenseDesc()
        d.D, d.F, d.path = D, F, path
        d.w_gate, d.w_up, d.w_down = _ptr(w_gate), _ptr(w_up), _ptr(w_down)
        d.rms_weight, d.rms_eps = _ptr(rms_weight), rms_eps
        self.desc = d
        self.D = D
        self.device = w_gate.device
        self.workspace = None
        self.T_max = 0
        self.reserve(T_max)

    def workspace_bytes(self, T: int) -> int:
        n = lib().moe_dense_ffn_workspace_size(ctypes.byref(self.desc), T)
        if n == 0:
            raise MoEError("moe_dense_ffn_workspace_size", Status.UNSUPPORTED_SHAPE)
        return n

    def reserve(self, T_max: int) -> None:
        if T_max <= self.T_max:
            return
        n = self.workspace_bytes(T_max)
        if self.workspace is None or self.workspace.numel() < n:
            self.workspace = torch.empty(n, dtype=torch.uint8, device=self.device)
        self.T_max = T_max

    def set_path(self, path: int) -> None:
        if path != self.desc.path:
            self.desc.path = path
            T_max, self.T_max = self.T_max, 0
            self.reserve(T_max)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        self.reserve(T)
        if out is None:
            out = torch.empty(T, self.D, dtype=torch.bfloat16, device=x.device)
        _check("moe_dense_ffn_forward", lib().moe_dense_ffn_forward(
            ctypes.byref(self.desc), _ptr(x), T, _ptr(out), _ptr(self.workspace), self.workspace.numel(),
            _stream(stream)))
        return out

    __call__ = forward

    def device_status(self, stream=None) -> int:
        """Synchronizes the stream; the device status of the last forward."""
        return lib().moe_ffn_device_status(_ptr(self.workspace), _stream(stream))
