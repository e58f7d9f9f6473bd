"""Thin Python binding of the C ABI in ``include/convrot.h``.

Functions carry the C names.  They only marshal arguments: torch tensors provide
device memory and the current CUDA stream, every step of the computation runs
in ``libconvrot.so``.  There is no CPU or PyTorch fallback: if the library
cannot be loaded the call raises.
"""
from __future__ import annotations

import ctypes
import threading

import torch

from . import _build

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(7)
CLIP_ABSMAX, CLIP_MSE = 0, 1
DTYPE_F16, DTYPE_BF16, DTYPE_F32 = 0, 1, 2
_TORCH_DTYPE = {torch.float16: DTYPE_F16, torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}

EXPORTED = (
    "convrot_quantize_weight", "convrot_rotate_quant_act", "convrot_workspace_bytes",
    "convrot_linear_w8a8", "convrot_linear_w4a4", "convrot_gemm_w8a8", "convrot_gemm_w4a4",
    "convrot_device_status", "convrot_status_string", "convrot_last_error", "convrot_version",
    "convrot_linear_w8a8_noalloc", "convrot_linear_quant_act", "convrot_linear_gemm",
    "convrot_linear_workspace_bytes", "convrot_tensorwise_workspace_bytes", "convrot_quantize_weight_tensorwise",
    "convrot_test_abandoned_wait", "convrot_linear_plan", "convrot_linear_w8a8_fused",
)


class LinearPlan(ctypes.Structure):
    """convrot_linear_plan_t: how a linear call runs (see include/convrot.h)."""
    _fields_ = [("launches", ctypes.c_int), ("gemm_kind", ctypes.c_int), ("tile_n", ctypes.c_int),
                ("cta_pair", ctypes.c_int), ("stream_k", ctypes.c_int), ("k_splits", ctypes.c_int),
                ("fused_available", ctypes.c_int), ("weights_widened", ctypes.c_int)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class ConvRotError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"convrot status {status}: {message}")
        self.status = status


_lib = None
_lock = threading.Lock()


def load_library(build_if_missing: bool = True) -> ctypes.CDLL:
    """Loads ``libconvrot.so`` from the package directory (building it with nvcc if absent)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if build_if_missing and _build.is_stale():
            _build.build()
        lib = ctypes.CDLL(_build.LIB_PATH)
        P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sig = {
            "convrot_quantize_weight": (i32, [P, i32, i64, i64, i32, i32, i32, P, P, P]),
            "convrot_rotate_quant_act": (i32, [P, i64, i64, i32, i32, P, P, P]),
            "convrot_workspace_bytes": (sz, [i64, i64, i32]),
            "convrot_linear_workspace_bytes": (sz, [i64, i64, i64, i32]),
            "convrot_tensorwise_workspace_bytes": (sz, [i64, i32]),
            "convrot_quantize_weight_tensorwise": (i32, [P, i32, i64, i64, i32, i32, i32, P, P, P, sz, P]),
            "convrot_linear_w8a8": (i32, [P, i64, i64, P, P, i64, P, i32, P, P, sz, P]),
            "convrot_linear_w4a4": (i32, [P, i64, i64, P, P, i64, P, i32, P, P, sz, P]),
            "convrot_linear_w8a8_fused": (i32, [P, i64, i64, P, P, i64, P, i32, P, P, sz, P]),
            "convrot_gemm_w8a8": (i32, [P, P, i64, P, P, i64, i64, P, P, P, P]),
            "convrot_gemm_w4a4": (i32, [P, P, i64, P, P, i64, i64, P, P, P, P]),
            "convrot_linear_w8a8_noalloc": (i32, [P, i64, i64, P, P, i64, P, i32, P, P]),
            "convrot_linear_quant_act": (i32, [P, i64, i64, i32, i32, P, sz, P]),
            "convrot_linear_gemm": (i32, [P, sz, i64, i64, i32, P, P, i64, P, P, P]),
            "convrot_device_status": (i32, [P]),
            "convrot_test_abandoned_wait": (i32, [i32, ctypes.c_uint64, P, P]),
            "convrot_linear_plan": (i32, [i64, i64, i64, i32, i32, sz, ctypes.POINTER(LinearPlan)]),
            "convrot_status_string": (ctypes.c_char_p, [i32]),
            "convrot_last_error": (ctypes.c_char_p, []),
            "convrot_version": (i32, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int):
    if status != OK:
        lib = load_library()
        raise ConvRotError(status, lib.convrot_last_error().decode() or lib.convrot_status_string(status).decode())


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def code_shape(rows: int, K: int, bits: int):
    return (rows, K) if bits == 8 else (rows, K // 2)


def code_dtype(bits: int):
    return torch.int8 if bits == 8 else torch.uint8


# ---------------------------------------------------------------------------- entry points

def convrot_quantize_weight(W: torch.Tensor, block: int, bits: int, clip_mode: int = CLIP_MSE, Wq=None,
                            w_scale=None, stream=None):
    """Offline rotate + clip search + per-row quantization of W (N x K fp16/bf16/fp32)."""
    _dev(W, "W")
    N, K = W.shape
    if Wq is None:
        Wq = torch.empty(code_shape(N, K, bits), dtype=code_dtype(bits), device=W.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=W.device)
    st = load_library().convrot_quantize_weight(_ptr(W), _TORCH_DTYPE[W.dtype], N, K, block, bits, clip_mode,
                                                _ptr(Wq), _ptr(w_scale), _stream(stream))
    _check(st)
    return Wq, w_scale


def convrot_tensorwise_workspace_bytes(N: int, clip_mode: int) -> int:
    return int(load_library().convrot_tensorwise_workspace_bytes(N, clip_mode))


def convrot_quantize_weight_tensorwise(W: torch.Tensor, block: int, bits: int, clip_mode: int = CLIP_MSE, Wq=None,
                                       w_scale=None, workspace=None, stream=None):
    """Offline rotate + clip search + quantization of W with one scale for the
    whole tensor (w_scale holds it for every row)."""
    _dev(W, "W")
    N, K = W.shape
    if Wq is None:
        Wq = torch.empty(code_shape(N, K, bits), dtype=code_dtype(bits), device=W.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = torch.empty(max(1, convrot_tensorwise_workspace_bytes(N, clip_mode)), dtype=torch.uint8,
                                device=W.device)
    st = load_library().convrot_quantize_weight_tensorwise(
        _ptr(W), _TORCH_DTYPE[W.dtype], N, K, block, bits, clip_mode, _ptr(Wq), _ptr(w_scale), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return Wq, w_scale


def convrot_rotate_quant_act(X: torch.Tensor, block: int, bits: int, Xq=None, x_scale=None, stream=None):
    """Online rotation + per-token quantization of X (M x K fp16)."""
    _dev(X, "X")
    if X.dtype != torch.float16:
        raise ValueError("X must be fp16")
    M, K = X.shape
    if Xq is None:
        Xq = torch.empty(code_shape(M, K, bits), dtype=code_dtype(bits), device=X.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=X.device)
    st = load_library().convrot_rotate_quant_act(_ptr(X), M, K, block, bits, _ptr(Xq), _ptr(x_scale),
                                                 _stream(stream))
    _check(st)
    return Xq, x_scale


def convrot_workspace_bytes(M: int, K: int, bits: int) -> int:
    return int(load_library().convrot_workspace_bytes(M, K, bits))


def convrot_linear_workspace_bytes(M: int, K: int, N: int, bits: int) -> int:
    """Workspace that also enables split-K in the linear's GEMM."""
    return int(load_library().convrot_linear_workspace_bytes(M, K, N, bits))


def _linear(fn_name, bits, X, Wq, w_scale, block, bias, Y, workspace, stream):
    _dev(X, "X")
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    if workspace is None:
        need = convrot_linear_workspace_bytes(M, K, N, bits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    fn = getattr(load_library(), fn_name)
    st = fn(_ptr(X), M, K, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), block, _ptr(Y), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return Y


def convrot_linear_w8a8(X, Wq, w_scale, block, bias=None, Y=None, workspace=None, stream=None):
    """Y = ConvRot W8A8 linear of X (fp16) with int8 weight codes Wq (N x K)."""
    return _linear("convrot_linear_w8a8", 8, X, Wq, w_scale, block, bias, Y, workspace, stream)


def convrot_linear_w8a8_fused(X, Wq, w_scale, block, bias=None, Y=None, workspace=None, stream=None):
    """The W8A8 linear as one GEMM kernel whose activation warps rotate and quantize X."""
    return _linear("convrot_linear_w8a8_fused", 8, X, Wq, w_scale, block, bias, Y, workspace, stream)


def convrot_linear_w4a4(X, Wq, w_scale, block, bias=None, Y=None, workspace=None, stream=None):
    """Y = ConvRot W4A4 linear of X (fp16) with packed int4 weight codes Wq (N x K/2)."""
    return _linear("convrot_linear_w4a4", 4, X, Wq, w_scale, block, bias, Y, workspace, stream)


def convrot_linear_quant_act(X, block, bits, workspace, stream=None):
    """First launch of a linear: rotate + quantize X into the linear's workspace."""
    _dev(X, "X")
    M, K = X.shape
    st = load_library().convrot_linear_quant_act(_ptr(X), M, K, block, bits, _ptr(workspace),
                                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)


def convrot_linear_gemm(workspace, M, K, bits, Wq, w_scale, bias=None, Y=None, stream=None):
    """Second launch of a linear: integer GEMM + dequant from the workspace."""
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=Wq.device)
    st = load_library().convrot_linear_gemm(_ptr(workspace), workspace.numel() * workspace.element_size(), M, K,
                                            bits, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), _ptr(Y), _stream(stream))
    _check(st)
    return Y


def _gemm(fn_name, Xq, x_scale, Wq, w_scale, K, bias, Y, acc_out, stream):
    M, N = Xq.shape[0], Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=Xq.device)
    fn = getattr(load_library(), fn_name)
    st = fn(_ptr(Xq), _ptr(x_scale), M, _ptr(Wq), _ptr(w_scale), N, K, _ptr(bias), _ptr(Y), _ptr(acc_out),
            _stream(stream))
    _check(st)
    return Y


def convrot_gemm_w8a8(Xq, x_scale, Wq, w_scale, bias=None, Y=None, acc_out=None, stream=None):
    """Integer GEMM + dequant epilogue on int8 codes (Xq M x K, Wq N x K)."""
    return _gemm("convrot_gemm_w8a8", Xq, x_scale, Wq, w_scale, Xq.shape[1], bias, Y, acc_out, stream)


def convrot_gemm_w4a4(Xq, x_scale, Wq, w_scale, bias=None, Y=None, acc_out=None, stream=None):
    """Integer GEMM + dequant epilogue on packed int4 codes (Xq M x K/2, Wq N x K/2)."""
    return _gemm("convrot_gemm_w4a4", Xq, x_scale, Wq, w_scale, Xq.shape[1] * 2, bias, Y, acc_out, stream)


def convrot_linear_w8a8_noalloc(X, Wq, w_scale, block, bias=None, Y=None, stream=None):
    """W8A8 ConvRot linear without a workspace: for callers that may not allocate
    device memory.  The codes and scales go to a fixed 16 MiB array inside the
    library (shared by all calls on a device), so M*K is limited to about 16 MiB."""
    _dev(X, "X")
    M, K = X.shape
    N = Wq.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    st = load_library().convrot_linear_w8a8_noalloc(_ptr(X), M, K, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), block,
                                                    _ptr(Y), _stream(stream))
    _check(st)
    return Y


def convrot_device_status(stream=None):
    """Synchronizes the stream and raises if a kernel recorded a device-side timeout."""
    _check(load_library().convrot_device_status(_stream(stream)))


def convrot_linear_plan(M: int, K: int, N: int, bits: int, block: int, workspace_bytes: int) -> dict:
    """How a linear of these sizes runs with this workspace (launches, fused, GEMM kind, tile)."""
    plan = LinearPlan()
    _check(load_library().convrot_linear_plan(M, K, N, bits, block, workspace_bytes, ctypes.byref(plan)))
    return plan.as_dict()


def convrot_test_abandoned_wait(kind: int, limit_ns: int, result: torch.Tensor, stream=None):
    """Diagnostics: one bounded device wait that runs out (kind 0: mbarrier,
    1: fused-prologue flag) after limit_ns; result is an int32[4] CUDA tensor."""
    _dev(result, "result")
    _check(load_library().convrot_test_abandoned_wait(kind, limit_ns, _ptr(result), _stream(stream)))


def convrot_version() -> int:
    return int(load_library().convrot_version())


class QuantizedLinear:
    """A ConvRot-quantized nn.Linear: holds the codes, scales, bias and a workspace."""

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None = None, block: int = 128, bits: int = 8,
                 clip_mode: int = CLIP_MSE):
        self.block, self.bits = block, bits
        self.N, self.K = weight.shape
        self.Wq, self.w_scale = convrot_quantize_weight(weight.contiguous(), block, bits, clip_mode)
        self.bias = None if bias is None else bias.to(torch.float16).contiguous()
        self._ws = None

    def workspace(self, M: int, device) -> torch.Tensor:
        need = convrot_linear_workspace_bytes(M, self.K, self.N, self.bits)
        if self._ws is None or self._ws.numel() < need or self._ws.device != device:
            self._ws = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
        return self._ws

    def __call__(self, X: torch.Tensor, Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        shape = X.shape
        X2 = X.reshape(-1, self.K).contiguous()
        ws = self.workspace(X2.shape[0], X2.device)
        fn = convrot_linear_w8a8 if self.bits == 8 else convrot_linear_w4a4
        out = fn(X2, self.Wq, self.w_scale, self.block, self.bias, Y, ws, stream)
        return out.reshape(*shape[:-1], self.N)
