"""CPU oracle for the ConvRot-quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``rotated_bit_quantized_block_b200``) never imports, links or executes it, and
the two share no code: the arithmetic lives in ``convrot_oracle.c`` (plain C,
float64 where the pages fix no precision, compiled with ``-ffp-contract=off``),
this module only marshals numpy arrays.

Each function cites the passage of the source pages that it follows:

* civarchive.com, "SAM 3.1 Multiplex ConvRot" release, "Quantization recipe":
  upcast to FP32, block-Hadamard ConvRot transform, MSE-optimized clipping
  scale, per-row scales; W8A8 / W4A4 operations with online dynamic activation
  quantization.
* trellis3d.app, "TRELLIS.2 INT8 ConvRot in ComfyUI", "What ConvRot changes":
  grouped, normalized Hadamard rotation before per-row weight quantization,
  the matching rotation applied to activations at runtime.
* salahadawi.com, "Explanation of INT8 ConvRot", "8-bit INT type models" table:
  INT8 encoding with row-wise scaling.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, library routines, brute force, page-printed values); none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import fcntl
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "convrot_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPE_F16, DTYPE_BF16, DTYPE_F32 = 0, 1, 2
CLIP_ABSMAX, CLIP_MSE = 0, 1
MSE_GRID = 51

_lib = None


def build(force: bool = False) -> str:
    """Compile ``convrot_oracle.c`` into ``liboracle.so`` (gcc, OpenMP)."""
    lock_path = _LIB + ".lock"
    with open(lock_path, "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                   "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
    sig = {
        "oracle_f16_to_f64": (f64, [ctypes.c_uint16]),
        "oracle_f32_to_f16": (ctypes.c_uint16, [f32]),
        "oracle_decode": (i32, [P, i32, i64, P]),
        "oracle_f32_to_f16_array": (None, [P, i64, P]),
        "oracle_hadamard": (i32, [i32, P]),
        "oracle_rotate": (i32, [P, i64, i64, i32, P, P]),
        "oracle_qmax": (i32, [i32]),
        "oracle_qmin": (i32, [i32]),
        "oracle_scale": (f32, [f32, f32, i32]),
        "oracle_inv_scale": (f32, [f32]),
        "oracle_quantize_value": (i32, [f32, f32, i32]),
        "oracle_quant_error": (f64, [P, i64, f32, i32]),
        "oracle_alpha": (f32, [i32]),
        "oracle_quantize_weight": (i32, [P, i32, i64, i64, i32, i32, i32, P, P, P, P]),
        "oracle_quantize_weight_tensorwise": (i32, [P, i32, i64, i64, i32, i32, i32, P, P, P, P]),
        "oracle_rotate_quant_act": (i32, [P, i64, i64, i32, i32, P, P]),
        "oracle_pack_int4": (i32, [P, i64, P]),
        "oracle_unpack_int4": (i32, [P, i64, P]),
        "oracle_weight_bytes": (i64, [i64, i64, i32]),
        "oracle_gemm_dequant": (i32, [P, P, i64, P, P, i64, i64, P, P, P]),
        "oracle_epilogue_value": (f32, [i32, f32, f32, f32]),
        "oracle_set_threads": (i32, [i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def set_threads(n: int) -> int:
    """OpenMP thread count used by the row loops (results do not depend on it)."""
    return _load().oracle_set_threads(int(n))


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def f16_bits(a) -> np.ndarray:
    """fp16 values (np.float16 array) -> their uint16 bit patterns."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float16)).view(np.uint16)


def decode(src_bits: np.ndarray, dtype: int) -> np.ndarray:
    """Upcast fp16 / bf16 bit patterns (uint16) or fp32 values to float64 exactly."""
    src = np.ascontiguousarray(src_bits)
    out = np.empty(src.shape, dtype=np.float64)
    _check(_load().oracle_decode(_ptr(src), dtype, src.size, _ptr(out)), "decode")
    return out


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> binary16 bit patterns, round to nearest even (hand-written)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f32_to_f16_array(_ptr(x), x.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------
# the rotation ("block-Hadamard ConvRot transform"; "grouped, normalized
# Hadamard rotation")
# ----------------------------------------------------------------------------

def hadamard(b: int) -> np.ndarray:
    """R_b = H_b / sqrt(b), Sylvester order, float64 (b x b)."""
    R = np.empty((b, b), dtype=np.float64)
    _check(_load().oracle_hadamard(int(b), _ptr(R)), "hadamard")
    return R


def rotate(X64: np.ndarray, b: int):
    """X (rows x K, float64) . blockdiag(R_b): returns (float64 product, fp32 rounding)."""
    X64 = np.ascontiguousarray(X64, dtype=np.float64)
    rows, K = X64.shape
    o64 = np.empty((rows, K), dtype=np.float64)
    o32 = np.empty((rows, K), dtype=np.float32)
    _check(_load().oracle_rotate(_ptr(X64), rows, K, int(b), _ptr(o64), _ptr(o32)), "rotate")
    return o64, o32


# ----------------------------------------------------------------------------
# quantization
# ----------------------------------------------------------------------------

def qmax(bits: int) -> int:
    return _load().oracle_qmax(bits)


def qmin(bits: int) -> int:
    return _load().oracle_qmin(bits)


def alpha(i: int) -> float:
    """Clip factor of MSE grid point i (i = 0 is 1.0, i = 50 is 0.5)."""
    return _load().oracle_alpha(int(i))


def scale(amax: float, alpha_: float, bits: int) -> float:
    return _load().oracle_scale(float(amax), float(alpha_), bits)


def quant_error(row32: np.ndarray, s: float, bits: int) -> float:
    """sum_k (x_k - s * q_k)^2 in float64 for one fp32 row under scale s."""
    row32 = np.ascontiguousarray(row32, dtype=np.float32)
    return _load().oracle_quant_error(_ptr(row32), row32.size, float(s), bits)


def quantize_weight(W, b: int, bits: int, clip_mode: int = CLIP_MSE, dtype: int = DTYPE_F16,
                    want_errs: bool = False):
    """Offline converter (recipe steps 1-4).

    ``W`` is N x K: uint16 fp16/bf16 bit patterns, np.float16 (treated as fp16
    bits) or float32 (with ``dtype=DTYPE_F32``).  Returns
    ``(codes int8 N x K unpacked, scales fp32 N, alpha_idx int32 N[, errs N x 51])``.
    """
    if isinstance(W, np.ndarray) and W.dtype == np.float16:
        W = W.view(np.uint16)
    W = np.ascontiguousarray(W)
    N, K = W.shape
    codes = np.empty((N, K), dtype=np.int8)
    scales = np.empty(N, dtype=np.float32)
    aidx = np.empty(N, dtype=np.int32)
    errs = np.empty((N, MSE_GRID), dtype=np.float64) if want_errs else None
    rc = _load().oracle_quantize_weight(_ptr(W), dtype, N, K, int(b), bits, clip_mode,
                                        _ptr(codes), _ptr(scales), _ptr(aidx), _ptr(errs))
    _check(rc, "quantize_weight")
    return (codes, scales, aidx, errs) if want_errs else (codes, scales, aidx)


def quantize_weight_tensorwise(W, b: int, bits: int, clip_mode: int = CLIP_MSE, dtype: int = DTYPE_F16,
                               want_errs: bool = False):
    """Tensor-wise variant of the converter: one scale for the whole weight
    tensor (salahadawi.com "Explanation of INT8 ConvRot", "8-bit INT type
    models" table, Tensor-wise scaling; civarchive.com release, downloads
    table, int8_tensorwise).  Returns ``(codes int8 N x K, scales fp32 N (all
    equal), alpha_idx int[, errs 51])``.
    """
    if isinstance(W, np.ndarray) and W.dtype == np.float16:
        W = W.view(np.uint16)
    W = np.ascontiguousarray(W)
    N, K = W.shape
    codes = np.empty((N, K), dtype=np.int8)
    scales = np.empty(N, dtype=np.float32)
    aidx = np.zeros(1, dtype=np.int32)
    errs = np.empty(MSE_GRID, dtype=np.float64) if want_errs else None
    rc = _load().oracle_quantize_weight_tensorwise(_ptr(W), dtype, N, K, int(b), bits, clip_mode,
                                                   _ptr(codes), _ptr(scales), _ptr(aidx), _ptr(errs))
    _check(rc, "quantize_weight_tensorwise")
    return (codes, scales, int(aidx[0]), errs) if want_errs else (codes, scales, int(aidx[0]))


def rotate_quant_act(X_f16, b: int, bits: int):
    """Online activation path: per-token dynamic absmax quantization of X.R.

    ``X_f16`` is M x K np.float16 (or its uint16 bits).  Returns
    ``(codes int8 M x K unpacked, scales fp32 M)``.
    """
    X = np.ascontiguousarray(X_f16)
    if X.dtype == np.float16:
        X = X.view(np.uint16)
    M, K = X.shape
    codes = np.empty((M, K), dtype=np.int8)
    scales = np.empty(M, dtype=np.float32)
    _check(_load().oracle_rotate_quant_act(_ptr(X), M, K, int(b), bits, _ptr(codes), _ptr(scales)),
           "rotate_quant_act")
    return codes, scales


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Pack int4 codes two per byte along the last axis (low nibble = even element)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    shape = codes.shape[:-1] + (codes.shape[-1] // 2,)
    out = np.empty(shape, dtype=np.uint8)
    _check(_load().oracle_pack_int4(_ptr(codes), codes.size, _ptr(out)), "pack_int4")
    return out


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    shape = packed.shape[:-1] + (packed.shape[-1] * 2,)
    out = np.empty(shape, dtype=np.int8)
    _check(_load().oracle_unpack_int4(_ptr(packed), out.size, _ptr(out)), "unpack_int4")
    return out


def weight_bytes(N: int, K: int, bits: int) -> int:
    """Stored bytes of a quantized N x K linear weight: codes + fp32 row scales."""
    return _load().oracle_weight_bytes(N, K, bits)


# ----------------------------------------------------------------------------
# GEMM + dequant epilogue
# ----------------------------------------------------------------------------

def gemm_dequant(qx, sx, qw, sw, bias_f16=None, want_acc: bool = False):
    """y = fp16(fma(fp32((float)acc * s_x[m]), s_w[n], bias[n])), acc = qx . qw^T (int).

    Codes are unpacked int8 (int4 values simply lie in [-8, 7]).  Returns y as
    np.float16 (M x N) and, if asked, the int32 accumulators.
    """
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = qx.shape
    N, K2 = qw.shape
    assert K == K2 and sx.shape == (M,) and sw.shape == (N,)
    bias = None
    if bias_f16 is not None:
        bias = np.ascontiguousarray(bias_f16)
        if bias.dtype == np.float16:
            bias = bias.view(np.uint16)
        assert bias.shape == (N,)
    y = np.empty((M, N), dtype=np.uint16)
    acc = np.empty((M, N), dtype=np.int32) if want_acc else None
    _check(_load().oracle_gemm_dequant(_ptr(qx), _ptr(sx), M, _ptr(qw), _ptr(sw), N, K, _ptr(bias),
                                       _ptr(acc), _ptr(y)), "gemm_dequant")
    y = y.view(np.float16)
    return (y, acc) if want_acc else y


def epilogue_value(acc: int, sx: float, sw: float, bias: float) -> float:
    """fp32 value of one output before the fp16 conversion: fma(fp32(acc * sx), sw, bias)."""
    return _load().oracle_epilogue_value(int(acc), float(sx), float(sw), float(bias))


def quantize_value(x: float, inv: float, bits: int) -> int:
    """clamp(rne(x * inv)) with the exact product."""
    return _load().oracle_quantize_value(float(x), float(inv), bits)


def linear(X_f16, w_codes, w_scales, b: int, bits: int, bias_f16=None):
    """The whole online path: rotate + per-token quant of X, integer GEMM, dequant."""
    qx, sx = rotate_quant_act(X_f16, b, bits)
    return gemm_dequant(qx, sx, w_codes, w_scales, bias_f16)
