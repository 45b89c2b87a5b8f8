"""CPU oracle for FP8 scaled quantization -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library (``fine_grained_block_b200``)
never does, and this package imports nothing from it: the two share no code.

The arithmetic lives in ``fp8_oracle.c`` (plain scalar C, see its header for
the pages and readings it follows).  This module only loads it and marshals
numpy arrays in and out.

Format / dtype numbering used here: fmt 0 = E4M3 (float8_e4m3fn), 1 = E5M2
(float8_e5m2); dtype 0 = fp32, 1 = bf16 (bf16 arrays are numpy uint16 holding
the bit pattern).
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

E4M3, E5M2 = 0, 1
F32, BF16 = 0, 1
MAX = {E4M3: 448.0, E5M2: 57344.0}

_lib = None


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        # ORACLE_LIB_PATH loads another build of the oracle source instead: the
        # pin-strength test uses it to run the pins against deliberately broken
        # copies and check that they fail.
        path = os.environ.get("ORACLE_LIB_PATH") or _build.build()
        L = ctypes.CDLL(path)
        c_i64, c_int, c_void = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        L.orc_fp8_decode.argtypes = [c_int, c_int]
        L.orc_fp8_decode.restype = ctypes.c_double
        L.orc_fp8_encode.argtypes = [ctypes.c_float, c_int]
        L.orc_fp8_encode.restype = c_int
        L.orc_fp8_top_code.argtypes = [c_int]
        L.orc_fp8_top_code.restype = c_int
        L.orc_selfcheck.argtypes = []
        L.orc_selfcheck.restype = c_int
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_amax.argtypes = [c_void, c_int, c_i64]
        L.orc_amax.restype = ctypes.c_float
        L.orc_scale_from_amax.argtypes = [ctypes.c_float, c_int]
        L.orc_scale_from_amax.restype = ctypes.c_float
        L.orc_quantize_per_tensor.argtypes = [c_void, c_int, c_i64, c_int, c_void, c_void, c_void, c_void]
        L.orc_quantize_per_tensor.restype = c_int
        L.orc_quantize_blockwise.argtypes = [c_void, c_int, c_i64, c_i64, c_int, c_int, c_int, c_void, c_void]
        L.orc_quantize_blockwise.restype = c_int
        L.orc_dequantize.argtypes = [c_void, c_int, c_i64, c_i64, c_int, c_int, c_void, c_void, c_int]
        L.orc_dequantize.restype = c_int
        L.orc_amax_history_update.argtypes = [c_void, c_void, c_int, ctypes.c_float, c_int, c_void]
        L.orc_amax_history_update.restype = c_int
        L.orc_amax_history_update_ex.argtypes = [c_void, c_void, c_int, ctypes.c_float, c_int, c_void, c_int,
                                                 ctypes.c_float, ctypes.c_float]
        L.orc_amax_history_update_ex.restype = c_int
        L.orc_quantize_per_tensor_transpose.argtypes = [c_void, c_int, c_i64, c_i64, c_int, c_void, c_void, c_void,
                                                        c_void, c_void]
        L.orc_quantize_per_tensor_transpose.restype = c_int
        L.orc_gemm_blockwise.argtypes = [c_void, c_void, c_int, c_void, c_void, c_int, c_i64, c_i64, c_i64, c_void]
        L.orc_gemm_blockwise.restype = c_int
        L.orc_gemm_blockwise_ex.argtypes = [c_void, c_void, c_int, c_void, c_void, c_int, c_int, c_i64, c_i64, c_i64,
                                            c_void]
        L.orc_gemm_blockwise_ex.restype = c_int
        L.orc_mx_exponent.argtypes = [ctypes.c_float, c_int, c_int]
        L.orc_mx_exponent.restype = c_int
        L.orc_quantize_mx.argtypes = [c_void, c_int, c_i64, c_i64, c_int, c_int, c_void, c_void]
        L.orc_quantize_mx.restype = c_int
        L.orc_dequantize_mx.argtypes = [c_void, c_int, c_i64, c_i64, c_void, c_void, c_int]
        L.orc_dequantize_mx.restype = c_int
        if L.orc_selfcheck() != 0:
            raise RuntimeError("oracle self-check failed: decoded table disagrees with the format table")
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _as_input(x: np.ndarray):
    """Return (contiguous array, dtype code) for an fp32 or bf16-bits input."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle input must be float32 or uint16 (bf16 bits), got {x.dtype}")


def _check(rc: int):
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")


# -- scalar helpers -----------------------------------------------------------

def decode(code: int, fmt: int) -> float:
    return lib().orc_fp8_decode(int(code), fmt)


def encode(v: float, fmt: int) -> int:
    return lib().orc_fp8_encode(float(v), fmt)


def top_code(fmt: int) -> int:
    return lib().orc_fp8_top_code(fmt)


def decode_table(fmt: int) -> np.ndarray:
    """float64 value of each of the 256 codes (NaN / +-Inf where the format has them)."""
    return np.array([decode(c, fmt) for c in range(256)], dtype=np.float64)


def scale_from_amax(amax: float, fmt: int) -> np.float32:
    return np.float32(lib().orc_scale_from_amax(float(amax), fmt))


def bf16_to_f32(h: int) -> float:
    return lib().orc_bf16_to_f32(int(h))


def f32_to_bf16(f: float) -> int:
    return lib().orc_f32_to_bf16(float(f))


# -- array entry points ---------------------------------------------------------

def encode_array(v: np.ndarray, fmt: int) -> np.ndarray:
    """Elementwise saturating RNE encode of an fp32 array (scale 1)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    q, s, a = quantize_per_tensor(v, fmt, scale=1.0)
    return q


def amax(x: np.ndarray) -> np.float32:
    x, dt = _as_input(x)
    return np.float32(lib().orc_amax(_ptr(x), dt, x.size))


def quantize_per_tensor(x: np.ndarray, fmt: int, scale: float | None = None):
    """Per-tensor quantize.  scale=None: current scaling; else delayed scaling with that scale.

    Returns (codes uint8 of x's shape, scale used float32, amax float32).
    """
    x, dt = _as_input(x)
    q = np.empty(x.shape, dtype=np.uint8)
    s_out = np.zeros(1, dtype=np.float32)
    a_out = np.zeros(1, dtype=np.float32)
    s_in = None if scale is None else np.array([scale], dtype=np.float32)
    _check(lib().orc_quantize_per_tensor(_ptr(x), dt, x.size, fmt,
                                         None if s_in is None else _ptr(s_in),
                                         _ptr(q), _ptr(s_out), _ptr(a_out)))
    return q, s_out[0], a_out[0]


def quantize_per_tensor_transpose(x: np.ndarray, fmt: int, scale: float | None = None):
    """Per-tensor quantize of a 2-D array with a transposed copy: (q [R, C], qt [C, R], scale, amax)."""
    x, dt = _as_input(x)
    if x.ndim != 2:
        raise ValueError("the transposing quantize takes a 2-D array")
    R, C = x.shape
    q = np.empty((R, C), dtype=np.uint8)
    qt = np.empty((C, R), dtype=np.uint8)
    s_out = np.zeros(1, dtype=np.float32)
    a_out = np.zeros(1, dtype=np.float32)
    s_in = None if scale is None else np.array([scale], dtype=np.float32)
    _check(lib().orc_quantize_per_tensor_transpose(_ptr(x), dt, R, C, fmt, None if s_in is None else _ptr(s_in),
                                                   _ptr(q), _ptr(qt), _ptr(s_out), _ptr(a_out)))
    return q, qt, s_out[0], a_out[0]


def quantize_blockwise_transpose(x: np.ndarray, br: int, bc: int, fmt: int):
    """The handbook's per_block applied to x and to x^T: (q, scales, qt, scales_t).

    The transposed operand of a weight- or data-gradient GEMM is quantized by the same rule along the
    other dimension; this is that definition written out, two calls of quantize_blockwise."""
    if np.asarray(x).ndim != 2:
        raise ValueError("the transposing blockwise quantize takes a 2-D array")
    q, s = quantize_blockwise(x, br, bc, fmt)
    qt, st = quantize_blockwise(np.ascontiguousarray(np.asarray(x).T), br, bc, fmt)
    return q, s, qt, st


def quantize_blockwise(x: np.ndarray, br: int, bc: int, fmt: int):
    """Blockwise quantize of a 2-D array.  Returns (codes, scales [ceil(R/br), ceil(C/bc)])."""
    x, dt = _as_input(x)
    if x.ndim != 2:
        raise ValueError("blockwise quantize takes a 2-D array")
    R, C = x.shape
    q = np.empty((R, C), dtype=np.uint8)
    scales = np.empty((math.ceil(R / br), math.ceil(C / bc)), dtype=np.float32)
    _check(lib().orc_quantize_blockwise(_ptr(x), dt, R, C, br, bc, fmt, _ptr(q), _ptr(scales)))
    return q, scales


def dequantize(q: np.ndarray, fmt: int, scales: np.ndarray, br: int = 0, bc: int = 0,
               out_dtype: int = F32) -> np.ndarray:
    """Dequantize codes.  br = bc = 0: one scale (scales[0]) for the whole tensor.

    out_dtype F32 returns float32, BF16 returns uint16 bf16 bits.
    """
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    if q.ndim == 1:
        R, C = 1, q.shape[0]
    elif q.ndim == 2:
        R, C = q.shape
    else:
        raise ValueError("dequantize takes a 1-D or 2-D array")
    y = np.empty(q.shape, dtype=np.float32 if out_dtype == F32 else np.uint16)
    _check(lib().orc_dequantize(_ptr(q), fmt, R, C, br, bc, _ptr(scales), _ptr(y), out_dtype))
    return y


def fake_quantize(x: np.ndarray, fmt: int, br: int = 1, bc: int = 128, scale: float | None = None):
    """Quantize -> dequantize round trip in x's dtype: the composition of the two oracle steps.

    br = bc = 0 is per tensor with the given scale.  Returns (y, scales) -- scales is the block
    scales, or the one-element scale array for per tensor."""
    x, dt = _as_input(x)
    if br == 0 and bc == 0:
        if scale is None:
            raise ValueError("per-tensor fake quantize needs a scale")
        q, s, _ = quantize_per_tensor(x, fmt, scale=scale)
        scales = np.array([s], dtype=np.float32)
    else:
        q, scales = quantize_blockwise(x if x.ndim == 2 else x.reshape(1, -1), br, bc, fmt)
    y = dequantize(q.reshape(x.shape) if x.ndim == 2 else q.reshape(1, -1), fmt, scales, br, bc, out_dtype=dt)
    return y.reshape(x.shape), scales


def gemm_blockwise(a: np.ndarray, sa: np.ndarray, a_fmt: int, b: np.ndarray, sb: np.ndarray, b_fmt: int,
                   b_block: int = 128):
    """C [M, N] (float64) = sum over 128-wide K chunks of (dec(a) dec(b)^T) / (sa * sb).

    b_block 128: B in 128x128 blocks, sb [ceil(N/128), ceil(K/128)]; b_block 1: B in 1x128 blocks along K
    (the weight-gradient operand), sb [N, ceil(K/128)]."""
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    M, K = a.shape
    N = b.shape[0]
    nkc = math.ceil(K / 128)
    if b_block not in (1, 128):
        raise ValueError("gemm_blockwise: b_block is 1 or 128")
    if b.shape[1] != K or sa.shape != (M, nkc) or sb.shape != (math.ceil(N / b_block), nkc):
        raise ValueError("gemm_blockwise: inconsistent shapes")
    c = np.empty((M, N), dtype=np.float64)
    _check(lib().orc_gemm_blockwise_ex(_ptr(a), _ptr(sa), a_fmt, _ptr(b), _ptr(sb), b_block, b_fmt, M, N, K,
                                       _ptr(c)))
    return c


MX_FIT, MX_OCP = 0, 1


def mx_exponent(amax: float, fmt: int, rule: int = MX_FIT) -> int:
    """k of the power-of-two scale 2^k of an MX block with this amax."""
    return lib().orc_mx_exponent(float(amax), fmt, rule)


def quantize_mx(x: np.ndarray, fmt: int, rule: int = MX_FIT):
    """MX quantize of a 2-D array: (codes, e8m0 [R, ceil(C/32)] uint8)."""
    x, dt = _as_input(x)
    if x.ndim != 2:
        raise ValueError("MX quantize takes a 2-D array")
    R, C = x.shape
    q = np.empty((R, C), dtype=np.uint8)
    e = np.empty((R, math.ceil(C / 32)), dtype=np.uint8)
    _check(lib().orc_quantize_mx(_ptr(x), dt, R, C, fmt, rule, _ptr(q), _ptr(e)))
    return q, e


def dequantize_mx(q: np.ndarray, fmt: int, e8m0: np.ndarray, out_dtype: int = F32) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    e8m0 = np.ascontiguousarray(e8m0, dtype=np.uint8)
    R, C = q.shape
    y = np.empty(q.shape, dtype=np.float32 if out_dtype == F32 else np.uint16)
    _check(lib().orc_dequantize_mx(_ptr(q), fmt, R, C, _ptr(e8m0), _ptr(y), out_dtype))
    return y


WINDOW_MAX, EMA = 0, 1


class AmaxHistory:
    """Delayed-scaling state: a window of past amax values (or their moving average) and the scale.

    algo WINDOW_MAX with margin 1.0 is the plain window of the PyTorch-FP8 page's DelayedScaler;
    margin and EMA are its s4.3 refinements."""

    def __init__(self, window: int, fmt: int, algo: int = WINDOW_MAX, alpha: float = 1.0, margin: float = 1.0):
        self.window = window
        self.fmt = fmt
        self.algo = algo
        self.alpha = alpha
        self.margin = margin
        self.history = np.zeros(window, dtype=np.float32)
        self.state = np.zeros(2, dtype=np.int32)
        self.scale = np.ones(1, dtype=np.float32)

    def update(self, amax_value: float) -> np.float32:
        if self.algo == WINDOW_MAX and self.margin == 1.0:
            _check(lib().orc_amax_history_update(_ptr(self.history), _ptr(self.state), self.window,
                                                 float(amax_value), self.fmt, _ptr(self.scale)))
        else:
            _check(lib().orc_amax_history_update_ex(_ptr(self.history), _ptr(self.state), self.window,
                                                    float(amax_value), self.fmt, _ptr(self.scale), self.algo,
                                                    float(self.alpha), float(self.margin)))
        return self.scale[0]
