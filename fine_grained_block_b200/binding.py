"""ctypes binding of ``libfp8q.so`` -- argument marshalling only.

Two layers with the C names:

* ``lib()`` returns the loaded ``ctypes.CDLL`` whose functions take the exact
  C arguments (device pointers as ints, sizes, enums, a stream handle).
* ``fp8_quantize_per_tensor``, ``fp8_quantize_blockwise``, ``fp8_dequantize``,
  ``fp8_quantize_mx``, ``fp8_dequantize_mx``, ``fp8_amax_history_update`` and
  the other wrappers below take torch CUDA tensors, allocate any
  output the caller did not pass (``torch.empty`` on the input's device), pass
  pointers and the current stream to the C function, and raise ``FP8Error`` on
  a nonzero status.  All computation happens in the library's kernels; there
  is no CPU fallback, and a missing library raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

E4M3, E5M2 = 0, 1
F32, BF16 = 0, 1

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp8q.so")
_lib = None

class FP8BlockTensor(ctypes.Structure):
    """struct fp8_block_tensor of include/fp8q.h."""
    _fields_ = [("x", ctypes.c_void_p), ("q", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class FP8CurrentTensor(ctypes.Structure):
    """struct fp8_current_tensor of include/fp8q.h."""
    _fields_ = [("x", ctypes.c_void_p), ("q", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("scale_out", ctypes.c_void_p), ("amax_out", ctypes.c_void_p)]


class FP8DelayedTensor(ctypes.Structure):
    """struct fp8_delayed_tensor of include/fp8q.h."""
    _fields_ = [("x", ctypes.c_void_p), ("q", ctypes.c_void_p), ("n", ctypes.c_int64), ("scale", ctypes.c_void_p),
                ("history", ctypes.c_void_p), ("state", ctypes.c_void_p), ("scale_used", ctypes.c_void_p),
                ("amax_out", ctypes.c_void_p)]


# Declared in include/fp8q.h: name -> (restype, argtypes)
_c_int, _i64, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
SIGNATURES = {
    "fp8_quantize_per_tensor": (_c_int, [_vp, _c_int, _i64, _c_int, _vp, _vp, _vp, _vp, _vp]),
    "fp8_quantize_blockwise": (_c_int, [_vp, _c_int, _i64, _i64, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "fp8_dequantize": (_c_int, [_vp, _c_int, _i64, _i64, _c_int, _c_int, _vp, _vp, _c_int, _vp]),
    "fp8_amax_history_update": (_c_int, [_vp, _vp, _c_int, _vp, _c_int, _vp, _vp]),
    "fp8_amax_history_update_ex": (_c_int, [_vp, _vp, _c_int, _vp, _c_int, _vp, _c_int, ctypes.c_float,
                                            ctypes.c_float, _vp]),
    "fp8_quantize_per_tensor_fused": (_c_int, [_vp, _c_int, _i64, _c_int, _vp, _vp, _vp, _vp, _vp]),
    "fp8_quantize_per_tensor_fused_noalloc": (_c_int, [_vp, _c_int, _i64, _c_int, _vp, _vp, _vp, _vp]),
    "fp8_amax": (_c_int, [_vp, _c_int, _i64, _vp, _vp]),
    "fp8_scale_from_amax": (_c_int, [_vp, _c_int, _vp, _vp]),
    "fp8_fake_quantize": (_c_int, [_vp, _c_int, _i64, _i64, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp]),
    "fp8_quantize_per_tensor_transpose": (_c_int, [_vp, _c_int, _i64, _i64, _c_int, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fp8_gemm_blockwise_ex": (_c_int, [_vp, _vp, _c_int, _vp, _vp, _c_int, _c_int, _i64, _i64, _i64, _vp, _c_int,
                                       _vp]),
    "fp8_quantize_blockwise_transpose": (_c_int, [_vp, _c_int, _i64, _i64, _c_int, _c_int, _c_int, _vp, _vp, _vp,
                                                  _vp, _vp]),
    "fp8_quantize_mx": (_c_int, [_vp, _c_int, _i64, _i64, _c_int, _c_int, _vp, _vp, _vp]),
    "fp8_dequantize_mx": (_c_int, [_vp, _c_int, _i64, _i64, _vp, _vp, _c_int, _vp]),
    "fp8_gemm_blockwise": (_c_int, [_vp, _vp, _c_int, _vp, _vp, _c_int, _i64, _i64, _i64, _vp, _c_int, _vp]),
    "fp8_quantize_delayed_step": (_c_int, [_vp, _c_int, _i64, _c_int, _vp, _vp, _vp, _c_int, _c_int, ctypes.c_float,
                                           ctypes.c_float, _vp, _vp, _vp, _vp, _vp]),
    "fp8_quantize_blockwise_grouped": (_c_int, [ctypes.POINTER(FP8BlockTensor), _c_int, _c_int, _c_int, _c_int,
                                                _c_int, _vp]),
    "fp8_quantize_delayed_step_grouped": (_c_int, [ctypes.POINTER(FP8DelayedTensor), _c_int, _c_int, _c_int, _c_int,
                                                   _c_int, ctypes.c_float, ctypes.c_float, _vp, _vp]),
    "fp8_quantize_per_tensor_grouped": (_c_int, [ctypes.POINTER(FP8CurrentTensor), _c_int, _c_int, _c_int, _vp]),
    "fp8_status_string": (ctypes.c_char_p, [_c_int]),
    "fp8_device_status": (_c_int, [_vp, _c_int, _vp]),
    "fp8_selftest_wait_timeout": (_c_int, [ctypes.c_uint32, _vp]),
}
DEVICE_STATUS_WAIT_TIMEOUT = 0x1
AMAX_WINDOW_MAX, AMAX_EMA = 0, 1
MX_FIT, MX_OCP = 0, 1
FUSED_WORKSPACE_BYTES = 16


class FP8Error(RuntimeError):
    """A libfp8q call returned an error status."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({fp8_status_string(status)})")


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libfp8q.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"{p} is missing: build it with `python -m fine_grained_block_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = L
    return L


lib = load_library


def fp8_status_string(status: int) -> str:
    return load_library().fp8_status_string(int(status)).decode()


# -- marshalling helpers ----------------------------------------------------------

_DTYPE_CODE = {torch.float32: F32, torch.bfloat16: BF16}


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libfp8q works on CUDA tensors only")
        if t is not None and not t.is_contiguous():
            raise ValueError("libfp8q needs contiguous tensors")


def _check(fn: str, status: int):
    if status != 0:
        raise FP8Error(fn, status)


# -- entry points -------------------------------------------------------------------

def fp8_quantize_per_tensor(x: torch.Tensor, fmt: int = E4M3, scale_in: torch.Tensor | None = None,
                            q: torch.Tensor | None = None, scale_out: torch.Tensor | None = None,
                            amax_out: torch.Tensor | None = None, want_amax: bool = True, stream=None):
    """Per-tensor quantize.  scale_in None = current scaling, else delayed (a 1-element fp32 CUDA tensor).

    Returns (q uint8 like x, scale_out [1] fp32, amax_out [1] fp32 or None)."""
    _need_cuda(x, scale_in, q, scale_out, amax_out)
    dev = x.device
    q = torch.empty(x.shape, dtype=torch.uint8, device=dev) if q is None else q
    scale_out = torch.empty(1, dtype=torch.float32, device=dev) if scale_out is None else scale_out
    if amax_out is None and (want_amax or scale_in is None):
        amax_out = torch.empty(1, dtype=torch.float32, device=dev)
    st = load_library().fp8_quantize_per_tensor(_ptr(x), _DTYPE_CODE[x.dtype], x.numel(), fmt, _ptr(scale_in),
                                                _ptr(q), _ptr(scale_out), _ptr(amax_out), _stream(stream))
    _check("fp8_quantize_per_tensor", st)
    return q, scale_out, amax_out


def fp8_quantize_per_tensor_transpose(x: torch.Tensor, fmt: int = E4M3, scale_in: torch.Tensor | None = None,
                                      with_q: bool = True, q: torch.Tensor | None = None,
                                      qt: torch.Tensor | None = None, scale_out: torch.Tensor | None = None,
                                      amax_out: torch.Tensor | None = None, stream=None):
    """Per-tensor quantize of a 2-D tensor with a transposed copy.  Returns (q or None, qt [C, R], scale, amax)."""
    _need_cuda(x, scale_in, q, qt, scale_out, amax_out)
    if x.dim() != 2:
        raise ValueError("the transposing quantize takes a 2-D tensor")
    R, C = x.shape
    dev = x.device
    if q is None and with_q:
        q = torch.empty((R, C), dtype=torch.uint8, device=dev)
    qt = torch.empty((C, R), dtype=torch.uint8, device=dev) if qt is None else qt
    scale_out = torch.empty(1, dtype=torch.float32, device=dev) if scale_out is None else scale_out
    amax_out = torch.empty(1, dtype=torch.float32, device=dev) if amax_out is None else amax_out
    st = load_library().fp8_quantize_per_tensor_transpose(_ptr(x), _DTYPE_CODE[x.dtype], R, C, fmt, _ptr(scale_in),
                                                          _ptr(q), _ptr(qt), _ptr(scale_out), _ptr(amax_out),
                                                          _stream(stream))
    _check("fp8_quantize_per_tensor_transpose", st)
    return q, qt, scale_out, amax_out


def fused_workspace(device="cuda") -> torch.Tensor:
    """A zeroed workspace for fp8_quantize_per_tensor_fused (one per stream)."""
    return torch.zeros(FUSED_WORKSPACE_BYTES // 4, dtype=torch.int32, device=device)


def fp8_quantize_per_tensor_fused(x: torch.Tensor, fmt: int = E4M3, workspace: torch.Tensor | None = None,
                                  q: torch.Tensor | None = None, scale_out: torch.Tensor | None = None,
                                  amax_out: torch.Tensor | None = None, stream=None):
    """Per-tensor current scaling in one pass when x fits on chip (else the two-pass path).

    Returns (q, scale_out [1], amax_out [1])."""
    _need_cuda(x, workspace, q, scale_out, amax_out)
    dev = x.device
    workspace = fused_workspace(dev) if workspace is None else workspace
    q = torch.empty(x.shape, dtype=torch.uint8, device=dev) if q is None else q
    scale_out = torch.empty(1, dtype=torch.float32, device=dev) if scale_out is None else scale_out
    amax_out = torch.empty(1, dtype=torch.float32, device=dev) if amax_out is None else amax_out
    st = load_library().fp8_quantize_per_tensor_fused(_ptr(x), _DTYPE_CODE[x.dtype], x.numel(), fmt, _ptr(q),
                                                      _ptr(scale_out), _ptr(amax_out), _ptr(workspace),
                                                      _stream(stream))
    _check("fp8_quantize_per_tensor_fused", st)
    return q, scale_out, amax_out


def fp8_amax(x: torch.Tensor, amax_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """max |x| into a 1-element fp32 CUDA tensor."""
    _need_cuda(x, amax_out)
    amax_out = torch.empty(1, dtype=torch.float32, device=x.device) if amax_out is None else amax_out
    _check("fp8_amax", load_library().fp8_amax(_ptr(x), _DTYPE_CODE[x.dtype], x.numel(), _ptr(amax_out),
                                               _stream(stream)))
    return amax_out


def fp8_scale_from_amax(amax: torch.Tensor, fmt: int = E4M3, scale_out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """MAX / max(amax, 1e-12) into a 1-element fp32 CUDA tensor."""
    _need_cuda(amax, scale_out)
    scale_out = torch.empty(1, dtype=torch.float32, device=amax.device) if scale_out is None else scale_out
    _check("fp8_scale_from_amax", load_library().fp8_scale_from_amax(_ptr(amax), fmt, _ptr(scale_out),
                                                                     _stream(stream)))
    return scale_out


def fp8_quantize_blockwise(x: torch.Tensor, block=(1, 128), fmt: int = E4M3, q: torch.Tensor | None = None,
                           scales: torch.Tensor | None = None, stream=None):
    """Blockwise quantize of a 2-D tensor with (1, 128) or (128, 128) blocks.  Returns (q, scales)."""
    _need_cuda(x, q, scales)
    if x.dim() != 2:
        raise ValueError("blockwise quantize takes a 2-D tensor")
    R, C = x.shape
    br, bc = block
    q = torch.empty((R, C), dtype=torch.uint8, device=x.device) if q is None else q
    if scales is None:
        scales = torch.empty((math.ceil(R / br), math.ceil(C / bc)), dtype=torch.float32, device=x.device)
    st = load_library().fp8_quantize_blockwise(_ptr(x), _DTYPE_CODE[x.dtype], R, C, br, bc, fmt, _ptr(q),
                                               _ptr(scales), _stream(stream))
    _check("fp8_quantize_blockwise", st)
    return q, scales


def fp8_quantize_blockwise_grouped(xs, block=(1, 128), fmt: int = E4M3, qs=None, scales=None, stream=None):
    """Blockwise quantize of several 2-D tensors (same dtype, cols % 128 == 0) in as few launches as possible.

    Returns (list of q, list of scales)."""
    xs = list(xs)
    if not xs:
        return [], []
    dt = xs[0].dtype
    br, bc = block
    qs = [torch.empty(x.shape, dtype=torch.uint8, device=x.device) for x in xs] if qs is None else list(qs)
    if scales is None:
        scales = [torch.empty((math.ceil(x.shape[0] / br), math.ceil(x.shape[1] / bc)), dtype=torch.float32,
                              device=x.device) for x in xs]
    arr = (FP8BlockTensor * len(xs))()
    for i, (x, q, s_) in enumerate(zip(xs, qs, scales)):
        _need_cuda(x, q, s_)
        if x.dim() != 2 or x.dtype != dt:
            raise ValueError("grouped quantize takes 2-D tensors of one dtype")
        arr[i] = FP8BlockTensor(_ptr(x), _ptr(q), _ptr(s_), x.shape[0], x.shape[1])
    st = load_library().fp8_quantize_blockwise_grouped(arr, len(xs), _DTYPE_CODE[dt], br, bc, fmt, _stream(stream))
    _check("fp8_quantize_blockwise_grouped", st)
    return qs, scales


def fp8_quantize_blockwise_transpose(x: torch.Tensor, block=(1, 128), fmt: int = E4M3, q=None, scales=None,
                                     qt=None, scales_t=None, stream=None):
    """Blockwise quantize of x and of x^T in one pass (rows, cols multiples of 128).

    Returns (q, scales, qt, scales_t) = fp8_quantize_blockwise(x, block) + fp8_quantize_blockwise(x.T, block)."""
    _need_cuda(x, q, scales, qt, scales_t)
    if x.dim() != 2:
        raise ValueError("the transposing blockwise quantize takes a 2-D tensor")
    R, C = x.shape
    br, bc = block
    dev = x.device
    q = torch.empty((R, C), dtype=torch.uint8, device=dev) if q is None else q
    qt = torch.empty((C, R), dtype=torch.uint8, device=dev) if qt is None else qt
    if scales is None:
        scales = torch.empty((R // br, C // bc), dtype=torch.float32, device=dev)
    if scales_t is None:
        scales_t = torch.empty((C // br, R // bc), dtype=torch.float32, device=dev)
    st = load_library().fp8_quantize_blockwise_transpose(_ptr(x), _DTYPE_CODE[x.dtype], R, C, br, bc, fmt, _ptr(q),
                                                         _ptr(scales), _ptr(qt), _ptr(scales_t), _stream(stream))
    _check("fp8_quantize_blockwise_transpose", st)
    return q, scales, qt, scales_t


def fp8_quantize_mx(x: torch.Tensor, fmt: int = E4M3, rule: int = MX_FIT, q: torch.Tensor | None = None,
                    e8m0: torch.Tensor | None = None, stream=None):
    """MX quantize of a 2-D tensor: 1x32 blocks, power-of-two scales.  Returns (q, e8m0 uint8 [R, ceil(C/32)])."""
    _need_cuda(x, q, e8m0)
    if x.dim() != 2:
        raise ValueError("MX quantize takes a 2-D tensor")
    R, C = x.shape
    q = torch.empty((R, C), dtype=torch.uint8, device=x.device) if q is None else q
    if e8m0 is None:
        e8m0 = torch.empty((R, math.ceil(C / 32)), dtype=torch.uint8, device=x.device)
    st = load_library().fp8_quantize_mx(_ptr(x), _DTYPE_CODE[x.dtype], R, C, fmt, rule, _ptr(q), _ptr(e8m0),
                                        _stream(stream))
    _check("fp8_quantize_mx", st)
    return q, e8m0


def fp8_dequantize_mx(q: torch.Tensor, e8m0: torch.Tensor, fmt: int = E4M3, out_dtype=torch.float32,
                      y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """MX dequantize: y = decode(q) * 2^(e8m0 - 127) per 1x32 block."""
    _need_cuda(q, e8m0, y)
    if q.dim() != 2:
        raise ValueError("MX dequantize takes a 2-D tensor")
    R, C = q.shape
    y = torch.empty((R, C), dtype=out_dtype, device=q.device) if y is None else y
    st = load_library().fp8_dequantize_mx(_ptr(q), fmt, R, C, _ptr(e8m0), _ptr(y), _DTYPE_CODE[y.dtype],
                                          _stream(stream))
    _check("fp8_dequantize_mx", st)
    return y


def fp8_gemm_blockwise(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor, sb: torch.Tensor, a_fmt: int = E4M3,
                       b_fmt: int = E4M3, out_dtype=torch.bfloat16, c: torch.Tensor | None = None,
                       stream=None, b_block: int = 128) -> torch.Tensor:
    """C [M, N] = A [M, K] (1x128 scales sa) x B [N, K]^T, FP8 tensor cores.

    b_block 128: B with 128x128 scales sb [N/128, K/128] (fp8_gemm_blockwise); b_block 1: B with 1x128
    scales sb [N, K/128], the weight-gradient form (fp8_gemm_blockwise_ex)."""
    _need_cuda(a, sa, b, sb, c)
    if a.dim() != 2 or b.dim() != 2 or a.shape[1] != b.shape[1]:
        raise ValueError("fp8_gemm_blockwise takes a [M, K] and b [N, K]")
    M, K = a.shape
    N = b.shape[0]
    c = torch.empty((M, N), dtype=out_dtype, device=a.device) if c is None else c
    if b_block == 128:
        st = load_library().fp8_gemm_blockwise(_ptr(a), _ptr(sa), a_fmt, _ptr(b), _ptr(sb), b_fmt, M, N, K, _ptr(c),
                                               _DTYPE_CODE[c.dtype], _stream(stream))
        _check("fp8_gemm_blockwise", st)
    else:
        st = load_library().fp8_gemm_blockwise_ex(_ptr(a), _ptr(sa), a_fmt, _ptr(b), _ptr(sb), b_block, b_fmt, M, N,
                                                  K, _ptr(c), _DTYPE_CODE[c.dtype], _stream(stream))
        _check("fp8_gemm_blockwise_ex", st)
    return c


def fp8_dequantize(q: torch.Tensor, scales: torch.Tensor, block=(0, 0), fmt: int = E4M3,
                   out_dtype=torch.bfloat16, y: torch.Tensor | None = None, stream=None):
    """Dequantize codes; block (0, 0) = per-tensor (scales[0]).  Returns y."""
    _need_cuda(q, scales, y)
    if q.dim() == 1:
        R, C = 1, q.shape[0]
    elif q.dim() == 2:
        R, C = q.shape
    else:
        raise ValueError("dequantize takes a 1-D or 2-D tensor")
    y = torch.empty(q.shape, dtype=out_dtype, device=q.device) if y is None else y
    st = load_library().fp8_dequantize(_ptr(q), fmt, R, C, block[0], block[1], _ptr(scales), _ptr(y),
                                       _DTYPE_CODE[y.dtype], _stream(stream))
    _check("fp8_dequantize", st)
    return y


def fp8_fake_quantize(x: torch.Tensor, block=(1, 128), fmt: int = E4M3, scale_in: torch.Tensor | None = None,
                      y: torch.Tensor | None = None, scales_out: torch.Tensor | None = None, stream=None):
    """Quantize -> dequantize round trip in x's dtype (block (0, 0) = per tensor with scale_in).  Returns y."""
    _need_cuda(x, scale_in, y, scales_out)
    if x.dim() == 1:
        R, C = 1, x.shape[0]
    elif x.dim() == 2:
        R, C = x.shape
    else:
        raise ValueError("fake quantize takes a 1-D or 2-D tensor")
    y = torch.empty_like(x) if y is None else y
    st = load_library().fp8_fake_quantize(_ptr(x), _DTYPE_CODE[x.dtype], R, C, block[0], block[1], fmt,
                                          _ptr(scale_in), _ptr(y), _ptr(scales_out), _stream(stream))
    _check("fp8_fake_quantize", st)
    return y


def fp8_amax_history_update(history: torch.Tensor, state: torch.Tensor, amax: torch.Tensor, scale: torch.Tensor,
                            fmt: int = E4M3, stream=None):
    """Push amax into the history ring and refresh scale in place (all 4 are CUDA tensors)."""
    _need_cuda(history, state, amax, scale)
    st = load_library().fp8_amax_history_update(_ptr(history), _ptr(state), history.numel(), _ptr(amax), fmt,
                                                _ptr(scale), _stream(stream))
    _check("fp8_amax_history_update", st)
    return scale


def fp8_device_status(clear: bool = False, device=None, stream=None) -> int:
    """The device status word (FP8_DEVICE_STATUS_* bits); synchronizes the stream to read it."""
    out = torch.zeros(1, dtype=torch.int32, device=device or "cuda")
    _check("fp8_device_status", load_library().fp8_device_status(_ptr(out), 1 if clear else 0, _stream(stream)))
    return int(out.item())


def fp8_selftest_wait_timeout(timeout_us: int = 1000, stream=None):
    """Launch a wait that can only time out (sets DEVICE_STATUS_WAIT_TIMEOUT after timeout_us)."""
    _check("fp8_selftest_wait_timeout", load_library().fp8_selftest_wait_timeout(int(timeout_us), _stream(stream)))


def fp8_amax_history_update_ex(history: torch.Tensor, state: torch.Tensor, amax: torch.Tensor, scale: torch.Tensor,
                               fmt: int = E4M3, algo: int = AMAX_WINDOW_MAX, alpha: float = 1.0,
                               margin: float = 1.0, stream=None):
    """Delayed-scaling update with a margin and window-max or EMA smoothing (PyTorch-FP8 page s4.3)."""
    _need_cuda(history, state, amax, scale)
    st = load_library().fp8_amax_history_update_ex(_ptr(history), _ptr(state), history.numel(), _ptr(amax), fmt,
                                                   _ptr(scale), algo, float(alpha), float(margin), _stream(stream))
    _check("fp8_amax_history_update_ex", st)
    return scale


def fp8_quantize_delayed_step(x: torch.Tensor, scale: torch.Tensor, history: torch.Tensor, state: torch.Tensor,
                              fmt: int = E5M2, algo: int = AMAX_WINDOW_MAX, alpha: float = 1.0, margin: float = 1.0,
                              q: torch.Tensor | None = None, scale_used: torch.Tensor | None = None,
                              amax_out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                              stream=None) -> torch.Tensor:
    """Cast x with *scale, then (same launch) push amax(x) into the history and rewrite *scale."""
    _need_cuda(x, scale, history, state, q, scale_used, amax_out, workspace)
    dev = x.device
    q = torch.empty(x.shape, dtype=torch.uint8, device=dev) if q is None else q
    scale_used = torch.empty(1, dtype=torch.float32, device=dev) if scale_used is None else scale_used
    amax_out = torch.empty(1, dtype=torch.float32, device=dev) if amax_out is None else amax_out
    workspace = fused_workspace(dev) if workspace is None else workspace
    st = load_library().fp8_quantize_delayed_step(_ptr(x), _DTYPE_CODE[x.dtype], x.numel(), fmt, _ptr(scale),
                                                  _ptr(history), _ptr(state), history.numel(), algo, alpha, margin,
                                                  _ptr(q), _ptr(scale_used), _ptr(amax_out), _ptr(workspace),
                                                  _stream(stream))
    _check("fp8_quantize_delayed_step", st)
    return q


def fp8_quantize_delayed_step_grouped(xs, scalers, qs=None, workspace: torch.Tensor | None = None, stream=None):
    """One delayed-scaling step for several tensors in as few launches as possible.

    scalers: one DelayedScaler per tensor (same fmt, window, algo, alpha and margin); each is stepped as
    scaler.step(x) would step it.  Returns the list of codes."""
    xs, scalers = list(xs), list(scalers)
    if len(xs) != len(scalers):
        raise ValueError("one scaler per tensor")
    if not xs:
        return []
    s0 = scalers[0]
    if any((s.fmt, s.history.numel(), s.algo, s.alpha, s.margin) !=
           (s0.fmt, s0.history.numel(), s0.algo, s0.alpha, s0.margin) for s in scalers):
        raise ValueError("grouped scalers must share fmt, window, algo, alpha and margin")
    dt = xs[0].dtype
    qs = [torch.empty(x.shape, dtype=torch.uint8, device=x.device) for x in xs] if qs is None else list(qs)
    if workspace is None:
        workspace = torch.zeros(len(xs) * FUSED_WORKSPACE_BYTES // 4, dtype=torch.int32, device=xs[0].device)
    arr = (FP8DelayedTensor * len(xs))()
    for i, (x, q, sc) in enumerate(zip(xs, qs, scalers)):
        _need_cuda(x, q)
        if x.dtype != dt:
            raise ValueError("grouped tensors must share one dtype")
        arr[i] = FP8DelayedTensor(_ptr(x), _ptr(q), x.numel(), _ptr(sc.scale), _ptr(sc.history), _ptr(sc.state),
                                  _ptr(sc.scale_used), _ptr(sc.amax))
    st = load_library().fp8_quantize_delayed_step_grouped(arr, len(xs), _DTYPE_CODE[dt], s0.fmt, s0.history.numel(),
                                                          s0.algo, s0.alpha, s0.margin, _ptr(workspace),
                                                          _stream(stream))
    _check("fp8_quantize_delayed_step_grouped", st)
    return qs


def fp8_quantize_per_tensor_grouped(xs, fmt: int = E4M3, qs=None, scales=None, amaxes=None, stream=None):
    """Per-tensor current scaling of several tensors in three launches per 128 tensors: each tensor gets
    its own amax and scale, exactly as from fp8_quantize_per_tensor(x, fmt).  Returns (codes, scales, amaxes),
    lists of CUDA tensors (codes in each x's shape, scales and amaxes of one element)."""
    xs = list(xs)
    if not xs:
        return [], [], []
    dt = xs[0].dtype
    dev = xs[0].device
    qs = [torch.empty(x.shape, dtype=torch.uint8, device=x.device) for x in xs] if qs is None else list(qs)
    scales = [torch.empty(1, dtype=torch.float32, device=dev) for _ in xs] if scales is None else list(scales)
    amaxes = [torch.empty(1, dtype=torch.float32, device=dev) for _ in xs] if amaxes is None else list(amaxes)
    arr = (FP8CurrentTensor * len(xs))()
    for i, (x, q, s_, a_) in enumerate(zip(xs, qs, scales, amaxes)):
        _need_cuda(x, q, s_, a_)
        if x.dtype != dt:
            raise ValueError("grouped tensors must share one dtype")
        arr[i] = FP8CurrentTensor(_ptr(x), _ptr(q), x.numel(), _ptr(s_), _ptr(a_))
    st = load_library().fp8_quantize_per_tensor_grouped(arr, len(xs), _DTYPE_CODE[dt], fmt, _stream(stream))
    _check("fp8_quantize_per_tensor_grouped", st)
    return qs, scales, amaxes


class DelayedScaler:
    """Device-resident delayed-scaling state (history ring, {pos, count}, scale), after the
    PyTorch-FP8 page's DelayedScaler (s4.2).  step(x) quantizes x with the current scale, then
    pushes amax(x) into the history -- all on the device, no host round trip.  fused=True (the
    default) does both in one launch (fp8_quantize_delayed_step); fused=False uses the two calls."""

    def __init__(self, window: int = 16, fmt: int = E5M2, device="cuda", algo: int = AMAX_WINDOW_MAX,
                 alpha: float = 1.0, margin: float = 1.0, fused: bool = True):
        self.fmt = fmt
        self.fused = fused
        self.workspace = fused_workspace(device) if fused else None
        self.algo, self.alpha, self.margin = algo, alpha, margin
        self.history = torch.zeros(window, dtype=torch.float32, device=device)
        self.state = torch.zeros(2, dtype=torch.int32, device=device)
        self.scale = torch.ones(1, dtype=torch.float32, device=device)
        self.amax = torch.zeros(1, dtype=torch.float32, device=device)
        self.scale_used = torch.ones(1, dtype=torch.float32, device=device)

    def step(self, x: torch.Tensor, q: torch.Tensor | None = None, stream=None):
        if self.fused:
            q = fp8_quantize_delayed_step(x, self.scale, self.history, self.state, self.fmt, self.algo, self.alpha,
                                          self.margin, q=q, scale_used=self.scale_used, amax_out=self.amax,
                                          workspace=self.workspace, stream=stream)
            return q, self.scale_used
        q, s, _ = fp8_quantize_per_tensor(x, self.fmt, scale_in=self.scale, q=q, scale_out=self.scale_used,
                                          amax_out=self.amax, stream=stream)
        if self.algo == AMAX_WINDOW_MAX and self.margin == 1.0:
            fp8_amax_history_update(self.history, self.state, self.amax, self.scale, self.fmt, stream=stream)
        else:
            fp8_amax_history_update_ex(self.history, self.state, self.amax, self.scale, self.fmt, self.algo,
                                       self.alpha, self.margin, stream=stream)
        return q, self.scale_used
