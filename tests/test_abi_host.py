"""The C-ABI library loads, exports every function include/fp8q.h declares, and
rejects bad arguments on the host before touching CUDA.  No compute runs here:
these calls return before any kernel launch, so they work without a GPU."""
import ctypes
import os
import re

import pytest

from fine_grained_block_b200 import build as fbuild
from fine_grained_block_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")

OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_FORMAT, ERR_DTYPE, ERR_CUDA, ERR_ARG = 0, -1, -2, -3, -4, -5, -6, -7


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fp8_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return binding.load_library()


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(["fp8_quantize_per_tensor", "fp8_quantize_blockwise", "fp8_dequantize",
                                           "fp8_amax_history_update", "fp8_status_string", "fp8_device_status",
                                           "fp8_fake_quantize", "fp8_amax", "fp8_scale_from_amax",
                                           "fp8_quantize_per_tensor_fused",
                                           "fp8_quantize_per_tensor_fused_noalloc", "fp8_amax_history_update_ex",
                                           "fp8_selftest_wait_timeout", "fp8_quantize_mx", "fp8_dequantize_mx",
                                           "fp8_quantize_per_tensor_transpose", "fp8_gemm_blockwise",
                                           "fp8_quantize_delayed_step", "fp8_quantize_blockwise_grouped",
                                           "fp8_quantize_delayed_step_grouped", "fp8_quantize_per_tensor_grouped",
                                           "fp8_quantize_blockwise_transpose", "fp8_gemm_blockwise_ex"])


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in binding.SIGNATURES
    assert set(binding.SIGNATURES) == set(declared_functions())


def test_exported_symbols_are_c_linkage():
    out = os.popen(f"nm -D --defined-only {binding.LIB_PATH}").read()
    exported = set(re.findall(r" T (fp8_\w+)$", out, flags=re.M))
    assert exported == set(declared_functions())


def test_status_strings(L):
    for st in (OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_FORMAT, ERR_DTYPE, ERR_CUDA, ERR_ARG):
        s = binding.fp8_status_string(st)
        assert s and s != "unknown status"
    assert binding.fp8_status_string(12345) == "unknown status"


# Fake (never dereferenced) device addresses: validation rejects before any use.
A16 = 0x7F0000000000
A4 = A16 + 4
A1 = A16 + 1


def test_blockwise_validation(L):
    f = L.fp8_quantize_blockwise
    assert f(A16, 1, 4, 256, 1, 128, 7, A16, A16, None) == ERR_FORMAT
    assert f(A16, 3, 4, 256, 1, 128, 0, A16, A16, None) == ERR_DTYPE
    assert f(A16, 1, -1, 256, 1, 128, 0, A16, A16, None) == ERR_SHAPE
    assert f(A16, 1, 4, 256, 2, 128, 0, A16, A16, None) == ERR_SHAPE
    assert f(A16, 1, 4, 256, 1, 64, 0, A16, A16, None) == ERR_SHAPE
    assert f(A16, 1, 4, 256, 128, 256, 0, A16, A16, None) == ERR_SHAPE
    assert f(None, 1, 4, 256, 1, 128, 0, A16, A16, None) == ERR_NULL
    assert f(A16, 1, 4, 256, 1, 128, 0, None, A16, None) == ERR_NULL
    assert f(A16, 1, 4, 256, 1, 128, 0, A16, None, None) == ERR_NULL
    assert f(A1, 1, 4, 256, 1, 128, 0, A16, A16, None) == ERR_ALIGN
    assert f(A16, 1, 4, 256, 1, 128, 0, A4, A16, None) == ERR_ALIGN
    assert f(A16, 1, 4, 256, 1, 128, 0, A16, A1, None) == ERR_ALIGN
    assert f(A16, 1, 1 << 62, 1 << 62, 1, 128, 0, A16, A16, None) == ERR_SHAPE
    # empty tensors: nothing to do, nothing launched, null pointers allowed
    assert f(None, 1, 0, 256, 1, 128, 0, None, None, None) == OK
    assert f(None, 1, 4, 0, 128, 128, 0, None, None, None) == OK


def test_dequant_validation(L):
    f = L.fp8_dequantize
    assert f(A16, 2, 4, 256, 1, 128, A16, A16, 1, None) == ERR_FORMAT
    assert f(A16, 0, 4, 256, 1, 128, A16, A16, 2, None) == ERR_DTYPE
    assert f(A16, 0, 4, 256, 1, 64, A16, A16, 1, None) == ERR_SHAPE
    assert f(A16, 0, 4, 256, 0, 128, A16, A16, 1, None) == ERR_SHAPE
    assert f(A16, 0, -4, 256, 0, 0, A16, A16, 1, None) == ERR_SHAPE
    assert f(None, 0, 4, 256, 0, 0, A16, A16, 1, None) == ERR_NULL
    assert f(A16, 0, 4, 256, 0, 0, None, A16, 1, None) == ERR_NULL
    assert f(A16, 0, 4, 256, 0, 0, A16, None, 1, None) == ERR_NULL
    assert f(A4, 0, 4, 256, 0, 0, A16, A16, 1, None) == ERR_ALIGN
    assert f(A16, 0, 4, 256, 0, 0, A16, A4, 1, None) == ERR_ALIGN
    assert f(A16, 0, 4, 256, 0, 0, A1, A16, 1, None) == ERR_ALIGN
    assert f(None, 0, 0, 0, 0, 0, None, None, 1, None) == OK


def test_per_tensor_validation(L):
    f = L.fp8_quantize_per_tensor
    assert f(A16, 1, 16, 5, None, A16, A16, A16, None) == ERR_FORMAT
    assert f(A16, 9, 16, 0, None, A16, A16, A16, None) == ERR_DTYPE
    assert f(A16, 1, -16, 0, None, A16, A16, A16, None) == ERR_SHAPE
    assert f(A16, 1, 16, 0, None, A16, None, A16, None) == ERR_NULL      # scale_out required
    assert f(A16, 1, 16, 0, None, A16, A16, None, None) == ERR_NULL      # amax_out required for current scaling
    assert f(None, 1, 16, 0, A16, A16, A16, None, None) == ERR_NULL
    assert f(A16, 1, 16, 0, A16, None, A16, None, None) == ERR_NULL
    assert f(A1, 1, 16, 0, None, A16, A16, A16, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, None, A4, A16, A16, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, A1, A16, A16, A16, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, None, A16, A1, A16, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, None, A16, A16, A1, None) == ERR_ALIGN


def test_fake_quant_validation(L):
    f = L.fp8_fake_quantize
    assert f(A16, 1, 4, 256, 1, 128, 3, None, A16, None, None) == ERR_FORMAT
    assert f(A16, 4, 4, 256, 1, 128, 0, None, A16, None, None) == ERR_DTYPE
    assert f(A16, 1, 4, 256, 1, 64, 0, None, A16, None, None) == ERR_SHAPE
    assert f(A16, 1, -4, 256, 1, 128, 0, None, A16, None, None) == ERR_SHAPE
    assert f(A16, 1, 4, 256, 0, 0, 0, None, A16, None, None) == ERR_NULL   # per tensor needs scale_in
    assert f(None, 1, 4, 256, 1, 128, 0, None, A16, None, None) == ERR_NULL
    assert f(A16, 1, 4, 256, 1, 128, 0, None, None, None, None) == ERR_NULL
    assert f(A1, 1, 4, 256, 1, 128, 0, None, A16, None, None) == ERR_ALIGN
    assert f(A16, 1, 4, 256, 1, 128, 0, None, A16 + 8, None, None) == ERR_ALIGN
    assert f(A16, 1, 4, 256, 1, 128, 0, None, A16 + 16, None, None) == ERR_ARG  # partial overlap
    assert f(None, 1, 0, 256, 1, 128, 0, None, None, None, None) == OK


def test_fused_per_tensor_validation(L):
    f = L.fp8_quantize_per_tensor_fused
    assert f(A16, 1, 16, 9, A16, A16, A16, A16, None) == ERR_FORMAT
    assert f(A16, 5, 16, 0, A16, A16, A16, A16, None) == ERR_DTYPE
    assert f(A16, 1, -1, 0, A16, A16, A16, A16, None) == ERR_SHAPE
    assert f(A16, 1, 16, 0, A16, A16, A16, None, None) == ERR_NULL   # workspace
    assert f(A16, 1, 16, 0, A16, None, A16, A16, None) == ERR_NULL
    assert f(A16, 1, 16, 0, A16, A16, None, A16, None) == ERR_NULL
    assert f(None, 1, 16, 0, A16, A16, A16, A16, None) == ERR_NULL
    assert f(A16, 1, 16, 0, A16, A16, A16, A16 + 8, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, A4, A16, A16, A16, None) == ERR_ALIGN


def test_fused_per_tensor_noalloc_validation(L):
    """The no-allocation entry point rejects bad arguments before it touches CUDA."""
    f = L.fp8_quantize_per_tensor_fused_noalloc
    assert f(A16, 1, 16, 9, A16, A16, A16, None) == ERR_FORMAT
    assert f(A16, 1, 16, -1, A16, A16, A16, None) == ERR_FORMAT
    assert f(A16, 5, 16, 0, A16, A16, A16, None) == ERR_DTYPE
    assert f(A16, 1, -1, 0, A16, A16, A16, None) == ERR_SHAPE
    assert f(A16, 1, 16, 0, A16, None, A16, None) == ERR_NULL   # scale_out
    assert f(A16, 1, 16, 0, A16, A16, None, None) == ERR_NULL   # amax_out
    assert f(A16, 1, 0, 0, A16, None, A16, None) == ERR_NULL    # scale_out is written even for n == 0
    assert f(None, 1, 16, 0, A16, A16, A16, None) == ERR_NULL   # x
    assert f(A16, 1, 16, 0, None, A16, A16, None) == ERR_NULL   # q
    assert f(A16 + 8, 1, 16, 0, A16, A16, A16, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, A16 + 4, A16, A16, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, A16, A16 + 2, A16, None) == ERR_ALIGN
    assert f(A16, 1, 16, 0, A16, A16, A16 + 1, None) == ERR_ALIGN


def test_per_tensor_grouped_validation(L):
    from fine_grained_block_b200.binding import FP8CurrentTensor
    f = L.fp8_quantize_per_tensor_grouped

    def arr(*ts):
        return (FP8CurrentTensor * len(ts))(*ts)
    good = FP8CurrentTensor(A16, A16, 16, A16, A16)
    assert f(arr(good), 1, 1, 9, None) == ERR_FORMAT
    assert f(arr(good), 1, 7, 0, None) == ERR_DTYPE
    assert f(arr(good), -1, 1, 0, None) == ERR_ARG
    assert f(None, 0, 1, 0, None) == OK          # nothing to do
    assert f(None, 2, 1, 0, None) == ERR_NULL
    assert f(arr(good, FP8CurrentTensor(A16, A16, -1, A16, A16)), 2, 1, 0, None) == ERR_SHAPE
    assert f(arr(good, FP8CurrentTensor(A16, A16, 16, None, A16)), 2, 1, 0, None) == ERR_NULL
    assert f(arr(good, FP8CurrentTensor(A16, A16, 16, A16, None)), 2, 1, 0, None) == ERR_NULL
    assert f(arr(good, FP8CurrentTensor(None, A16, 16, A16, A16)), 2, 1, 0, None) == ERR_NULL
    assert f(arr(good, FP8CurrentTensor(A16 + 8, A16, 16, A16, A16)), 2, 1, 0, None) == ERR_ALIGN
    assert f(arr(good, FP8CurrentTensor(A16, A16 + 4, 16, A16, A16)), 2, 1, 0, None) == ERR_ALIGN
    assert f(arr(good, FP8CurrentTensor(A16, A16, 16, A16 + 2, A16)), 2, 1, 0, None) == ERR_ALIGN


def test_amax_and_scale_validation(L):
    assert L.fp8_amax(A16, 7, 16, A16, None) == ERR_DTYPE
    assert L.fp8_amax(A16, 1, -1, A16, None) == ERR_SHAPE
    assert L.fp8_amax(A16, 1, 16, None, None) == ERR_NULL
    assert L.fp8_amax(None, 1, 16, A16, None) == ERR_NULL
    assert L.fp8_amax(A1, 1, 16, A16, None) == ERR_ALIGN
    assert L.fp8_amax(A16, 1, 16, A16 + 2, None) == ERR_ALIGN
    assert L.fp8_scale_from_amax(A16, 2, A16, None) == ERR_FORMAT
    assert L.fp8_scale_from_amax(None, 0, A16, None) == ERR_NULL
    assert L.fp8_scale_from_amax(A16, 0, None, None) == ERR_NULL
    assert L.fp8_scale_from_amax(A16 + 1, 0, A16, None) == ERR_ALIGN


def test_history_validation(L):
    f = L.fp8_amax_history_update
    assert f(A16, A16, 16, A16, 3, A16, None) == ERR_FORMAT
    assert f(A16, A16, 0, A16, 1, A16, None) == ERR_ARG
    assert f(A16, A16, 70000, A16, 1, A16, None) == ERR_ARG
    assert f(None, A16, 16, A16, 1, A16, None) == ERR_NULL
    assert f(A16, None, 16, A16, 1, A16, None) == ERR_NULL
    assert f(A16, A16, 16, None, 1, A16, None) == ERR_NULL
    assert f(A16, A16, 16, A16, 1, None, None) == ERR_NULL
    assert f(A1, A16, 16, A16, 1, A16, None) == ERR_ALIGN
    assert f(A16, A16 + 2, 16, A16, 1, A16, None) == ERR_ALIGN


def test_history_ex_validation(L):
    f = L.fp8_amax_history_update_ex
    assert f(A16, A16, 16, A16, 3, A16, 0, 1.0, 1.0, None) == ERR_FORMAT
    assert f(A16, A16, 16, A16, 0, A16, 2, 1.0, 1.0, None) == ERR_ARG
    assert f(A16, A16, 16, A16, 0, A16, 1, 1.5, 1.0, None) == ERR_ARG
    assert f(A16, A16, 16, A16, 0, A16, 1, -0.1, 1.0, None) == ERR_ARG
    assert f(A16, A16, 16, A16, 0, A16, 0, 1.0, 0.0, None) == ERR_ARG
    assert f(A16, A16, 16, A16, 0, A16, 0, 1.0, float("nan"), None) == ERR_ARG
    assert f(A16, A16, 0, A16, 0, A16, 0, 1.0, 1.0, None) == ERR_ARG
    assert f(None, A16, 16, A16, 0, A16, 0, 1.0, 1.0, None) == ERR_NULL
    assert f(A16, A16, 16, A16, 0, A1, 0, 1.0, 1.0, None) == ERR_ALIGN


def test_transpose_validation(L):
    f = L.fp8_quantize_per_tensor_transpose
    assert f(A16, 1, 4, 64, 9, None, A16, A16, A16, A16, None) == ERR_FORMAT
    assert f(A16, 7, 4, 64, 0, None, A16, A16, A16, A16, None) == ERR_DTYPE
    assert f(A16, 1, -4, 64, 0, None, A16, A16, A16, A16, None) == ERR_SHAPE
    assert f(A16, 1, 4, 64, 0, None, A16, A16, None, A16, None) == ERR_NULL      # scale_out
    assert f(A16, 1, 4, 64, 0, None, A16, A16, A16, None, None) == ERR_NULL      # current scaling needs amax_out
    assert f(A16, 1, 4, 64, 0, A16, A16, None, A16, None, None) == ERR_NULL      # qt
    assert f(A16, 1, 4, 64, 0, A16, A16, A1, A16, None, None) == ERR_ALIGN
    assert f(A16, 1, 4, 64, 0, A16, A1, A16, A16, None, None) == ERR_ALIGN


def test_gemm_ex_validation(L):
    f = L.fp8_gemm_blockwise_ex
    ok = (A16, A16, 0, A16, A16, 1, 0, 128, 256, 128, A16, 1, None)
    def call(**kw):
        args = list(ok)
        names = ["a", "sa", "a_fmt", "b", "sb", "b_block_rows", "b_fmt", "M", "N", "K", "c", "c_dtype", "stream"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return f(*args)
    assert call(b_block_rows=2) == ERR_SHAPE and call(b_block_rows=0) == ERR_SHAPE
    assert call(a_fmt=3) == ERR_FORMAT and call(b_fmt=3) == ERR_FORMAT
    assert call(c_dtype=5) == ERR_DTYPE
    assert call(N=100) == ERR_SHAPE and call(K=100) == ERR_SHAPE and call(M=-1) == ERR_SHAPE
    assert call(M=0) == OK
    assert call(c=None) == ERR_NULL and call(sb=None) == ERR_NULL
    assert call(a=A16 + 8) == ERR_ALIGN and call(sb=A1) == ERR_ALIGN and call(c=A16 + 4) == ERR_ALIGN


def test_blockwise_transpose_validation(L):
    f = L.fp8_quantize_blockwise_transpose
    ok = (A16, 1, 256, 384, 1, 128, 0, A16, A16, A16, A16, None)
    def call(**kw):
        args = list(ok)
        names = ["x", "dtype", "rows", "cols", "br", "bc", "fmt", "q", "scales", "qt", "scales_t", "stream"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return f(*args)
    assert call(fmt=9) == ERR_FORMAT
    assert call(dtype=7) == ERR_DTYPE
    assert call(br=128, bc=1) == ERR_SHAPE                # only 1x128 and 128x128
    assert call(br=32) == ERR_SHAPE
    assert call(rows=200) == ERR_SHAPE                    # rows and cols multiples of 128
    assert call(cols=100) == ERR_SHAPE
    assert call(rows=-128) == ERR_SHAPE
    assert call(rows=0) == OK and call(cols=0, x=None) == OK  # nothing to do
    for name in ("x", "q", "scales", "qt", "scales_t"):
        assert call(**{name: None}) == ERR_NULL, name
    for name in ("x", "q", "qt"):
        assert call(**{name: A16 + 8}) == ERR_ALIGN, name
    assert call(scales=A1) == ERR_ALIGN and call(scales_t=A1) == ERR_ALIGN


def test_delayed_step_validation(L):
    f = L.fp8_quantize_delayed_step
    ok = (A16, 1, 64, 0, A16, A16, A16, 16, 0, 1.0, 1.0, A16, A16 + 16, A16, A16, None)
    def call(**kw):
        args = list(ok)
        names = ["x", "dtype", "n", "fmt", "scale", "history", "state", "window", "algo", "alpha", "margin", "q",
                 "scale_used", "amax_out", "workspace", "stream"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return f(*args)
    assert call(fmt=5) == ERR_FORMAT
    assert call(dtype=4) == ERR_DTYPE
    assert call(n=-1) == ERR_SHAPE
    assert call(window=0) == ERR_ARG
    assert call(algo=3) == ERR_ARG
    assert call(alpha=2.0) == ERR_ARG
    assert call(margin=0.0) == ERR_ARG
    assert call(scale_used=A16) == ERR_ARG          # the same pointer as scale
    assert call(workspace=None) == ERR_NULL
    assert call(q=None) == ERR_NULL
    assert call(history=A1) == ERR_ALIGN
    assert call(workspace=A16 + 4) == ERR_ALIGN


def test_grouped_validation(L):
    T = binding.FP8BlockTensor
    g = L.fp8_quantize_blockwise_grouped
    good = (T * 2)(T(A16, A16, A16, 128, 256), T(A16, A16, A16, 3, 128))
    assert g(good, 2, 1, 1, 128, 9, None) == ERR_FORMAT
    assert g(good, 2, 3, 1, 128, 0, None) == ERR_DTYPE
    assert g(good, -1, 1, 1, 128, 0, None) == ERR_ARG
    assert g(good, 2, 1, 64, 128, 0, None) == ERR_SHAPE
    assert g(None, 0, 1, 1, 128, 0, None) == OK            # nothing to do
    assert g(None, 2, 1, 1, 128, 0, None) == ERR_NULL
    assert g((T * 1)(T(A16, A16, A16, 4, 100)), 1, 1, 1, 128, 0, None) == ERR_SHAPE   # cols % 128
    assert g((T * 1)(T(A16, None, A16, 4, 128)), 1, 1, 1, 128, 0, None) == ERR_NULL
    assert g((T * 1)(T(A1, A16, A16, 4, 128)), 1, 1, 1, 128, 0, None) == ERR_ALIGN


def test_delayed_grouped_validation(L):
    T = binding.FP8DelayedTensor
    g = L.fp8_quantize_delayed_step_grouped
    one = (T * 1)(T(A16, A16, 64, A16, A16, A16, A16 + 16, A16, ))
    assert g(one, 1, 1, 7, 16, 0, 1.0, 1.0, A16, None) == ERR_FORMAT
    assert g(one, 1, 9, 0, 16, 0, 1.0, 1.0, A16, None) == ERR_DTYPE
    assert g(one, -1, 1, 0, 16, 0, 1.0, 1.0, A16, None) == ERR_ARG
    assert g(one, 1, 1, 0, 0, 0, 1.0, 1.0, A16, None) == ERR_ARG
    assert g(one, 1, 1, 0, 16, 0, 1.0, -1.0, A16, None) == ERR_ARG
    assert g(None, 0, 1, 0, 16, 0, 1.0, 1.0, None, None) == OK
    assert g(one, 1, 1, 0, 16, 0, 1.0, 1.0, None, None) == ERR_NULL
    assert g(one, 1, 1, 0, 16, 0, 1.0, 1.0, A16 + 8, None) == ERR_ALIGN
    same = (T * 1)(T(A16, A16, 64, A16, A16, A16, A16, A16))
    assert g(same, 1, 1, 0, 16, 0, 1.0, 1.0, A16, None) == ERR_ARG     # scale_used == scale
    neg = (T * 1)(T(A16, A16, -1, A16, A16, A16, A16 + 16, A16))
    assert g(neg, 1, 1, 0, 16, 0, 1.0, 1.0, A16, None) == ERR_SHAPE


def test_gemm_validation(L):
    g = L.fp8_gemm_blockwise
    assert g(A16, A16, 2, A16, A16, 0, 128, 256, 128, A16, 1, None) == ERR_FORMAT
    assert g(A16, A16, 0, A16, A16, 0, 128, 256, 128, A16, 3, None) == ERR_DTYPE
    assert g(A16, A16, 0, A16, A16, 0, 128, 128, 128, A16, 1, None) == ERR_SHAPE   # N % 256
    assert g(A16, A16, 0, A16, A16, 0, 128, 256, 100, A16, 1, None) == ERR_SHAPE   # K % 128
    assert g(A16, A16, 0, A16, A16, 0, -1, 256, 128, A16, 1, None) == ERR_SHAPE
    assert g(None, None, 0, None, None, 0, 0, 256, 128, None, 1, None) == OK        # M = 0: nothing to do
    assert g(A16, A16, 0, A16, A16, 0, 128, 256, 128, None, 1, None) == ERR_NULL
    assert g(A16, None, 0, A16, A16, 0, 128, 256, 128, A16, 1, None) == ERR_NULL
    assert g(A1, A16, 0, A16, A16, 0, 128, 256, 128, A16, 1, None) == ERR_ALIGN
    assert g(A16, A16, 0, A16, A16, 0, 128, 256, 128, A1, 1, None) == ERR_ALIGN


def test_mx_validation(L):
    q = L.fp8_quantize_mx
    assert q(A16, 1, 4, 64, 2, 0, A16, A16, None) == ERR_FORMAT
    assert q(A16, 2, 4, 64, 0, 0, A16, A16, None) == ERR_DTYPE
    assert q(A16, 1, 4, 64, 0, 2, A16, A16, None) == ERR_ARG
    assert q(A16, 1, -1, 64, 0, 0, A16, A16, None) == ERR_SHAPE
    assert q(A16, 1, 1 << 40, 1 << 40, 0, 0, A16, A16, None) == ERR_SHAPE
    assert q(None, 1, 0, 64, 0, 0, None, None, None) == OK  # empty: nothing to do
    assert q(A16, 1, 4, 64, 0, 0, A16, None, None) == ERR_NULL
    assert q(A1, 1, 4, 64, 0, 0, A16, A1, None) == ERR_ALIGN
    d = L.fp8_dequantize_mx
    assert d(A16, 0, 4, 64, A16, A16, 2, None) == ERR_DTYPE
    assert d(A16, 5, 4, 64, A16, A16, 0, None) == ERR_FORMAT
    assert d(A16, 0, 4, -3, A16, A16, 0, None) == ERR_SHAPE
    assert d(A16, 0, 4, 64, None, A16, 0, None) == ERR_NULL
    assert d(A16, 0, 4, 64, A1, A1, 0, None) == ERR_ALIGN


def test_diagnostics_validation(L):
    assert L.fp8_device_status(None, 0, None) == ERR_NULL
    assert L.fp8_device_status(A1, 0, None) == ERR_ALIGN
    assert L.fp8_selftest_wait_timeout(0, None) == ERR_ARG
    assert L.fp8_selftest_wait_timeout(20_000_000, None) == ERR_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.fp8_quantize_blockwise(x)
    with pytest.raises(ValueError):
        binding.fp8_quantize_per_tensor(x)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        binding.load_library(str(tmp_path / "nope.so"))
