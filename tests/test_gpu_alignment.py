"""GPU parity with 16- but not 32-byte aligned buffers.

Every streaming kernel uses 32-byte lanes when its buffers allow them and
16-byte lanes otherwise; these tests drive each entry point down the 16-byte
path (inputs and outputs placed 16 bytes past a 32-byte boundary) and require
the same bytes as the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs
from parity_util import assert_bytes_equal, fp32_bits, host_input

pytestmark = pytest.mark.gpu


def at16(shape, dtype, src=None):
    """A CUDA tensor whose data starts 16 bytes past a 32-byte boundary (copied from src if given)."""
    esz = torch.empty(0, dtype=dtype).element_size()
    n = int(np.prod(shape)) if len(shape) else 1
    buf = torch.empty(n + 64 // esz, dtype=dtype, device="cuda")
    base = buf.data_ptr()
    skip = ((16 - base % 32) % 32) // esz
    t = buf[skip:skip + n].view(shape)
    assert t.data_ptr() % 32 == 16
    if src is not None:
        t.copy_(src.to("cuda"))
    return t


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("fmt", [B.E4M3, B.E5M2])
def test_blockwise_and_dequant(dtype, fmt):
    R, C = 384, 1024
    x_cpu = inputs.random_matrix(R, C, seed=8000, dtype=dtype, outlier_frac=0.01, factor=1e3)
    xh = host_input(x_cpu)
    x = at16((R, C), dtype, x_cpu)
    for block in ((1, 128), (128, 128)):
        q = at16((R, C), torch.uint8)
        s = torch.empty((R // block[0], C // 128), dtype=torch.float32, device="cuda")
        B.fp8_quantize_blockwise(x, block, fmt, q=q, scales=s)
        oq, os_ = oracle.quantize_blockwise(xh, *block, fmt)
        torch.cuda.synchronize()
        assert_bytes_equal(s, fp32_bits(os_), f"{block} scales")
        assert_bytes_equal(q, oq, f"{block} codes")
        for out_dtype, oc in ((torch.float32, oracle.F32), (torch.bfloat16, oracle.BF16)):
            y = at16((R, C), out_dtype)
            B.fp8_dequantize(q, s, block, fmt, out_dtype, y=y)
            torch.cuda.synchronize()
            assert_bytes_equal(y, oracle.dequantize(oq, fmt, os_, *block, oc), f"{block} dequant {out_dtype}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_per_tensor_current_delayed_and_step(dtype):
    n = (1 << 20) + 5
    x_cpu = inputs.random_matrix(1, n, seed=8100, dtype=dtype, outlier_frac=1e-3, factor=1e3).reshape(-1)
    xh = host_input(x_cpu)
    x = at16((n,), dtype, x_cpu)
    for scale in (None, 3.5):
        q = at16((n,), torch.uint8)
        s_in = None if scale is None else torch.tensor([scale], dtype=torch.float32, device="cuda")
        _, s, a = B.fp8_quantize_per_tensor(x, B.E5M2, scale_in=s_in, q=q)
        oq, os_, oa = oracle.quantize_per_tensor(xh, B.E5M2, scale)
        torch.cuda.synchronize()
        assert_bytes_equal(q, oq, f"per-tensor scale={scale} codes")
        assert_bytes_equal(s, fp32_bits([os_]), "scale")
        assert_bytes_equal(a, fp32_bits([oa]), "amax")
        y = at16((n,), torch.bfloat16)
        B.fp8_dequantize(q.view(1, n), s, (0, 0), B.E5M2, torch.bfloat16, y=y.view(1, n))
        torch.cuda.synchronize()
        assert_bytes_equal(y, oracle.dequantize(oq.reshape(1, n), B.E5M2, np.array([os_], np.float32), 0, 0,
                                                oracle.BF16).reshape(-1), "per-tensor dequant")
    sc = B.DelayedScaler(window=2, fmt=B.E5M2)
    ref = oracle.AmaxHistory(2, B.E5M2)
    for k in range(4):
        q, s_used = sc.step(x, q=at16((n,), torch.uint8))
        oq, _, oa = oracle.quantize_per_tensor(xh, B.E5M2, float(ref.scale[0]))
        ref.update(oa)
        torch.cuda.synchronize()
        assert_bytes_equal(q, oq, f"delayed step {k}")
        assert_bytes_equal(sc.scale, fp32_bits(ref.scale), f"delayed step {k} next scale")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fake_quant(dtype):
    R, C = 256, 512
    x_cpu = inputs.random_matrix(R, C, seed=8200, dtype=dtype, outlier_frac=0.01, factor=1e3)
    xh = host_input(x_cpu)
    x = at16((R, C), dtype, x_cpu)
    for block in ((1, 128), (128, 128)):
        y = at16((R, C), dtype)
        B.fp8_fake_quantize(x, block, B.E4M3, y=y)
        torch.cuda.synchronize()
        want, _ = oracle.fake_quantize(xh, B.E4M3, *block)
        assert_bytes_equal(y, want, f"fake quant {block}")
