"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark uses.

Every element is compared with the (threaded) oracle: the 16384x7168
activations, 32 delayed steps of the 8192x8192 gradients, and the size sweep
from 2^20 to 2^30 elements in all three of its modes with their dequant.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs
from parity_util import (assert_bytes_equal, fp32_bits, host_input, oracle_amax, oracle_blockwise, oracle_cast,
                         oracle_dequant, oracle_per_tensor, to_cuda)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_activations_16384x7168_1x128():
    a = inputs.activation_outlier_channels()
    xh = host_input(a)
    x = to_cuda(a)
    q, s = B.fp8_quantize_blockwise(x, (1, 128), B.E4M3)
    assert tuple(s.shape) == (16384, 56)
    oq, os_ = oracle_blockwise(xh, 1, 128, oracle.E4M3)
    assert_bytes_equal(s, fp32_bits(os_), "scales")
    assert_bytes_equal(q, oq, "codes")
    y = B.fp8_dequantize(q, s, (1, 128), B.E4M3, torch.bfloat16)
    assert_bytes_equal(y, oracle_dequant(oq, oracle.E4M3, os_, 1, 128, oracle.BF16), "dequant bf16")


def test_gradients_8192_delayed_e5m2_32_steps():
    W, steps = 16, 32
    base = inputs.gradient_base()
    sc = B.DelayedScaler(window=W, fmt=B.E5M2)
    ref = oracle.AmaxHistory(W, oracle.E5M2)
    q = torch.empty(8192, 8192, dtype=torch.uint8, device="cuda")
    zero_frac = []
    for k in range(steps):
        g = inputs.gradient_step(base, k)
        gh = host_input(g)
        s_ref = ref.scale[0]
        q, s_used = sc.step(to_cuda(g), q=q)
        oq, os_, oa = oracle_per_tensor(gh, oracle.E5M2, scale=float(s_ref))
        ref.update(oa)
        torch.cuda.synchronize()
        assert_bytes_equal(s_used, fp32_bits([os_]), f"step {k} scale used")
        assert_bytes_equal(sc.amax, fp32_bits([oa]), f"step {k} amax")
        assert_bytes_equal(sc.scale, fp32_bits(ref.scale), f"step {k} next scale")
        assert_bytes_equal(q, oq, f"step {k} codes")
        zero_frac.append(float(((q & 0x7F) == 0).float().mean()))
    assert sc.state.cpu().tolist() == ref.state.tolist()
    assert_bytes_equal(sc.history, fp32_bits(ref.history), "history")
    # with s = 1 the smallest gradients flush to zero; with the window scale they do not
    assert min(zero_frac[:W]) > 0.1 and max(zero_frac[W:]) < 1e-3


def _row_chunks(R, rows_per_chunk):
    return [(r0, min(R, r0 + rows_per_chunk)) for r0 in range(0, R, rows_per_chunk)]


@pytest.mark.parametrize("log2_n", [20, 22, 24, 26, 28, 30])
def test_sweep_full(log2_n):
    """The size sweep, every element: 1x128 E4M3, 128x128 E4M3 and per-tensor current E5M2, each with its
    bf16 dequant, compared with the oracle in chunks of 2^24 elements (whole block rows), so the host holds
    one chunk of expected values at a time."""
    t = inputs.sweep_tensor(log2_n)
    xh = host_input(t)
    x = to_cuda(t)
    del t
    R, C = xh.shape
    chunks = _row_chunks(R, max(128, (1 << 24) // C))
    for block in ((1, 128), (128, 128)):
        br = block[0]
        q, s = B.fp8_quantize_blockwise(x, block, B.E4M3)
        y = B.fp8_dequantize(q, s, block, B.E4M3, torch.bfloat16)
        for r0, r1 in chunks:
            oq, os_ = oracle_blockwise(xh[r0:r1], *block, oracle.E4M3)
            assert_bytes_equal(s[r0 // br:math.ceil(r1 / br)], fp32_bits(os_), f"{block} scales rows {r0}..")
            assert_bytes_equal(q[r0:r1], oq, f"{block} codes rows {r0}..")
            assert_bytes_equal(y[r0:r1], oracle_dequant(oq, oracle.E4M3, os_, *block, oracle.BF16),
                               f"{block} dequant rows {r0}..")
        del q, s, y
    q, s, a = B.fp8_quantize_per_tensor(x, B.E5M2)
    y = B.fp8_dequantize(q, s, (0, 0), B.E5M2, torch.bfloat16)
    oa = oracle_amax(xh)
    os_ = oracle.scale_from_amax(oa, oracle.E5M2)
    assert_bytes_equal(a, fp32_bits([oa]), "amax")
    assert_bytes_equal(s, fp32_bits([os_]), "scale")
    for r0, r1 in chunks:
        oq = oracle_cast(xh[r0:r1], oracle.E5M2, os_)
        assert_bytes_equal(q[r0:r1], oq, f"per-tensor codes rows {r0}..")
        assert_bytes_equal(y[r0:r1], oracle_dequant(oq, oracle.E5M2, np.array([os_], np.float32), 0, 0,
                                                    oracle.BF16), f"per-tensor dequant rows {r0}..")


def test_fake_quant_activations_16384x7168():
    a = inputs.activation_outlier_channels()
    xh = host_input(a)
    from parity_util import oracle_dequant
    oq, os_ = oracle_blockwise(xh, 1, 128, oracle.E4M3)
    oy = oracle_dequant(oq, oracle.E4M3, os_, 1, 128, oracle.BF16)
    x = to_cuda(a)
    y = B.fp8_fake_quantize(x, (1, 128), B.E4M3)
    assert_bytes_equal(y, oy, "fake quant 1x128")
    del y
    B.fp8_fake_quantize(x, (1, 128), B.E4M3, y=x)  # in place
    assert_bytes_equal(x, oy, "fake quant 1x128 in place")
