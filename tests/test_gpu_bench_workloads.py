"""GPU parity on the benchmark's other workloads, at their full sizes and in the calls it times.

- MX 1x32 quantize and dequantize of the bf16 16384x7168 activations (outlier channels);
- the transposing per-tensor cast of the same activations, delayed (given scale) and current;
- 1x128 quantization of the same activations and of their transpose in one pass;
- the blockwise GEMM at 16384x4096x7168: the whole last 256-row tile row of C and sampled rows;
- the weight-gradient GEMM at 4096x7168x16384 (B in 1x128 blocks): whole sampled rows of dW;
- 128 weights of 1024x1024 in one grouped 128x128 call;
- one grouped delayed-scaling step over 128 gradients of 2^20 elements.

Every expected value comes from the oracle (threaded over independent row chunks where large).
"""
import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs
from parity_util import (assert_bytes_equal, fp32_bits, host_input, oracle_blockwise, oracle_dequant_mx, oracle_gemm,
                         oracle_mx, oracle_per_tensor, to_cuda)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def activations():
    a = inputs.activation_outlier_channels()
    return a, host_input(a)


def test_mx_activations_16384x7168(activations):
    a, xh = activations
    x = to_cuda(a)
    q, e8 = B.fp8_quantize_mx(x, B.E4M3, B.MX_FIT)
    assert tuple(e8.shape) == (16384, 224)
    oq, oe = oracle_mx(xh, oracle.E4M3, oracle.MX_FIT)
    assert_bytes_equal(e8, oe, "MX scale bytes")
    assert_bytes_equal(q, oq, "MX codes")
    y = B.fp8_dequantize_mx(q, e8, B.E4M3, torch.bfloat16)
    assert_bytes_equal(y, oracle_dequant_mx(oq, oracle.E4M3, oe, oracle.BF16), "MX dequant bf16")


@pytest.mark.parametrize("scale", [0.25, None], ids=["delayed", "current"])
def test_transpose_activations_16384x7168(activations, scale):
    a, xh = activations
    x = to_cuda(a)
    s_in = None if scale is None else torch.tensor([scale], dtype=torch.float32, device="cuda")
    q, qt, s, am = B.fp8_quantize_per_tensor_transpose(x, B.E4M3, s_in)
    oq, os_, oa = oracle_per_tensor(xh, oracle.E4M3, scale=scale)
    assert_bytes_equal(s, fp32_bits([os_]), "scale")
    assert_bytes_equal(am, fp32_bits([oa]), "amax")
    assert_bytes_equal(q, oq, "q")
    # qt is q transposed, by definition of the second output
    assert_bytes_equal(qt, np.ascontiguousarray(oq.T), "qt")


def test_blockwise_transpose_activations_16384x7168(activations):
    a, xh = activations
    x = to_cuda(a)
    q, s, qt, st = B.fp8_quantize_blockwise_transpose(x, (1, 128), B.E4M3)
    oq, os_ = oracle_blockwise(xh, 1, 128, oracle.E4M3)
    assert_bytes_equal(s, fp32_bits(os_), "scales")
    assert_bytes_equal(q, oq, "q")
    del q, s, oq, os_
    oqt, ost = oracle_blockwise(np.ascontiguousarray(xh.T), 1, 128, oracle.E4M3)
    assert_bytes_equal(st, fp32_bits(ost), "scales_t")
    assert_bytes_equal(qt, oqt, "qt")


def test_gemm_16384x4096x7168_full_last_tile_row_and_sampled_rows():
    """The benchmark's GEMM shape: every output of the last 256-row tile row (one CTA pair's tiles, the
    last round of the persistent schedule, all 16 column tiles) and 12 sampled rows elsewhere."""
    M, N, K = 16384, 4096, 7168
    x = inputs.random_matrix(M, K, seed=6, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e2)
    w = inputs.random_matrix(N, K, seed=7, dtype=torch.bfloat16, scale=0.02)
    qa, sa = oracle_blockwise(host_input(x), 1, 128, oracle.E4M3)
    qb, sb = oracle_blockwise(host_input(w), 128, 128, oracle.E4M3)
    c = B.fp8_gemm_blockwise(to_cuda(torch.from_numpy(qa)), to_cuda(torch.from_numpy(sa)),
                             to_cuda(torch.from_numpy(qb)), to_cuda(torch.from_numpy(sb)), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 255, 256, 4095, 8191, 8192, 12000, 15000, 16000] + list(range(M - 256, M))
    want = oracle_gemm(qa[rows], sa[rows], oracle.E4M3, qb, sb, oracle.E4M3)
    mag = oracle_gemm(qa[rows] & 0x7F, sa[rows], oracle.E4M3, qb & 0x7F, sb, oracle.E4M3)
    got = c[torch.as_tensor(rows, device="cuda")].float().cpu().numpy().astype(np.float64)
    # fp32 sums of 56 promoted chunks (2^-12 of the absolute sum), then one bf16 rounding of the result
    tol = 2.0 ** -12 * mag + 2.0 ** -8 * np.abs(want)
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} sampled outputs outside the bound"


def test_weight_gradient_gemm_4096x7168x16384_sampled_rows():
    """The benchmark's weight-gradient GEMM shape (B in 1x128 blocks, E5M2 x E4M3; M < N, so the row tile
    is fastest): whole rows of dW from every row tile, against the oracle."""
    M, N, K = 4096, 7168, 16384
    dyt = inputs.random_matrix(M, K, seed=8, dtype=torch.bfloat16, scale=1e-3, outlier_frac=1e-3, factor=1e2)
    xt = inputs.random_matrix(N, K, seed=9, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e2)
    qa, sa = oracle_blockwise(host_input(dyt), 1, 128, oracle.E5M2)
    qb, sb = oracle_blockwise(host_input(xt), 1, 128, oracle.E4M3)
    c = B.fp8_gemm_blockwise(to_cuda(torch.from_numpy(qa)), to_cuda(torch.from_numpy(sa)),
                             to_cuda(torch.from_numpy(qb)), to_cuda(torch.from_numpy(sb)), a_fmt=B.E5M2,
                             b_fmt=B.E4M3, out_dtype=torch.bfloat16, b_block=1)
    torch.cuda.synchronize()
    rows = [0, 255, 256, 1000, 2047, 2048, 3333, 4095]
    want = oracle_gemm(qa[rows], sa[rows], oracle.E5M2, qb, sb, oracle.E4M3, b_block=1)
    mag = oracle_gemm(qa[rows] & 0x7F, sa[rows], oracle.E5M2, qb & 0x7F, sb, oracle.E4M3, b_block=1)
    got = c[torch.as_tensor(rows, device="cuda")].float().cpu().numpy().astype(np.float64)
    tol = 2.0 ** -12 * mag + 2.0 ** -8 * np.abs(want)
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} sampled outputs outside the bound"


def test_grouped_128_weights_1024x1024():
    ws = [inputs.random_matrix(1024, 1024, seed=100 + i, dtype=torch.bfloat16, scale=0.02) for i in range(128)]
    qs, ss = B.fp8_quantize_blockwise_grouped([to_cuda(w) for w in ws], (128, 128), B.E4M3)
    torch.cuda.synchronize()
    for i, (w, q, s) in enumerate(zip(ws, qs, ss)):
        oq, os_ = oracle.quantize_blockwise(host_input(w), 128, 128, oracle.E4M3)
        assert_bytes_equal(s, fp32_bits(os_), f"weight {i} scales")
        assert_bytes_equal(q, oq, f"weight {i} codes")


def test_grouped_delayed_step_128_gradients_2pow20():
    xs = [inputs.random_matrix(1, 1 << 20, seed=300 + i, dtype=torch.bfloat16, scale=1e-3).reshape(-1)
          for i in range(128)]
    scalers = [B.DelayedScaler(window=16, fmt=B.E5M2) for _ in xs]
    refs = [oracle.AmaxHistory(16, oracle.E5M2) for _ in xs]
    xd = [to_cuda(x) for x in xs]
    for step in range(2):
        qs = B.fp8_quantize_delayed_step_grouped(xd, scalers)
        torch.cuda.synchronize()
        for i, (x, q, sc, ref) in enumerate(zip(xs, qs, scalers, refs)):
            oq, os_, oa = oracle.quantize_per_tensor(host_input(x), oracle.E5M2, scale=float(ref.scale[0]))
            ref.update(oa)
            assert_bytes_equal(sc.scale_used, fp32_bits([os_]), f"step {step} tensor {i} scale used")
            assert_bytes_equal(sc.amax, fp32_bits([oa]), f"step {step} tensor {i} amax")
            assert_bytes_equal(sc.scale, fp32_bits(ref.scale), f"step {step} tensor {i} next scale")
            assert_bytes_equal(sc.history, fp32_bits(ref.history), f"step {step} tensor {i} history")
            assert sc.state.cpu().tolist() == ref.state.tolist()
            assert_bytes_equal(q, oq, f"step {step} tensor {i} codes")
