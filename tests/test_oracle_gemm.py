"""Pins of the oracle's blockwise-scaled GEMM (the consumer of the codes).

Mixed-precision handbook, "FP8 training", closing notes: FP8 products with
fp32 accumulation, the partial sum promoted every 128 elements where the
1x128 / 128x128 scales are applied.  The oracle sums exact FP8 products per
128-chunk and divides by the two scales; here it is checked against a hand
example and against the other order of the same mathematics (dequantize each
operand first, then one float64 matrix product).
"""
import math

import numpy as np
import pytest

import oracle
from oracle import E4M3, E5M2


def test_hand_example_two_chunks():
    # K = 256: two chunks.  Every code 0x38 (= 1.0 in E4M3), so each chunk's
    # partial sum is 128.  sa = [2, 4], sb = [1, 0.5]:
    # C = 128 / (2 * 1) + 128 / (4 * 0.5) = 64 + 64 = 128.
    a = np.full((1, 256), 0x38, dtype=np.uint8)
    b = np.full((1, 256), 0x38, dtype=np.uint8)
    c = oracle.gemm_blockwise(a, np.array([[2.0, 4.0]], np.float32), E4M3, b, np.array([[1.0, 0.5]], np.float32),
                              E4M3)
    assert c.shape == (1, 1) and c[0, 0] == 128.0
    # sign: 0xB8 = -1.0 in one operand flips the chunk it sits in
    a[0, :128] = 0xB8
    c = oracle.gemm_blockwise(a, np.array([[2.0, 4.0]], np.float32), E4M3, b, np.array([[1.0, 0.5]], np.float32),
                              E4M3)
    assert c[0, 0] == 0.0


@pytest.mark.parametrize("a_fmt,b_fmt", [(E4M3, E4M3), (E5M2, E4M3), (E4M3, E5M2)])
@pytest.mark.parametrize("M,N,K", [(3, 130, 384), (17, 256, 256), (5, 7, 200)])
def test_equals_dequantize_then_matmul(a_fmt, b_fmt, M, N, K):
    rng = np.random.default_rng(M * 1000 + N + K)
    x = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-3, 3, (M, 1)))).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qa, sa = oracle.quantize_blockwise(x, 1, 128, a_fmt)
    qb, sb = oracle.quantize_blockwise(w, 128, 128, b_fmt)
    c = oracle.gemm_blockwise(qa, sa, a_fmt, qb, sb, b_fmt)
    # the other order: dequantize in float64 with the scales broadcast over
    # their blocks, then a single library matrix product
    da = oracle.decode_table(a_fmt)[qa].astype(np.float64) / np.repeat(sa.astype(np.float64), 128, axis=1)[:, :K]
    sbx = np.repeat(np.repeat(sb.astype(np.float64), 128, axis=0), 128, axis=1)[:N, :K]
    db = oracle.decode_table(b_fmt)[qb].astype(np.float64) / sbx
    ref = da @ db.T
    mag = np.abs(da) @ np.abs(db).T
    assert np.all(np.abs(c - ref) <= 1e-13 * mag + 1e-300)
    # and the product approximates x w^T within the quantization error
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    assert np.all(np.abs(c - exact) <= 0.25 * (np.abs(x) @ np.abs(w).T) + 1e-30)


def test_hand_example_b_rows_scaled_separately():
    # B with 1x128 blocks: each row of B has its own scale per chunk.  K = 128,
    # every code 1.0: each partial sum is 128.  sa = [2]; sb = [[1], [4]]:
    # C[0][0] = 128 / (2 * 1) = 64, C[0][1] = 128 / (2 * 4) = 16.
    a = np.full((1, 128), 0x38, dtype=np.uint8)
    b = np.full((2, 128), 0x38, dtype=np.uint8)
    c = oracle.gemm_blockwise(a, np.array([[2.0]], np.float32), E4M3, b, np.array([[1.0], [4.0]], np.float32), E4M3,
                              b_block=1)
    assert c.tolist() == [[64.0, 16.0]]
    # the same B under 128x128 blocks has one scale for both rows
    c = oracle.gemm_blockwise(a, np.array([[2.0]], np.float32), E4M3, b, np.array([[4.0]], np.float32), E4M3)
    assert c.tolist() == [[16.0, 16.0]]


@pytest.mark.parametrize("a_fmt,b_fmt", [(E4M3, E4M3), (E5M2, E5M2), (E5M2, E4M3)])
@pytest.mark.parametrize("M,N,K", [(3, 130, 384), (17, 256, 256), (5, 7, 200)])
def test_weight_gradient_form_equals_dequantize_then_matmul(a_fmt, b_fmt, M, N, K):
    """dW = dY^T X: both operands 1x128 along K (tokens), from the quantizer of x^T."""
    rng = np.random.default_rng(M * 7 + N + K)
    dy_t = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-4, 0, (M, 1)))).astype(np.float32)
    x_t = (rng.standard_normal((N, K)) * np.exp(rng.uniform(-2, 2, (N, 1)))).astype(np.float32)
    qa, sa = oracle.quantize_blockwise(dy_t, 1, 128, a_fmt)
    qb, sb = oracle.quantize_blockwise(x_t, 1, 128, b_fmt)
    assert sb.shape == (N, math.ceil(K / 128))
    c = oracle.gemm_blockwise(qa, sa, a_fmt, qb, sb, b_fmt, b_block=1)
    da = oracle.decode_table(a_fmt)[qa].astype(np.float64) / np.repeat(sa.astype(np.float64), 128, axis=1)[:, :K]
    db = oracle.decode_table(b_fmt)[qb].astype(np.float64) / np.repeat(sb.astype(np.float64), 128, axis=1)[:, :K]
    ref = da @ db.T
    mag = np.abs(da) @ np.abs(db).T
    assert np.all(np.abs(c - ref) <= 1e-13 * mag + 1e-300)
    exact = dy_t.astype(np.float64) @ x_t.astype(np.float64).T
    assert np.all(np.abs(c - exact) <= 0.25 * (np.abs(dy_t) @ np.abs(x_t).T) + 1e-30)
