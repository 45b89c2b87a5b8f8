"""GPU parity of the consumer GEMM (fp8_gemm_blockwise) against the oracle.

The tensor cores sum each 128-product chunk in an order of their own, so this
is not bit-exact.  With B in 1x128 blocks the factor is RN(1/sa) and RN(1/sb[n])
applied as two roundings, 3 x 2^-24 instead of 2^-23; the bound below holds.  The bound is derived from the arithmetic: every FP8 product
is exact in fp32; a chunk sum of 128 products carries at most a relative
2^-14 of the chunk's absolute sum (allowing an accumulator narrower than fp32,
the limitation the handbook's promotion works around); the factor
RN(1/RN(sa*sb)) adds 2^-23; the fp32 fma accumulation over K/128 chunks adds
(K/128) * 2^-24.  With S[m][n] the same GEMM over absolute values,
    |C_gpu - C_exact| <= (2^-14 + 2^-23 + (K/128) 2^-24) * S    (+ half a bf16
ulp of |C| for bf16 output).  The test uses 2^-12 * S, well inside which a
wrong block, scale or index (an O(1) relative error) cannot hide.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs
from parity_util import host_input, to_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _clear_device_status():
    """Start this module with a clear device status word (other tests set its bits on purpose)."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert B.load_library().fp8_device_status(st.data_ptr(), 1, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    yield


def oracle_codes(M, N, K, a_fmt, b_fmt, seed):
    x = inputs.random_matrix(M, K, seed=seed, dtype=torch.bfloat16, outlier_frac=0.01, factor=1e2)
    w = inputs.random_matrix(N, K, seed=seed + 1, dtype=torch.bfloat16, scale=0.02)
    qa, sa = oracle.quantize_blockwise(host_input(x), 1, 128, a_fmt)
    qb, sb = oracle.quantize_blockwise(host_input(w), 128, 128, b_fmt)
    return qa, sa, qb, sb


def check_gemm(qa, sa, a_fmt, qb, sb, b_fmt, c_gpu, what, rows=None, b_block=128):
    """Compare c_gpu (torch, [M, N]) with the oracle on the given rows (all by default)."""
    if rows is not None:
        qa, sa = qa[rows], sa[rows]
        c_gpu = c_gpu[torch.as_tensor(rows, device=c_gpu.device)]
    want = oracle.gemm_blockwise(qa, sa, a_fmt, qb, sb, b_fmt, b_block=b_block)
    mag = oracle.gemm_blockwise(qa & 0x7F, sa, a_fmt, qb & 0x7F, sb, b_fmt, b_block=b_block)
    got = c_gpu.float().cpu().numpy().astype(np.float64)
    tol = 2.0 ** -12 * mag
    if c_gpu.dtype == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(want)
    err = np.abs(got - want)
    bad = err > tol
    assert not np.isnan(got).any(), what
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside the bound; worst "
                           f"{float((err / np.maximum(mag, 1e-30)).max()):.3g} of S")
    return float((err / np.maximum(mag, 1e-30)).max())


SHAPES = [(128, 256, 128), (256, 512, 1024), (200, 256, 384), (1, 256, 128), (130, 768, 640)]


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_matches_oracle(out_dtype):
    for i, (M, N, K) in enumerate(SHAPES):
        qa, sa, qb, sb = oracle_codes(M, N, K, B.E4M3, B.E4M3, seed=5000 + i)
        c = B.fp8_gemm_blockwise(to_cuda(torch.from_numpy(qa)), to_cuda(torch.from_numpy(sa)),
                                 to_cuda(torch.from_numpy(qb)), to_cuda(torch.from_numpy(sb)), out_dtype=out_dtype)
        torch.cuda.synchronize()
        check_gemm(qa, sa, B.E4M3, qb, sb, B.E4M3, c, f"{M}x{N}x{K} {out_dtype}")


def test_gemm_consumes_the_gpu_quantizers_output():
    """x (bf16) -> 1x128 codes, w (bf16) -> 128x128 codes, both on the GPU, then the GEMM."""
    M, N, K = 512, 1024, 2048
    x = inputs.random_matrix(M, K, seed=5100, dtype=torch.bfloat16, outlier_frac=0.01, factor=1e2, device="cuda")
    w = (inputs.random_matrix(N, K, seed=5101, dtype=torch.float32, device="cuda") * 0.02).to(torch.bfloat16)
    qa, sa = B.fp8_quantize_blockwise(x, (1, 128), B.E4M3)
    qb, sb = B.fp8_quantize_blockwise(w, (128, 128), B.E4M3)
    c = B.fp8_gemm_blockwise(qa, sa, qb, sb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    check_gemm(qa.cpu().numpy(), sa.cpu().numpy(), B.E4M3, qb.cpu().numpy(), sb.cpu().numpy(), B.E4M3, c,
               "quantize -> gemm")
    # against the unquantized product: within the quantization error of both operands
    ref = x.double() @ w.double().T
    mag = x.double().abs() @ w.double().abs().T
    assert bool(((c.double() - ref).abs() <= 0.15 * mag).all())


def test_gemm_large_sampled_rows():
    M, N, K = 4096, 4096, 4096
    qa, sa, qb, sb = oracle_codes(M, N, K, B.E4M3, B.E4M3, seed=5200)
    c = B.fp8_gemm_blockwise(to_cuda(torch.from_numpy(qa)), to_cuda(torch.from_numpy(sa)),
                             to_cuda(torch.from_numpy(qb)), to_cuda(torch.from_numpy(sb)), out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 2047, 2900, 4094, 4095]
    check_gemm(qa, sa, B.E4M3, qb, sb, B.E4M3, c, "4096^3 sampled rows", rows=rows)


@pytest.mark.parametrize("b_block", [128, 1])
def test_gemm_more_tiles_than_pairs_row_tile_order(b_block):
    """M < N: the persistent CTA pairs take the tiles with the row tile fastest.  1024 x 8192 is 4 x 32 =
    128 pair tiles, more than the 74 pairs, so pairs take several tiles; sampled rows cover every row tile
    and every column tile."""
    M, N, K = 1024, 8192, 256
    x = inputs.random_matrix(M, K, seed=5150 + b_block, dtype=torch.bfloat16, outlier_frac=0.01, factor=1e2)
    w = inputs.random_matrix(N, K, seed=5160 + b_block, dtype=torch.bfloat16, scale=0.02, outlier_frac=0.01,
                             factor=1e2)
    qa, sa = oracle.quantize_blockwise(host_input(x), 1, 128, B.E4M3)
    qb, sb = oracle.quantize_blockwise(host_input(w), b_block, 128, B.E4M3)
    c = B.fp8_gemm_blockwise(to_cuda(torch.from_numpy(qa)), to_cuda(torch.from_numpy(sa)),
                             to_cuda(torch.from_numpy(qb)), to_cuda(torch.from_numpy(sb)), out_dtype=torch.float32,
                             b_block=b_block)
    torch.cuda.synchronize()
    rows = [0, 127, 128, 255, 256, 511, 512, 700, 767, 768, 1023]
    check_gemm(qa, sa, B.E4M3, qb, sb, B.E4M3, c, f"{M}x{N}x{K} B block {b_block}", rows=rows, b_block=b_block)


def test_gemm_k_zero_and_empty():
    a = torch.zeros(64, 0, dtype=torch.uint8, device="cuda")
    b = torch.zeros(256, 0, dtype=torch.uint8, device="cuda")
    s = torch.zeros(1, dtype=torch.float32, device="cuda")
    c = torch.full((64, 256), 7.0, dtype=torch.float32, device="cuda")
    B.fp8_gemm_blockwise(a, s, b, s, c=c)
    torch.cuda.synchronize()
    assert bool((c == 0).all())


@pytest.mark.parametrize("a_fmt,b_fmt", [(B.E5M2, B.E4M3), (B.E4M3, B.E5M2), (B.E5M2, B.E5M2)])
def test_gemm_mixed_formats(a_fmt, b_fmt):
    """kind::f8f6f4 takes each operand's format separately: E5M2 gradients against E4M3 activations."""
    for i, (M, N, K) in enumerate([(128, 256, 256), (384, 512, 768)]):
        qa, sa, qb, sb = oracle_codes(M, N, K, a_fmt, b_fmt, seed=5300 + 10 * i + 3 * a_fmt + b_fmt)
        c = B.fp8_gemm_blockwise(to_cuda(torch.from_numpy(qa)), to_cuda(torch.from_numpy(sa)),
                                 to_cuda(torch.from_numpy(qb)), to_cuda(torch.from_numpy(sb)), a_fmt=a_fmt,
                                 b_fmt=b_fmt, out_dtype=torch.float32)
        torch.cuda.synchronize()
        check_gemm(qa, sa, a_fmt, qb, sb, b_fmt, c, f"{M}x{N}x{K} fmts {a_fmt},{b_fmt}")


# -- B with 1x128 blocks: the weight-gradient form --------------------------------------------------

@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_b_1x128_matches_oracle(out_dtype):
    """Per-column, per-chunk B scales (sb [N, K/128]): the reciprocal ring and the two-factor promotion."""
    for i, (M, N, K) in enumerate(SHAPES + [(512, 1024, 1024)]):
        x = inputs.random_matrix(M, K, seed=5400 + i, dtype=torch.bfloat16, outlier_frac=0.01, factor=1e2)
        w = inputs.random_matrix(N, K, seed=5500 + i, dtype=torch.bfloat16, outlier_frac=0.01, factor=1e2)
        qa, sa = oracle.quantize_blockwise(host_input(x), 1, 128, B.E4M3)
        qb, sb = oracle.quantize_blockwise(host_input(w), 1, 128, B.E4M3)
        c = B.fp8_gemm_blockwise(to_cuda(torch.from_numpy(qa)), to_cuda(torch.from_numpy(sa)),
                                 to_cuda(torch.from_numpy(qb)), to_cuda(torch.from_numpy(sb)), out_dtype=out_dtype,
                                 b_block=1)
        torch.cuda.synchronize()
        check_gemm(qa, sa, B.E4M3, qb, sb, B.E4M3, c, f"1x128 B {M}x{N}x{K}", b_block=1)


def test_weight_gradient_from_the_transposing_quantizer():
    """dW = dY^T X: dY [T, out] (E5M2) and X [T, in] (E4M3) go through fp8_quantize_blockwise_transpose; its
    transposed outputs are the GEMM's operands, both 1x128 along the tokens."""
    T, n_out, n_in = 1024, 256, 512
    dy = inputs.random_matrix(T, n_out, seed=5600, dtype=torch.bfloat16, scale=1e-3, outlier_frac=1e-3, factor=1e2)
    x = inputs.random_matrix(T, n_in, seed=5601, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e2)
    _, _, qdt, sdt = B.fp8_quantize_blockwise_transpose(to_cuda(dy), (1, 128), B.E5M2)
    _, _, qxt, sxt = B.fp8_quantize_blockwise_transpose(to_cuda(x), (1, 128), B.E4M3)
    dw = B.fp8_gemm_blockwise(qdt, sdt, qxt, sxt, a_fmt=B.E5M2, b_fmt=B.E4M3, out_dtype=torch.float32, b_block=1)
    torch.cuda.synchronize()
    check_gemm(qdt.cpu().numpy(), sdt.cpu().numpy(), B.E5M2, qxt.cpu().numpy(), sxt.cpu().numpy(), B.E4M3, dw,
               "weight gradient", b_block=1)
    ref = dy.double().T @ x.double()
    mag = dy.double().abs().T @ x.double().abs()
    # E5M2 and E4M3 codes are within 2^-3 and 2^-4 of their inputs: 0.125 + 0.0625 + their product < 0.2
    assert bool(((dw.double().cpu() - ref).abs() <= 0.2 * mag).all())


def test_gemm_reports_no_wait_timeout():
    """After every GEMM above, the device status word has no wait-timeout bit."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = B.load_library().fp8_device_status(st.data_ptr(), 0, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) & B.DEVICE_STATUS_WAIT_TIMEOUT == 0
