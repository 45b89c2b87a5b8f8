"""GPU parity past the 32-bit index range: a bf16 tensor of [2^19 + 256, 4096] = 2^31 + 2^20 elements.

Element indices pass 2^31 and the input's byte offsets pass 2^31 (at element 2^30) and 2^32 (at element
2^31), so every kernel's index arithmetic must be 64-bit.  Expected values come from the oracle on whole
bands of rows: 256 rows around each of those crossings, the first and last 256 rows, and random rows
(block results depend only on their block).  The transposed copy is compared on the whole qt rows whose
flat index passes 2^31.  The per-tensor amax is the oracle's over the whole tensor.
"""
import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs
from parity_util import assert_bytes_equal, fp32_bits, host_input, oracle_amax

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

R, C = (1 << 19) + 256, 4096
EDGE = (1 << 31) // C  # the first row past element 2^31


HALF = (1 << 30) // C  # the first row whose bf16 byte offset passes 2^31
BANDS = [(0, 256), (HALF - 128, HALF + 128), (EDGE - 128, EDGE + 128), (R - 256, R)]


@pytest.fixture(scope="module")
def big():
    x = inputs.random_matrix(R, C, seed=31, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e3, device="cuda")
    rng = np.random.default_rng(31)
    band_rows = np.concatenate([np.arange(a, b) for a, b in BANDS])
    rows = np.unique(np.concatenate([band_rows, rng.integers(0, R, 24)]))
    tile_rows = np.unique(np.concatenate([[a // 128 + i for a, b in BANDS for i in range((b - a) // 128)],
                                          rng.integers(0, R // 128, 3)]))
    yield x, rows, tile_rows
    del x
    torch.cuda.empty_cache()


def host_rows(t, rows):
    return host_input(t[torch.as_tensor(rows, device=t.device)].cpu())


def test_max_size_1x128_and_dequant(big):
    x, rows, _ = big
    q, s = B.fp8_quantize_blockwise(x, (1, 128), B.E4M3)
    y = B.fp8_dequantize(q, s, (1, 128), B.E4M3, torch.bfloat16)
    xh = host_rows(x, rows)
    oq, os_ = oracle.quantize_blockwise(xh, 1, 128, oracle.E4M3)
    idx = torch.as_tensor(rows, device="cuda")
    assert_bytes_equal(q[idx], oq, "1x128 codes")
    assert_bytes_equal(s[idx], fp32_bits(os_), "1x128 scales")
    assert_bytes_equal(y[idx], oracle.dequantize(oq, oracle.E4M3, os_, 1, 128, oracle.BF16), "1x128 dequant")
    # every block holds a top code (each block's amax maps to MAX)
    top = oracle.top_code(oracle.E4M3)
    assert bool(((q & 0x7F).view(R, C // 128, 128).amax(dim=2) == top).all())


def test_max_size_128x128_and_dequant(big):
    x, _, tile_rows = big
    q, s = B.fp8_quantize_blockwise(x, (128, 128), B.E4M3)
    y = B.fp8_dequantize(q, s, (128, 128), B.E4M3, torch.bfloat16)
    for tr in tile_rows:
        sl = slice(int(tr) * 128, int(tr) * 128 + 128)
        oq, os_ = oracle.quantize_blockwise(host_input(x[sl].cpu()), 128, 128, oracle.E4M3)
        assert_bytes_equal(q[sl], oq, f"128x128 tile row {tr} codes")
        assert_bytes_equal(s[int(tr):int(tr) + 1], fp32_bits(os_), f"128x128 tile row {tr} scales")
        assert_bytes_equal(y[sl], oracle.dequantize(oq, oracle.E4M3, os_, 128, 128, oracle.BF16),
                           f"128x128 tile row {tr} dequant")


def test_max_size_per_tensor_current_and_dequant(big):
    x, rows, _ = big
    q, s, a = B.fp8_quantize_per_tensor(x, B.E5M2)
    oa = oracle_amax(host_input(x.cpu()))
    os_ = oracle.scale_from_amax(oa, oracle.E5M2)
    assert_bytes_equal(a, fp32_bits([oa]), "amax")
    assert_bytes_equal(s, fp32_bits([os_]), "scale")
    y = B.fp8_dequantize(q, s, (0, 0), B.E5M2, torch.bfloat16)
    idx = torch.as_tensor(rows, device="cuda")
    xh = host_rows(x, rows)
    oq, _, _ = oracle.quantize_per_tensor(xh, oracle.E5M2, scale=float(os_))
    assert_bytes_equal(q[idx], oq, "per-tensor codes")
    assert_bytes_equal(y[idx], oracle.dequantize(oq, oracle.E5M2, np.array([os_], np.float32), 0, 0, oracle.BF16),
                       "per-tensor dequant")


def test_max_size_mx_and_dequant(big):
    x, rows, _ = big
    q, e8 = B.fp8_quantize_mx(x, B.E4M3, B.MX_FIT)
    y = B.fp8_dequantize_mx(q, e8, B.E4M3, torch.bfloat16)
    idx = torch.as_tensor(rows, device="cuda")
    oq, oe = oracle.quantize_mx(host_rows(x, rows), oracle.E4M3, oracle.MX_FIT)
    assert_bytes_equal(q[idx], oq, "MX codes")
    assert_bytes_equal(e8[idx], oe, "MX scale bytes")
    assert_bytes_equal(y[idx], oracle.dequantize_mx(oq, oracle.E4M3, oe, oracle.BF16), "MX dequant")


def test_max_size_fake_quant_and_delayed_step(big):
    x, rows, _ = big
    idx = torch.as_tensor(rows, device="cuda")
    xh = host_rows(x, rows)
    y = B.fp8_fake_quantize(x, (1, 128), B.E4M3)
    oq, os_ = oracle.quantize_blockwise(xh, 1, 128, oracle.E4M3)
    assert_bytes_equal(y[idx], oracle.dequantize(oq, oracle.E4M3, os_, 1, 128, oracle.BF16), "fake quant")
    del y
    # one delayed step in one launch: the cast uses the given scale; amax over the whole tensor
    sc = B.DelayedScaler(window=2, fmt=B.E5M2)
    sc.scale.fill_(0.5)
    q, used = sc.step(x)
    oa = oracle_amax(host_input(x.cpu()))
    assert_bytes_equal(used, fp32_bits([0.5]), "scale used")
    assert_bytes_equal(sc.amax, fp32_bits([oa]), "delayed amax")
    oq, _, _ = oracle.quantize_per_tensor(xh, oracle.E5M2, scale=0.5)
    assert_bytes_equal(q[idx], oq, "delayed codes")


def test_max_size_transpose(big):
    x, rows, _ = big
    q, qt, s, a = B.fp8_quantize_per_tensor_transpose(x, B.E4M3, torch.tensor([0.25], device="cuda"))
    idx = torch.as_tensor(rows, device="cuda")
    oq, _, _ = oracle.quantize_per_tensor(host_rows(x, rows), oracle.E4M3, scale=0.25)
    assert_bytes_equal(q[idx], oq, "transpose q rows")
    # qt column r is q row r
    assert_bytes_equal(qt[:, idx].t().contiguous(), oq, "transpose qt columns")
    # the whole qt rows whose flat index c * R + r passes 2^31 (and the last one): x's columns c
    c0 = (1 << 31) // R
    assert c0 * R < (1 << 31) < (c0 + 1) * R
    for c in sorted({c0, C - 1}):
        oqc, _, _ = oracle.quantize_per_tensor(host_input(x[:, c].contiguous().cpu()), oracle.E4M3, scale=0.25)
        assert_bytes_equal(qt[c], oqc, f"transpose qt row {c}")
