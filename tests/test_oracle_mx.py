"""Pins of the oracle's MX (1x32, power-of-two scale) quantization.

Mixed-precision handbook, section "FP8 training", closing notes: Blackwell's
MX formats let each run of 32 elements share one scale factor in hardware.
The scale is a power of two 2^k, stored as the E8M0 byte 127 - k of the
dequant multiplier 2^-k.  The two rules for k (fit: largest 2^k with
amax * 2^k <= MAX; OCP: k = emax_elem - floor(log2 amax)) are checked here
against hand-computed bytes, against inequalities evaluated a different way
(numpy float64 ldexp / log2), and against the already pinned 1x32 blockwise
quantizer in the cases where both must agree.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import E4M3, E5M2, MX_FIT, MX_OCP

MAX = {E4M3: 448.0, E5M2: 57344.0}
EMAX = {E4M3: 8, E5M2: 15}
HALF_ULP_REL = {E4M3: 2.0 ** -4, E5M2: 2.0 ** -3}
MIN_NORMAL = {E4M3: 2.0 ** -6, E5M2: 2.0 ** -14}


def _byte_of_block(amax, fmt, rule):
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 5] = amax
    return int(oracle.quantize_mx(x, fmt, rule)[1][0, 0])


# (fmt, rule, amax, expected byte), each worked out by hand:
HAND = [
    (E4M3, MX_FIT, 1.0, 119),          # 256 <= 448 < 512: k = 8
    (E4M3, MX_FIT, 1.75, 119),         # 1.75 * 256 = 448 exactly: k = 8
    (E4M3, MX_FIT, 1.7500001, 120),    # just above 448 at k = 8: k = 7
    (E4M3, MX_FIT, 448.0, 127),        # k = 0, byte 127 is the multiplier 1
    (E4M3, MX_FIT, 0.001, 109),        # 2^18 = 262144 <= 448000 < 2^19: k = 18
    (E4M3, MX_FIT, 0.0, 79),           # eps 1e-12: 2^48 <= 4.48e14 < 2^49: k = 48
    (E4M3, MX_OCP, 1.0, 119),          # floor(log2 1) = 0: k = 8
    (E4M3, MX_OCP, 1.9, 119),          # floor(log2 1.9) = 0: k = 8 (1.9 * 256 saturates)
    (E4M3, MX_OCP, 448.0, 127),        # floor(log2 448) = 8: k = 0
    (E4M3, MX_OCP, 512.0, 128),        # floor(log2 512) = 9: k = -1
    (E4M3, MX_OCP, 0.001, 109),        # floor(log2 0.001) = -10: k = 18
    (E5M2, MX_FIT, 1.0, 112),          # 2^15 = 32768 <= 57344 < 2^16: k = 15
    (E5M2, MX_FIT, 57344.0, 127),      # k = 0
    (E5M2, MX_FIT, 60000.0, 128),      # 60000 > 57344: k = -1
    (E5M2, MX_OCP, 60000.0, 127),      # floor(log2 60000) = 15: k = 0 (saturates)
    (E5M2, MX_FIT, 0.0, 72),           # 2^55 <= 5.7344e16 < 2^56: k = 55
    (E4M3, MX_FIT, float("inf"), 255),  # no power of two fits: the NaN byte
    (E5M2, MX_OCP, float("inf"), 255),
]


@pytest.mark.parametrize("fmt,rule,amax,byte", HAND)
def test_scale_byte_matches_hand_computed(fmt, rule, amax, byte):
    assert _byte_of_block(amax, fmt, rule) == byte


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_exponent_rules_hold_as_inequalities(fmt):
    rng = np.random.default_rng(11)
    amaxes = np.ldexp(rng.uniform(1.0, 2.0, 4000), rng.integers(-39, 120, 4000)).astype(np.float32)
    # add the binade edges and the 1.75 boundary of both formats' MAX
    edges = [np.float32(np.ldexp(m, e)) for e in range(-30, 100, 7) for m in (1.0, 1.75, 2.0 - 2.0 ** -23)]
    amaxes = np.concatenate([amaxes, np.array(edges, dtype=np.float32),
                             np.nextafter(np.array(edges, dtype=np.float32), np.float32(np.inf))])
    for a in amaxes:
        a64 = float(a)
        k = oracle.mx_exponent(a, fmt, MX_FIT)
        assert np.ldexp(a64, k) <= MAX[fmt] < np.ldexp(a64, k + 1), (a64, k)
        k1 = oracle.mx_exponent(a, fmt, MX_OCP)
        assert 2.0 ** EMAX[fmt] <= np.ldexp(a64, k1) < 2.0 ** (EMAX[fmt] + 1), (a64, k1)
        # the rules differ exactly when a's significand is above MAX's (1.75)
        sig = a64 / 2.0 ** math.floor(math.log2(a64))
        assert (k1 - k) == (1 if sig > 1.75 else 0), (a64, k, k1)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("cols", [32, 96, 100, 7])
def test_power_of_two_ratio_matches_blockwise_1x32(fmt, cols):
    """Blocks whose amax is MAX / 2^k: the fit scale is exactly the pages'
    MAX / amax, so codes and scales equal those of 1x32 blockwise scaling."""
    rng = np.random.default_rng(12 + cols)
    rows = 5
    x = rng.uniform(-1.0, 1.0, (rows, cols)).astype(np.float32)
    nb = math.ceil(cols / 32)
    ks = rng.integers(-20, 30, (rows, nb))
    for r in range(rows):
        for b in range(nb):
            c0, c1 = 32 * b, min(32 * b + 32, cols)
            amax = MAX[fmt] * 2.0 ** -int(ks[r, b])
            x[r, c0:c1] *= np.float32(amax * 0.999)
            x[r, c0 + int(rng.integers(0, c1 - c0))] = np.float32(-amax if (r + b) % 2 else amax)
    q, e = oracle.quantize_mx(x, fmt, MX_FIT)
    qb, sb = oracle.quantize_blockwise(x, 1, 32, fmt)
    assert np.array_equal(q, qb)
    assert np.array_equal(e.astype(np.int64), 127 - ks)
    assert np.array_equal(sb, np.ldexp(np.float32(1.0), ks).astype(np.float32))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("rule", [MX_FIT, MX_OCP])
def test_dequant_equals_blockwise_division_by_the_scale(fmt, rule):
    """decode(q) * 2^(byte - 127) and decode(q) / 2^k are the same real number,
    so the MX dequant must equal the pinned blockwise dequant given s = 2^k."""
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((6, 160)) * np.exp(rng.uniform(-20, 20, (6, 1)))).astype(np.float32)
    q, e = oracle.quantize_mx(x, fmt, rule)
    s = np.ldexp(np.float32(1.0), 127 - e.astype(np.int64)).astype(np.float32)
    for out in (oracle.F32, oracle.BF16):
        y = oracle.dequantize_mx(q, fmt, e, out)
        yb = oracle.dequantize(q, fmt, s, 1, 32, out)
        assert np.array_equal(y, yb)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_fit_round_trip_error_and_range_use(fmt):
    rng = np.random.default_rng(14)
    x = (rng.standard_normal((8, 256)) * np.exp(rng.uniform(-8, 8, (8, 256)))).astype(np.float32)
    q, e = oracle.quantize_mx(x, fmt, MX_FIT)
    y = oracle.dequantize_mx(q, fmt, e).astype(np.float64)
    dec = oracle.decode_table(fmt)[q]
    k = 127 - e.astype(np.int64)
    kx = np.repeat(k, 32, axis=1)
    scaled = np.abs(x.astype(np.float64)) * np.ldexp(1.0, kx)
    normal = scaled >= MIN_NORMAL[fmt]
    err = np.abs(y - x)
    assert np.all(err[normal] <= HALF_ULP_REL[fmt] * np.abs(x[normal].astype(np.float64)) * (1 + 1e-12))
    # fit never saturates: every decoded magnitude stays within MAX, and the
    # block's largest element lands in the top binade of the range (k is the
    # largest exponent that fits, so 2^(k+1) would overflow)
    assert np.all(np.abs(dec) <= MAX[fmt])
    top = np.abs(dec).reshape(8, 8, 32).max(axis=2)
    assert np.all(top >= MAX[fmt] / 2 / (1 + HALF_ULP_REL[fmt]))


def test_special_blocks():
    x = np.ones((2, 64), dtype=np.float32)
    x[0, 3] = np.inf     # block (0, 0) holds Inf
    x[1, 32:] = 0.0      # block (1, 1) is all zeros
    for fmt in (E4M3, E5M2):
        q, e = oracle.quantize_mx(x, fmt, MX_FIT)
        assert e[0, 0] == 0xFF
        assert e[1, 1] == 127 - (48 if fmt == E4M3 else 55)
        assert np.all(q[1, 32:] == 0)
        y = oracle.dequantize_mx(q, fmt, e)
        assert np.all(np.isnan(y[0, :32]))
        assert np.all(y[0, 32:] == 1.0) and np.all(y[1, :32] == 1.0) and np.all(y[1, 32:] == 0.0)


def test_bf16_input_widens_exactly():
    rng = np.random.default_rng(15)
    bits = (rng.integers(0, 1 << 16, (4, 96)) & 0xFFFF).astype(np.uint16)
    bits[(bits & 0x7F80) == 0x7F80] = 0x3F80  # no Inf/NaN patterns
    wide = (bits.astype(np.uint32) << 16).view(np.float32)
    for fmt in (E4M3, E5M2):
        for rule in (MX_FIT, MX_OCP):
            q1, e1 = oracle.quantize_mx(bits, fmt, rule)
            q2, e2 = oracle.quantize_mx(wide, fmt, rule)
            assert np.array_equal(q1, q2) and np.array_equal(e1, e2)
