"""Pins for the oracle's FP8 decode / encode, against things other than itself.

- the format table of the PyTorch-FP8 page, s1.2 (constants, exhaustively)
- torch's own CPU float8 dtypes (decode of every code; RNE cast in range)
- a brute-force nearest-value search in exact rational arithmetic
- the closed-form error bound of round-to-nearest
- the scalar experiment of the PyTorch-FP8 page, s2.2
"""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_rows

FMTS = {"e4m3fn": oracle.E4M3, "e5m2": oracle.E5M2}
TORCH_FP8 = {oracle.E4M3: torch.float8_e4m3fn, oracle.E5M2: torch.float8_e5m2}


def table():
    out = {}
    for name, sign, eb, mb, bias, mx, mn_exp, sub_exp in golden_rows("format_table.txt"):
        out[FMTS[name]] = dict(exp_bits=int(eb), man_bits=int(mb), bias=int(bias), max=float(mx),
                               min_normal=2.0 ** int(mn_exp), min_sub=2.0 ** int(sub_exp))
    return out


def f32(v):
    return struct.unpack("<f", struct.pack("<f", v))[0]


def torch_decode_all(fmt):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(TORCH_FP8[fmt]).to(torch.float64).numpy()


def torch_encode(vals, fmt):
    t = torch.as_tensor(np.asarray(vals, dtype=np.float32))
    return t.to(TORCH_FP8[fmt]).view(torch.uint8).numpy()


def test_selfcheck():
    assert oracle.lib().orc_selfcheck() == 0


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_format_table_constants(fmt):
    t = table()[fmt]
    vals = oracle.decode_table(fmt)
    pos = vals[:128]
    finite = pos[np.isfinite(pos)]
    # largest finite value and its code
    assert finite.max() == t["max"]
    top = oracle.top_code(fmt)
    assert vals[top] == t["max"]
    assert top == {oracle.E4M3: 0x7E, oracle.E5M2: 0x7B}[fmt]
    # smallest subnormal is code 1; smallest normal is the first code with exponent field 1
    assert vals[1] == t["min_sub"]
    assert vals[1 << t["man_bits"]] == t["min_normal"]
    # 1.0 sits at exponent field == bias, mantissa 0
    assert vals[t["bias"] << t["man_bits"]] == 1.0
    # each binade holds 2^man_bits codes: code + 2^M doubles the value across the normal range
    M = t["man_bits"]
    for c in range(1 << M, top + 1 - (1 << M)):
        assert vals[c + (1 << M)] == 2 * vals[c]
    # subnormals are evenly spaced by the smallest subnormal
    for c in range(1, 1 << M):
        assert vals[c] == c * t["min_sub"]
    # zero and negative zero
    assert vals[0] == 0.0 and math.copysign(1.0, vals[0x80]) == -1.0


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_decode_matches_torch_every_code(fmt):
    ours = oracle.decode_table(fmt)
    ref = torch_decode_all(fmt)
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(ours[~both_nan], ref[~both_nan])


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_decode_sign_symmetry_and_order(fmt):
    vals = oracle.decode_table(fmt)
    top = oracle.top_code(fmt)
    for c in range(0, top + 1):
        assert vals[c | 0x80] == -vals[c]
    assert np.all(np.diff(vals[: top + 1]) > 0)
    # no finite code above top; the E4M3 all-ones code is NaN, E5M2 keeps Inf and NaN
    if fmt == oracle.E4M3:
        assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    else:
        assert vals[0x7C] == math.inf and vals[0xFC] == -math.inf
        assert all(np.isnan(vals[c]) for c in (0x7D, 0x7E, 0x7F))


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_decode_identity(fmt):
    top = oracle.top_code(fmt)
    for c in list(range(top + 1)) + [c | 0x80 for c in range(top + 1)]:
        v = oracle.decode(c, fmt)
        assert oracle.encode(v, fmt) == c, hex(c)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_all_bf16_patterns_vs_torch(fmt):
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    mx = oracle.MAX[fmt]
    keep = np.isfinite(v) & (np.abs(v) <= mx)
    v = v[keep]
    ours = oracle.encode_array(v, fmt)
    ref = torch_encode(v, fmt)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(ours[i]), hex(ref[i])) for i in bad[:10]]


def _exact_nearest(v, fmt, values):
    """Brute force: exact nearest value among all finite codes, ties to the even code, |v| clamped to max."""
    sign = 0x80 if math.copysign(1.0, v) < 0 else 0
    a = Fraction(abs(v))
    a = min(a, Fraction(oracle.MAX[fmt]))
    best = None
    for c, val in values:
        d = abs(Fraction(val) - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_midpoints_brute_force(fmt):
    # value set from torch (a library decode), not from the oracle
    ref_vals = torch_decode_all(fmt)
    values = [(c, ref_vals[c]) for c in range(128) if np.isfinite(ref_vals[c])]
    probes = []
    for (c0, v0), (c1, v1) in zip(values, values[1:]):
        mid = f32((v0 + v1) / 2)
        assert mid == (v0 + v1) / 2  # midpoints of 4-bit values are exact in fp32
        for p in (mid, np.nextafter(np.float32(mid), np.float32(0)),
                  np.nextafter(np.float32(mid), np.float32(np.inf)), v0, v1):
            probes += [float(p), -float(p)]
    probes += [0.0, -0.0, oracle.MAX[fmt] * 1.0001, 1e30, 7e-46]
    for p in probes:
        p = f32(p)
        assert oracle.encode(p, fmt) == _exact_nearest(p, fmt, values), p


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_random_fp32_vs_torch(fmt):
    rng = np.random.default_rng(1234 + fmt)
    mx = oracle.MAX[fmt]
    # log-uniform magnitudes across the whole range including fp32 subnormals, random sign
    e = rng.uniform(-150, math.log2(mx), size=200_000)
    v = (np.exp2(e) * rng.choice([-1.0, 1.0], size=e.size)).astype(np.float32)
    v = v[np.abs(v) <= mx]
    ours = oracle.encode_array(v, fmt)
    ref = torch_encode(v, fmt)
    assert np.array_equal(ours, ref)


def nearest_code_rule(v: np.ndarray, fmt: int, t: dict) -> np.ndarray:
    """The encoding's definition, vectorised in float64 and written from the format table alone.

    The finite magnitudes of the table, in code order, are searched for the two neighbours of |v|; the
    nearer one wins, a tie goes to the even code, and anything beyond the largest value takes the largest
    code.  The sign bit of v is the code's sign bit (so -0 and negatives that round to zero give 0x80).
    Every quantity is exact in float64: v is an fp32 value and the table's values have 4 significant bits."""
    M, bias = t["man_bits"], t["bias"]
    # magnitudes grow with the code; the finite ones are those up to the table's largest value
    vals = np.array([v_ for v_ in (_table_value(c, M, bias) for c in range(128)) if v_ <= t["max"]])
    top = vals.size - 1
    a = np.abs(v.astype(np.float64))
    hi = np.minimum(np.searchsorted(vals, a, side="left"), top)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - vals[lo], vals[hi] - a
    pick = np.where(d_hi < d_lo, hi, lo)
    tie = (d_hi == d_lo) & (hi != lo)
    pick = np.where(tie, np.where(hi % 2 == 0, hi, lo), pick)
    pick = np.where(a >= vals[top], top, pick)
    pick = np.where(a <= 0.0, 0, pick)
    sign = (v.view(np.uint32) >> 31).astype(np.int64) << 7
    return (pick | sign).astype(np.uint8)


def _table_value(code: int, M: int, bias: int) -> float:
    e, m = code >> M, code & ((1 << M) - 1)
    if e == 0:
        return m * 2.0 ** (1 - bias - M)
    return (1 + m / 2 ** M) * 2.0 ** (e - bias)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encode_ten_million_random_fp32_vs_nearest_code_rule(fmt):
    """10^7 random fp32 values (log-uniform magnitudes from the fp32 subnormals to 4x the format's
    largest value, random sign, plus random bit patterns of finite fp32 values) against the encoding's
    definition: nearest finite code, ties to the even code, saturation beyond the largest value."""
    t = table()[fmt]
    rng = np.random.default_rng(7_000_000 + fmt)
    n = 10_000_000
    e = rng.uniform(-152, math.log2(t["max"]) + 2, size=n - n // 10)
    v = (np.exp2(e) * rng.choice([-1.0, 1.0], size=e.size)).astype(np.float32)
    bits = rng.integers(0, 1 << 32, size=n // 10, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]  # finite patterns only
    v = np.concatenate([v, bits.view(np.float32)])
    want = nearest_code_rule(v, fmt, t)
    got = oracle.encode_array(v, fmt)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{bad.size} mismatches, first {v[bad[0]]!r}: got {got[bad[0]]:#x} want {want[bad[0]]:#x}"


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_saturation(fmt):
    top = oracle.top_code(fmt)
    mx = oracle.MAX[fmt]
    for v in (mx, mx * 1.0001, mx * 1.07, mx * 1.2, 1e6, 3.0e38, math.inf):
        assert oracle.encode(v, fmt) == top
        assert oracle.encode(-v, fmt) == 0x80 | top
    if fmt == oracle.E4M3:
        assert oracle.encode(449.0, fmt) == 0x7E
        assert oracle.encode(1e4, fmt) == 0x7E
    else:
        assert oracle.encode(6e4, fmt) == 0x7B


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_round_to_nearest_error_bound(fmt):
    """|decode(encode(x)) - x| <= half the code spacing at x (closed form from the format table)."""
    t = table()[fmt]
    M = t["man_bits"]
    rng = np.random.default_rng(99 + fmt)
    e = rng.uniform(-20, math.log2(t["max"]), size=50_000)
    v = np.exp2(e).astype(np.float32)
    v = v[v <= t["max"]]
    q = oracle.encode_array(v, fmt)
    dec = oracle.decode_table(fmt)[q]
    err = np.abs(dec - v.astype(np.float64))
    normal = v >= t["min_normal"]
    spacing = np.where(normal, np.exp2(np.floor(np.log2(v.astype(np.float64))) - M), t["min_sub"])
    assert np.all(err <= spacing / 2)
    # relative bound on the normal range: 2^-(M+1)
    assert np.all(err[normal] / v[normal] <= 2.0 ** -(M + 1))


def test_scalar_experiment_facts():
    """The page's scalar experiment (PyTorch-FP8 page, s2.2), with round-to-nearest-even pinned."""
    t = table()
    for value, e4, e5 in golden_rows("scalar_experiment.txt"):
        v = f32(float(value))
        for fmt, fact in ((oracle.E4M3, e4), (oracle.E5M2, e5)):
            got = oracle.decode(oracle.encode(v, fmt), fmt)
            if fact == "-":
                continue
            if fact == "exact":
                assert got == v, (value, fmt)
            elif fact == "inexact":
                assert got != v, (value, fmt)
            elif fact.startswith("one_of:"):
                allowed = [float(a) for a in fact.split(":", 1)[1].split("|")]
                assert got in allowed, (value, fmt, got)
            elif fact == "zero_or_subnormal":
                assert got == 0.0 or abs(got) < t[fmt]["min_normal"], (value, fmt, got)
            elif fact == "nonzero":
                assert got != 0.0, (value, fmt)
            else:
                raise AssertionError(f"unknown fact {fact}")
    # the nearest choice where the page allows two: 1.1 is 0.025 from 1.125 and 0.1 from 1.0
    assert oracle.decode(oracle.encode(1.1, oracle.E4M3), oracle.E4M3) == 1.125
    # the page's minimum normal lands exactly on code 0x08
    assert oracle.encode(0.015625, oracle.E4M3) == 0x08
    # a true tie: 1.125 lies halfway between E5M2's 1.0 and 1.25 and goes to the even code (1.0)
    assert oracle.encode(1.125, oracle.E5M2) == 0x3C


def test_bf16_rounding_vs_torch():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    # add exact ties and near-ties
    base = rng.integers(0, 2**16, size=20_000, dtype=np.uint64).astype(np.uint32) << 16
    bits = np.concatenate([bits, base | 0x8000, base | 0x7FFF, base | 0x8001])
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    L = oracle.lib()
    ours = np.array([L.orc_f32_to_bf16(float(x)) for x in v[:5000]], dtype=np.uint16)
    assert np.array_equal(ours, ref[:5000])
    # bulk check through dequantize's bf16 path is in the scaling tests; widen is exact
    for h in (0x0000, 0x8000, 0x3F80, 0x7F7F, 0x0001, 0xC2F7):
        assert np.float32(L.orc_bf16_to_f32(h)).view(np.uint32) == (h << 16)
