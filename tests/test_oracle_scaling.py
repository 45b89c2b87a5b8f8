"""Pins for the oracle's scaling modes (amax, scale, quantize, dequantize, history).

What pins them, other than the oracle itself:
- the relative-error table printed by the handbook page ("FP8 training")
- the handbook's exercise 2 (0.01 under a 5000 outlier becomes 0)
- torch CPU ops restating the handbook's per_tensor / per_block steps (reshape,
  amax, clamp, the library's float8 cast) with this library's multiply form
- the closed form of delayed scaling (PyTorch-FP8 page, s4.2 DelayedScaler)
- invariants: each block whose amax is above eps holds a +-max code; an all
  zero block gives code 0 and scale max/eps
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_rows
from fine_grained_block_b200 import inputs

TORCH_FP8 = {oracle.E4M3: torch.float8_e4m3fn, oracle.E5M2: torch.float8_e5m2}
EPS32 = np.float32(1e-12)


def rel_err(q, x):
    q = np.asarray(q, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    return float(np.linalg.norm(q - x) / np.linalg.norm(x))


# -- handbook "FP8 training": per-tensor vs 1x128 relative error ----------------

def test_handbook_relative_error_table():
    printed = {float(f): (float(t), float(b)) for f, t, b in golden_rows("p3_relerr.txt")}
    for factor, a in inputs.relerr_outlier_tensors():
        x = a.numpy()
        q, s, _ = oracle.quantize_per_tensor(x, oracle.E4M3)
        y_t = oracle.dequantize(q, oracle.E4M3, np.array([s]))
        qb, sb = oracle.quantize_blockwise(x, 1, 128, oracle.E4M3)
        y_b = oracle.dequantize(qb, oracle.E4M3, sb, 1, 128)
        t = rel_err(y_t[:, 128:], x[:, 128:]) * 100
        b = rel_err(y_b[:, 128:], x[:, 128:]) * 100
        want_t, want_b = printed[factor]
        # the page prints one decimal
        assert round(t, 1) == want_t, (factor, t)
        assert round(b, 1) == want_b, (factor, b)
    # per-tensor error grows with the outlier; the block error stays at the format's precision
    errs = []
    for factor, a in inputs.relerr_outlier_tensors():
        x = a.numpy()
        q, s, _ = oracle.quantize_per_tensor(x, oracle.E4M3)
        errs.append(rel_err(oracle.dequantize(q, oracle.E4M3, np.array([s]))[:, 128:], x[:, 128:]))
    assert errs[0] < errs[1] < errs[2]


def test_handbook_exercise_small_value_flushes():
    for amax, value, fmt, expect in golden_rows("exercise_outlier.txt"):
        assert fmt == "e4m3fn"
        rng = np.random.default_rng(5)
        x = rng.uniform(-1, 1, size=4096).astype(np.float32)
        x[17] = np.float32(amax)
        x[100] = np.float32(value)
        q, s, a = oracle.quantize_per_tensor(x, oracle.E4M3)
        assert a == np.float32(amax)
        assert s == np.float32(448.0 / float(amax))
        got = oracle.decode(int(q[100]), oracle.E4M3)
        assert got == float(expect) and math.copysign(1, got) == math.copysign(1, float(expect))
        # the page's reasoning: value * s is below half the smallest subnormal
        assert abs(float(value)) * float(s) < 2.0 ** -10
        # and a good share of the values in [-1, 1] land in the subnormal range or at 0,
        # keeping at most the 3 mantissa bits of a subnormal
        dec = oracle.decode_table(oracle.E4M3)[q]
        small = np.abs(x) < 1
        assert np.mean(np.abs(dec[small]) < 2.0 ** -6) > 0.1


# -- torch restatements of the handbook's per_tensor / per_block -------------------

def torch_blockwise(x: torch.Tensor, br: int, bc: int, fmt: int):
    """The handbook's per_block with reshape / amax / clamp(1e-12), scale = MAX / amax multiplied in.

    Ragged edges are handled by zero padding (zeros never raise an amax)."""
    MAX = oracle.MAX[fmt]
    x = x.to(torch.float32)
    R, C = x.shape
    Rp, Cp = -(-R // br) * br, -(-C // bc) * bc
    xp = torch.zeros(Rp, Cp, dtype=torch.float32)
    xp[:R, :C] = x
    b = xp.reshape(Rp // br, br, Cp // bc, bc)
    amax = b.abs().amax(dim=(1, 3), keepdim=True).clamp(min=1e-12)
    s = torch.tensor(MAX, dtype=torch.float32) / amax
    q = (b * s).clamp(-MAX, MAX).to(TORCH_FP8[fmt]).view(torch.uint8)
    return q.reshape(Rp, Cp)[:R, :C].numpy(), s.reshape(Rp // br, Cp // bc).numpy()


def torch_per_tensor(x: torch.Tensor, fmt: int, scale=None):
    MAX = oracle.MAX[fmt]
    x = x.to(torch.float32)
    amax = x.abs().max() if x.numel() else torch.tensor(0.0)
    s = (torch.tensor(MAX, dtype=torch.float32) / amax.clamp(min=1e-12)) if scale is None \
        else torch.tensor(scale, dtype=torch.float32)
    q = (x * s).clamp(-MAX, MAX).to(TORCH_FP8[fmt]).view(torch.uint8)
    return q.numpy(), s.item(), amax.item()


def as_oracle_input(t: torch.Tensor):
    if t.dtype == torch.bfloat16:
        return inputs.bf16_bits(t)
    return t.numpy()


SHAPES = [(1, 128), (3, 256), (128, 128), (130, 384), (257, 640), (64, 100), (200, 77), (5, 1)]


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("block", [(1, 128), (128, 128)])
def test_blockwise_vs_torch_handbook_form(fmt, dtype, block):
    br, bc = block
    for i, (R, C) in enumerate(SHAPES):
        x = inputs.random_matrix(R, C, seed=100 + i, dtype=dtype, outlier_frac=0.01, factor=1e3)
        q, s = oracle.quantize_blockwise(as_oracle_input(x), br, bc, fmt)
        qt, st = torch_blockwise(x, br, bc, fmt)
        assert np.array_equal(s, st), (R, C)
        assert np.array_equal(q, qt), (R, C)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_per_tensor_vs_torch_handbook_form(fmt, dtype):
    for i, n in enumerate([1, 7, 128, 1000, 65537]):
        x = inputs.random_matrix(1, n, seed=200 + i, dtype=dtype, outlier_frac=0.002, factor=1e4)
        q, s, a = oracle.quantize_per_tensor(as_oracle_input(x), fmt)
        qt, st, at = torch_per_tensor(x, fmt)
        assert a == np.float32(at) and s == np.float32(st)
        assert np.array_equal(q, qt)
        # delayed form: a given scale, values may saturate
        q2, s2, a2 = oracle.quantize_per_tensor(as_oracle_input(x), fmt, scale=3.0)
        qt2, _, _ = torch_per_tensor(x, fmt, scale=3.0)
        assert s2 == np.float32(3.0) and a2 == a
        assert np.array_equal(q2, qt2)


def test_empty_inputs():
    q, s, a = oracle.quantize_per_tensor(np.zeros(0, dtype=np.float32), oracle.E4M3)
    assert q.size == 0 and a == 0.0 and s == np.float32(448.0 / np.float64(EPS32))
    q, s = oracle.quantize_blockwise(np.zeros((0, 256), dtype=np.float32), 1, 128, oracle.E4M3)
    assert q.size == 0 and s.shape == (0, 2)
    q, s = oracle.quantize_blockwise(np.zeros((4, 0), dtype=np.float32), 128, 128, oracle.E4M3)
    assert q.size == 0 and s.shape == (1, 0)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_block_invariants(fmt):
    top = oracle.top_code(fmt)
    x = inputs.random_matrix(256, 512, seed=11, dtype=torch.bfloat16, outlier_frac=0.003, factor=1e3)
    xb = inputs.bf16_bits(x).copy()
    # zero out a whole 1x128 block and a whole 128x128 block
    xb[5, 128:256] = 0
    xb[128:256, 384:512] = 0x8000  # negative zeros
    for br, bc in ((1, 128), (128, 128)):
        q, s = oracle.quantize_blockwise(xb, br, bc, fmt)
        for bi in range(s.shape[0]):
            for bj in range(s.shape[1]):
                blk = q[bi * br:(bi + 1) * br, bj * bc:(bj + 1) * bc]
                xv = (xb[bi * br:(bi + 1) * br, bj * bc:(bj + 1) * bc].astype(np.uint32) << 16).view(np.float32)
                if np.abs(xv).max() == 0:
                    assert s[bi, bj] == np.float32(oracle.MAX[fmt] / np.float64(EPS32))
                    assert np.all((blk & 0x7F) == 0)
                else:
                    assert np.any((blk & 0x7F) == top), (br, bi, bj)
                    assert np.all((blk & 0x7F) <= top)


# -- dequantize ---------------------------------------------------------------

@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_dequantize_vs_torch(fmt):
    rng = np.random.default_rng(21 + fmt)
    top = oracle.top_code(fmt)
    R, C = 256, 384
    codes = rng.integers(0, top + 1, size=(R, C)).astype(np.uint8) | (rng.integers(0, 2, size=(R, C)) * 0x80).astype(np.uint8)
    scales_1x128 = np.exp2(rng.uniform(-30, 40, size=(R, 3))).astype(np.float32)
    scales_128 = np.exp2(rng.uniform(-30, 40, size=(2, 3))).astype(np.float32)
    qv = torch.from_numpy(codes).view(TORCH_FP8[fmt]).to(torch.float32)
    cases = [
        (1, 128, scales_1x128, torch.from_numpy(np.repeat(scales_1x128, 128, axis=1))),
        (128, 128, scales_128, torch.from_numpy(np.repeat(np.repeat(scales_128, 128, 0), 128, 1))),
        (0, 0, scales_128.reshape(-1)[:1], torch.from_numpy(scales_128.reshape(-1)[:1])),
    ]
    for br, bc, sc, sfull in cases:
        ref = qv / sfull  # fp32 division, the page's "/ scale"
        y = oracle.dequantize(codes, fmt, sc, br, bc, out_dtype=oracle.F32)
        assert np.array_equal(y.view(np.uint32), ref.numpy().view(np.uint32))
        yb = oracle.dequantize(codes, fmt, sc, br, bc, out_dtype=oracle.BF16)
        refb = ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(yb, refb)


def test_round_trip_error_bound():
    """Quantize then dequantize stays within half a code spacing of x * s, divided back by s."""
    x = inputs.random_matrix(128, 1024, seed=31, dtype=torch.float32).numpy()
    q, s = oracle.quantize_blockwise(x, 1, 128, oracle.E4M3)
    y = oracle.dequantize(q, oracle.E4M3, s, 1, 128)
    srep = np.repeat(s, 128, axis=1).astype(np.float64)
    xs = x.astype(np.float64) * srep
    err = np.abs(y.astype(np.float64) * srep - xs)
    # E4M3: normal spacing is 2^(e-3); allow the fp32 rounding of the product and of the quotient
    bound = np.maximum(np.exp2(np.floor(np.log2(np.maximum(np.abs(xs), 2.0 ** -6))) - 4), 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-6) + np.abs(xs) * 2.0 ** -22)


# -- delayed scaling: closed form -----------------------------------------------

@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_delayed_scaling_closed_form(fmt):
    W, steps = 16, 32
    base = inputs.gradient_base(rows=64, cols=256)
    hist = oracle.AmaxHistory(W, fmt)
    amaxes, used = [], []
    for k in range(steps):
        g = inputs.gradient_step(base, k)
        s_used = hist.scale[0]
        q, s, a = oracle.quantize_per_tensor(inputs.bf16_bits(g), fmt, scale=float(s_used))
        qt, _, at = torch_per_tensor(g, fmt, scale=float(s_used))
        assert np.array_equal(q, qt) and a == np.float32(at)
        used.append(s)
        amaxes.append(float(a))
        hist.update(a)
    MAX = oracle.MAX[fmt]
    for k in range(steps):
        if k < W:
            assert used[k] == np.float32(1.0), k
        else:
            window = max(amaxes[k - W:k])
            assert used[k] == np.float32(MAX / max(window, float(EPS32))), k
    assert hist.state[1] == W and hist.state[0] == steps % W


def test_delayed_scaling_underflow_then_recovers():
    """Gradients of 1e-6 flush to zero in E5M2 at scale 1, and survive once the window scale applies."""
    base = inputs.gradient_base(rows=64, cols=256)
    g = inputs.gradient_step(base, 0)
    gb = inputs.bf16_bits(g)
    q1, _, _ = oracle.quantize_per_tensor(gb, oracle.E5M2, scale=1.0)
    frac_zero_s1 = np.mean((q1 & 0x7F) == 0)
    q2, s2, _ = oracle.quantize_per_tensor(gb, oracle.E5M2)
    frac_zero_cur = np.mean((q2 & 0x7F) == 0)
    assert frac_zero_s1 > 0.1 and frac_zero_cur == 0.0


# -- the fp32 product rounds before the cast -------------------------------------

def test_product_rounded_to_fp32_before_cast():
    """x * s is an fp32 op in the pages' code, so it rounds to fp32 before the cast.

    Find products whose exact value lies just off an E4M3 midpoint but whose
    fp32 rounding lands on it.  The oracle must follow the fp32 value (and agree
    with torch's x * s then cast); rounding the exact product instead would pick
    the neighbour on the exact value's side, which differs for some of them."""
    rng = np.random.default_rng(3)
    found = differs = 0
    for _ in range(400_000):
        x = np.float32(rng.uniform(1, 2))
        j = int(rng.integers(0, 7))
        target = np.float32(1.0625 + 0.125 * j)  # midpoint between E4M3 codes 0x38+j and 0x39+j
        s = np.float32(target / x)
        p32 = np.float32(np.float64(x) * np.float64(s))
        exact = np.float64(x) * np.float64(s)
        if p32 != target or exact == np.float64(target):
            continue
        found += 1
        code = int(oracle.quantize_per_tensor(np.array([x]), oracle.E4M3, scale=float(s))[0][0])
        ref = (torch.tensor([x]) * torch.tensor(s)).to(torch.float8_e4m3fn).view(torch.uint8).item()
        assert code == ref
        assert code in (0x38 + j, 0x39 + j) and code % 2 == 0  # the tie went to the even code
        exact_side = 0x39 + j if exact > np.float64(target) else 0x38 + j
        differs += int(exact_side != code)
        if found >= 60:
            break
    assert found >= 20 and differs >= 5


# -- fake quantization (quantize -> dequantize round trip) -------------------------

@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fake_quantize_vs_torch_handbook_quant(fmt, dtype):
    """The handbook's quant(): scale, clamp, cast to FP8, cast back and undo the scale, in x's dtype."""
    MAX = oracle.MAX[fmt]
    for br, bc in ((1, 128), (128, 128)):
        x = inputs.random_matrix(256, 384, seed=71, dtype=dtype, outlier_frac=0.01, factor=1e3)
        y, s = oracle.fake_quantize(as_oracle_input(x), fmt, br, bc)
        xf = x.float()
        b = xf.reshape(256 // br, br, 3, 128)
        st = torch.tensor(MAX) / b.abs().amax(dim=(1, 3), keepdim=True).clamp(min=1e-12)
        ref = ((b * st).clamp(-MAX, MAX).to(TORCH_FP8[fmt]).to(torch.float32) / st).reshape(256, 384).to(dtype)
        assert np.array_equal(s, st.reshape(256 // br, 3).numpy())
        assert np.array_equal(y, as_oracle_input(ref))
    x = inputs.random_matrix(1, 1000, seed=72, dtype=dtype).reshape(-1)
    y, _ = oracle.fake_quantize(as_oracle_input(x), fmt, 0, 0, scale=123.0)
    s = torch.tensor(123.0)
    ref = ((x.float() * s).clamp(-MAX, MAX).to(TORCH_FP8[fmt]).to(torch.float32) / s).to(dtype)
    assert np.array_equal(y, as_oracle_input(ref))


# -- delayed scaling refinements (PyTorch-FP8 page s4.3: margin, moving average) ---------

def _amax_sequence(seed, steps):
    rng = np.random.default_rng(seed)
    return np.exp(rng.uniform(np.log(1e-6), np.log(1e4), size=steps)).astype(np.float32)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_window_max_with_margin_one_is_the_plain_window(fmt):
    seq = _amax_sequence(1, 40)
    plain = oracle.AmaxHistory(16, fmt)
    ex = oracle.AmaxHistory(16, fmt, algo=oracle.WINDOW_MAX, margin=1.0)
    for a in seq:  # the extended entry point, called directly with margin exactly 1
        s1 = plain.update(a)
        lib = oracle.lib()
        assert lib.orc_amax_history_update_ex(ex.history.ctypes.data, ex.state.ctypes.data, 16, float(a), fmt,
                                              ex.scale.ctypes.data, 0, 1.0, 1.0) == 0
        assert ex.scale[0] == s1 and np.array_equal(ex.history, plain.history)
        assert np.array_equal(ex.state, plain.state)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_margin_keeps_the_window_max_below_max(fmt):
    MAX = oracle.MAX[fmt]
    seq = _amax_sequence(2, 40)
    h = oracle.AmaxHistory(8, fmt, algo=oracle.WINDOW_MAX, margin=1.1)
    plain = oracle.AmaxHistory(8, fmt)
    for k, a in enumerate(seq):
        s = h.update(a)
        s0 = plain.update(a)
        if k >= 7:
            m = float(max(seq[k - 7:k + 1]))
            # the window max lands at MAX / 1.1, never at MAX: within fp32 rounding of the two steps
            assert abs(m * float(s) * 1.1 / MAX - 1.0) < 4e-7
            # and the margin divides the plain scale (up to one rounding each)
            assert abs(float(s) * 1.1 / float(s0) - 1.0) < 4e-7
            # quantizing that max element gives a code below the format's top code
            code = oracle.encode(np.float32(np.float32(m) * s), fmt)
            assert (code & 0x7F) < oracle.top_code(fmt)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_ema_alpha_one_is_the_latest_amax_and_alpha_zero_the_first(fmt):
    seq = _amax_sequence(3, 30)
    h1 = oracle.AmaxHistory(4, fmt, algo=oracle.EMA, alpha=1.0)
    h0 = oracle.AmaxHistory(4, fmt, algo=oracle.EMA, alpha=0.0)
    for k, a in enumerate(seq):
        s1 = h1.update(a)
        s0 = h0.update(a)
        if k >= 3:
            assert s1 == oracle.scale_from_amax(a, fmt)
            assert s0 == oracle.scale_from_amax(seq[0], fmt)
        else:
            assert s1 == 1.0 and s0 == 1.0  # warm-up: the scale keeps its initial value


def test_ema_interior_alpha_hand_example():
    """One moving-average update at alpha = 5/8, worked by hand from the reading of the PyTorch-FP8
    page's smoothing (s4.2-4.3): m' = RN(RN(alpha * amax) + RN(RN(1 - alpha) * m)), every step fp32.

    u = 2^-23 (the fp32 spacing in [1, 2)).  m = 1 + 13u, amax = 4 + 8u, 1 - alpha = 3/8 exactly.
      alpha * amax = 2.5 + 5u.     In [2, 4) the spacing is 2u: 2.5 + 2.5(2u), a tie; the even
                                   significand is 2.5 + 2(2u) = 2.5 + 4u.
      (3/8) * m = 0.375 + 4.875u.  In [0.25, 0.5) the spacing is u/4: 0.375 + 19.5(u/4), a tie; the
                                   even significand is 0.375 + 20(u/4) = 0.375 + 5u.
      sum = 2.875 + 9u = 2.875 + 4.5(2u), a tie; the even significand is 2.875 + 4(2u) = 2.875 + 8u.
    So m' = 2.875 + 2^-20 (0x40380004).  Two plausible other orders give other values, so the example
    tells them apart: the exact value rounded once is 2.875 + 10u (0x40380005), and m + alpha*(amax - m)
    with each step rounded is 2.875 + 12u (0x40380006)."""
    h = oracle.AmaxHistory(2, oracle.E4M3, algo=oracle.EMA, alpha=0.625)
    m0 = np.float32(1 + 13 * 2.0 ** -23)
    a1 = np.float32(4 + 8 * 2.0 ** -23)
    assert h.update(m0) == np.float32(1.0)  # warm-up: the first update sets m and keeps the scale
    assert h.history[0].view(np.uint32) == m0.view(np.uint32)
    s = h.update(a1)
    assert int(h.history[0].view(np.uint32)) == 0x40380004
    assert float(h.history[0]) == 2.875 + 2.0 ** -20
    # the window (warm-up length 2) is full, so the scale follows from m: RN(448 / m), an IEEE fp32 division
    assert s.view(np.uint32) == (np.float32(448.0) / np.float32(2.875 + 2.0 ** -20)).view(np.uint32)


@pytest.mark.parametrize("alpha", [0.01, 0.1, 0.5, 0.9])
def test_ema_stays_inside_the_seen_range(alpha):
    seq = _amax_sequence(4, 200)
    h = oracle.AmaxHistory(1, oracle.E4M3, algo=oracle.EMA, alpha=alpha)
    for k, a in enumerate(seq):
        h.update(a)
        m = float(h.history[0])
        lo, hi = float(seq[:k + 1].min()), float(seq[:k + 1].max())
        assert lo * (1 - 1e-6) <= m <= hi * (1 + 1e-6)
    # a constant amax is (to fp32 rounding) a fixed point
    h = oracle.AmaxHistory(1, oracle.E4M3, algo=oracle.EMA, alpha=alpha)
    for _ in range(50):
        h.update(3.25)
    assert abs(float(h.history[0]) / 3.25 - 1) < 1e-6


def test_transposed_per_tensor_output_hand_example():
    """2x3 example worked by hand from the E4M3 bit layout (bias 7): 1 = 0x38,
    2 = 0x40, 448 = 0x7E, -1 = 0xB8, 0.5 = 0x30, 0 = 0x00.  amax 448 gives
    s = 1 under current scaling, the same as a delayed scale of 1."""
    x = np.array([[1.0, 2.0, 448.0], [-1.0, 0.5, 0.0]], dtype=np.float32)
    want_q = np.array([[0x38, 0x40, 0x7E], [0xB8, 0x30, 0x00]], dtype=np.uint8)
    want_qt = np.array([[0x38, 0xB8], [0x40, 0x30], [0x7E, 0x00]], dtype=np.uint8)
    for scale in (None, 1.0):
        q, qt, s, a = oracle.quantize_per_tensor_transpose(x, oracle.E4M3, scale)
        assert np.array_equal(q, want_q) and np.array_equal(qt, want_qt)
        assert s == 1.0 and a == 448.0


def test_transposed_output_is_the_per_tensor_codes():
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((37, 53)) * 10).astype(np.float32)
    for fmt in (oracle.E4M3, oracle.E5M2):
        q, qt, s, a = oracle.quantize_per_tensor_transpose(x, fmt)
        q1, s1, a1 = oracle.quantize_per_tensor(x, fmt)
        assert np.array_equal(q, q1) and s == s1 and a == a1
        assert qt.shape == (53, 37)
        assert all(qt[c, r] == q1[r, c] for r in range(37) for c in range(53))


# -- blockwise quantization of x and of x^T ---------------------------------------------------------

@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("shape", [(128, 128), (256, 384), (200, 300), (1, 5), (130, 129)])
def test_square_blocks_commute_with_transposition(fmt, shape):
    """128x128 blocks of x^T are the blocks of x transposed, so quantizing x^T gives the transposed codes
    and scales (ragged edges included)."""
    x = inputs.random_matrix(*shape, seed=7100 + shape[0], dtype=torch.float32, outlier_frac=0.01, factor=1e3)
    q, s, qt, st = oracle.quantize_blockwise_transpose(x.numpy(), 128, 128, fmt)
    assert np.array_equal(qt, q.T)
    assert np.array_equal(st.view(np.uint32), s.T.view(np.uint32))


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_1x128_blocks_of_the_transpose_are_columns(fmt):
    """For 1x128 blocks, qt's scales are MAX / max(amax, eps) over 128-row runs of x's columns (numpy fp32
    arithmetic, IEEE division), and every block of qt holds a top code (its amax element maps to MAX)."""
    R, C = 384, 256
    x = inputs.random_matrix(R, C, seed=7200, dtype=torch.float32, outlier_frac=0.01, factor=1e3).numpy()
    x[:128, 5] = 0.0  # an all-zero column block: scale MAX / eps, codes 0
    q, s, qt, st = oracle.quantize_blockwise_transpose(x, 1, 128, fmt)
    assert q.shape == (R, C) and s.shape == (R, C // 128) and qt.shape == (C, R) and st.shape == (C, R // 128)
    amax = np.abs(x).reshape(R // 128, 128, C).max(axis=1).T.astype(np.float32)  # [C, R/128]
    want = np.float32(oracle.MAX[fmt]) / np.maximum(amax, EPS32)
    assert np.array_equal(st.view(np.uint32), want.astype(np.float32).view(np.uint32))
    top = oracle.top_code(fmt)
    mag = (qt & 0x7F).reshape(C, R // 128, 128).max(axis=2)
    assert (mag[amax > EPS32] == top).all()
    assert (qt[5, :128] & 0x7F == 0).all()
    # q is the plain 1x128 quantization of x
    q2, s2 = oracle.quantize_blockwise(x, 1, 128, fmt)
    assert np.array_equal(q, q2) and np.array_equal(s.view(np.uint32), s2.view(np.uint32))
