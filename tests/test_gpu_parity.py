"""GPU parity: the CUDA library (called through its C ABI) against the CPU oracle.

Bar: FP8 codes bit-exact, fp32 scales and amax bit-exact, dequantized fp32 /
bf16 bit-exact (0 ulp), on the same seeded inputs.  Output buffers carry guard
bands that must come back untouched.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs
from parity_util import (Guarded, assert_bytes_equal, fp32_bits, host_input, oracle_blockwise, oracle_dequant,
                         oracle_dequant_mx, oracle_mx, oracle_per_tensor, to_cuda)

pytestmark = pytest.mark.gpu

FMTS = [oracle.E4M3, oracle.E5M2]
DT = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16}


def run_blockwise(x_cpu: torch.Tensor, block, fmt):
    R, C = x_cpu.shape
    br, bc = block
    x = to_cuda(x_cpu)
    gq = Guarded((R, C), torch.uint8)
    gs = Guarded((math.ceil(R / br), math.ceil(C / bc)), torch.float32)
    B.fp8_quantize_blockwise(x, block, fmt, q=gq.t, scales=gs.t)
    torch.cuda.synchronize()
    gq.check()
    gs.check()
    return gq.t, gs.t


def run_dequant(q: torch.Tensor, scales: torch.Tensor, block, fmt, out_dtype):
    gy = Guarded(tuple(q.shape), out_dtype)
    B.fp8_dequantize(q, scales, block, fmt, out_dtype, y=gy.t)
    torch.cuda.synchronize()
    gy.check()
    return gy.t


def check_blockwise_roundtrip(x_cpu, block, fmt, what, dequant=True):
    br, bc = block
    xh = host_input(x_cpu)
    q, s = run_blockwise(x_cpu, block, fmt)
    oq, os_ = oracle_blockwise(xh, br, bc, fmt)
    assert_bytes_equal(s, fp32_bits(os_), f"{what} scales")
    assert_bytes_equal(q, oq, f"{what} codes")
    if dequant:
        for out_dtype, oc in ((torch.float32, oracle.F32), (torch.bfloat16, oracle.BF16)):
            y = run_dequant(q, s, block, fmt, out_dtype)
            oy = oracle_dequant(oq, fmt, os_, br, bc, oc)
            assert_bytes_equal(y, oy, f"{what} dequant {out_dtype}")
    return q, s


def run_per_tensor(x_cpu: torch.Tensor, fmt, scale=None):
    x = to_cuda(x_cpu)
    gq = Guarded(tuple(x.shape), torch.uint8)
    s_out = torch.empty(1, dtype=torch.float32, device="cuda")
    a_out = torch.empty(1, dtype=torch.float32, device="cuda")
    s_in = None if scale is None else torch.tensor([scale], dtype=torch.float32, device="cuda")
    B.fp8_quantize_per_tensor(x, fmt, scale_in=s_in, q=gq.t, scale_out=s_out, amax_out=a_out)
    torch.cuda.synchronize()
    gq.check()
    return gq.t, s_out, a_out


def check_per_tensor(x_cpu, fmt, what, scale=None, dequant=True):
    xh = host_input(x_cpu)
    q, s, a = run_per_tensor(x_cpu, fmt, scale)
    oq, os_, oa = oracle_per_tensor(xh, fmt, scale)
    assert_bytes_equal(a, fp32_bits([oa]), f"{what} amax")
    assert_bytes_equal(s, fp32_bits([os_]), f"{what} scale")
    assert_bytes_equal(q, oq, f"{what} codes")
    if dequant:
        q2 = q.reshape(-1) if q.dim() != 2 else q
        oq2 = oq.reshape(q2.shape)
        for out_dtype, oc in ((torch.float32, oracle.F32), (torch.bfloat16, oracle.BF16)):
            y = run_dequant(q2, s, (0, 0), fmt, out_dtype)
            oy = oracle_dequant(oq2, fmt, np.array([os_], np.float32), 0, 0, oc)
            assert_bytes_equal(y, oy, f"{what} dequant {out_dtype}")
    return q, s, a


# -- the scalar experiment (PyTorch-FP8 page s2.2) and special values ------------

def special_values():
    v = list(inputs.SCALAR_VALUES)
    v += [-x for x in inputs.SCALAR_VALUES]
    v += [0.0, -0.0, 1e4, 6e4, 1e6, 3.0e38, -3.0e38, 464.0, 480.0, 61440.0, 2.0 ** -10, 2.0 ** -17,
          1e-40, -1e-40, 1.0625, 1.1875, 0.0009765625, 0.00146484375, 2.0 ** -9 * 0.5, 2.0 ** -16 * 0.5,
          float("inf"), float("-inf")]
    return torch.tensor(v, dtype=torch.float32)


@pytest.mark.parametrize("fmt", FMTS)
def test_scalar_cast_at_scale_one(fmt):
    x = special_values()
    q, s, a = run_per_tensor(x, fmt, scale=1.0)
    want = np.array([oracle.encode(float(v), fmt) for v in x.numpy()], dtype=np.uint8)
    assert_bytes_equal(q, want, "scale-1 cast")
    assert s.item() == 1.0


# -- config: fp32 256x1024 with outlier columns (handbook "FP8 training") ---------

@pytest.mark.parametrize("fmt", FMTS)
def test_outlier_tensors_per_tensor_and_1x128(fmt):
    for factor, a in inputs.relerr_outlier_tensors():
        check_per_tensor(a, fmt, f"per-tensor x{factor}")
        check_blockwise_roundtrip(a, (1, 128), fmt, f"1x128 x{factor}")
        check_blockwise_roundtrip(a, (128, 128), fmt, f"128x128 x{factor}")


def test_outlier_tensors_relative_error_from_gpu():
    """The handbook's printed table, reproduced from the GPU's own round trip."""
    from conftest import golden_rows
    printed = {float(f): (float(t), float(b)) for f, t, b in golden_rows("p3_relerr.txt")}
    for factor, a in inputs.relerr_outlier_tensors():
        x = to_cuda(a)
        q, s, _ = B.fp8_quantize_per_tensor(x, B.E4M3)
        yt = B.fp8_dequantize(q, s, (0, 0), B.E4M3, torch.float32)
        qb, sb = B.fp8_quantize_blockwise(x, (1, 128), B.E4M3)
        yb = B.fp8_dequantize(qb, sb, (1, 128), B.E4M3, torch.float32)
        n = x[:, 128:].double()
        t = ((yt[:, 128:].double() - n).norm() / n.norm()).item() * 100
        b = ((yb[:, 128:].double() - n).norm() / n.norm()).item() * 100
        assert (round(t, 1), round(b, 1)) == printed[factor]


# -- config: bf16 weight 4096x4096, N(0, 0.02^2), 128x128 ------------------------

@pytest.mark.parametrize("fmt", FMTS)
def test_weight_4096_128x128(fmt):
    w = inputs.weight_4096()
    check_blockwise_roundtrip(w, (128, 128), fmt, "weight 128x128")


def test_weight_4096_1x128_and_per_tensor():
    w = inputs.weight_4096()
    check_blockwise_roundtrip(w, (1, 128), oracle.E4M3, "weight 1x128")
    check_per_tensor(w, oracle.E5M2, "weight per-tensor")


# -- ragged shapes, both dtypes, both formats --------------------------------------

SHAPES = [(1, 128), (3, 256), (128, 128), (130, 384), (257, 640), (129, 1280), (64, 100), (200, 77), (5, 1),
          (1, 8), (2, 136), (300, 4096)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("block", [(1, 128), (128, 128)])
def test_ragged_blockwise(fmt, dtype, block):
    for i, (R, C) in enumerate(SHAPES):
        x = inputs.random_matrix(R, C, seed=1000 + i, dtype=dtype, outlier_frac=0.01, factor=1e3)
        check_blockwise_roundtrip(x, block, fmt, f"{block} {R}x{C} {dtype}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_ragged_per_tensor(fmt, dtype):
    for i, n in enumerate([1, 3, 7, 8, 9, 127, 4096, 4097, 65536 + 5, 1 << 20, (1 << 20) + 3]):
        x = inputs.random_matrix(1, n, seed=2000 + i, dtype=dtype, outlier_frac=0.001, factor=1e3).reshape(-1)
        check_per_tensor(x, fmt, f"per-tensor n={n} {dtype}")
        check_per_tensor(x, fmt, f"delayed n={n} {dtype}", scale=7.5)


def test_empty_inputs():
    x = torch.zeros(0, dtype=torch.bfloat16, device="cuda")
    q, s, a = B.fp8_quantize_per_tensor(x, B.E4M3)
    torch.cuda.synchronize()
    assert a.item() == 0.0
    assert fp32_bits([s.item()])[0] == fp32_bits([oracle.scale_from_amax(0.0, oracle.E4M3)])[0]
    q, s, a = B.fp8_quantize_per_tensor(x, B.E5M2, scale_in=torch.tensor([3.0], device="cuda"))
    torch.cuda.synchronize()
    assert s.item() == 3.0 and a.item() == 0.0
    q, s = B.fp8_quantize_blockwise(torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda"))
    assert q.numel() == 0 and s.numel() == 0
    y = B.fp8_dequantize(torch.zeros(0, 128, dtype=torch.uint8, device="cuda"),
                         torch.ones(1, device="cuda"), (0, 0))
    assert y.numel() == 0


# -- edge values -------------------------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
def test_edge_value_blocks(fmt):
    R, C = 256, 512
    x = inputs.random_matrix(R, C, seed=77, dtype=torch.float32)
    x[0, :128] = 0.0                       # all-zero block
    x[1, :128] = -0.0                      # all negative zero
    x[2, :128] = 1e-42                     # fp32 subnormals only
    x[3, :128] = torch.linspace(-1e-30, 1e-30, 128)
    x[4, 128:256] = 3.0e38                 # near fp32 max
    x[5, 256:384] = torch.tensor([2.0 ** k for k in range(-64, 64)])
    x[6, :] = 1.0                           # constant row: every element hits MAX
    x[128:256, 384:512] = 0.0              # an all-zero 128x128 tile
    x[7, 5] = 1e-45
    for block in ((1, 128), (128, 128)):
        check_blockwise_roundtrip(x, block, fmt, f"edge {block}")
        check_blockwise_roundtrip(x.to(torch.bfloat16), block, fmt, f"edge bf16 {block}")
    check_per_tensor(x, fmt, "edge per-tensor")
    check_per_tensor(x, fmt, "edge delayed saturating", scale=1e30)
    check_per_tensor(x, fmt, "edge delayed tiny scale", scale=1e-30)


@pytest.mark.parametrize("fmt", FMTS)
def test_dequant_every_code_with_extreme_scales(fmt):
    """All finite codes against scales across the whole fp32 range (the bit-exact division)."""
    top = oracle.top_code(fmt)
    codes = np.array([c for c in range(256) if (c & 0x7F) <= top], dtype=np.uint8)
    R = 64
    q = np.ascontiguousarray(np.tile(codes, (R, 2))[:, :256])  # every finite code in each row
    scales = np.exp2(np.linspace(-126, 127, R)).astype(np.float32).reshape(R, 1)
    scales = np.repeat(scales, 2, axis=1)
    scales[5, 0] = 1.4e-45   # subnormal scale
    scales[6, 1] = 3.4e38
    scales[7, 0] = 448.0 / 1e-12
    scales[8:16] *= -1       # negative scales: the sign of zero quotients must follow IEEE
    scales[16, 0] = 2.0 ** -100
    scales[16, 1] = 2.0 ** -101
    scales[17, 0] = 2.0 ** 100
    scales[17, 1] = 2.0 ** 101
    qg = to_cuda(torch.from_numpy(q))
    sg = to_cuda(torch.from_numpy(scales))
    for out_dtype, oc in ((torch.float32, oracle.F32), (torch.bfloat16, oracle.BF16)):
        y = run_dequant(qg, sg, (1, 128), fmt, out_dtype)
        oy = oracle.dequantize(q, fmt, scales, 1, 128, oc)
        assert_bytes_equal(y, oy, f"dequant extremes {out_dtype}")
        y0 = run_dequant(qg, sg[7:8, 0].contiguous(), (0, 0), fmt, out_dtype)
        oy0 = oracle.dequantize(q, fmt, scales[7:8, 0], 0, 0, oc)
        assert_bytes_equal(y0, oy0, f"dequant per-tensor {out_dtype}")


# -- invariants that hold at any size ----------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
def test_every_block_holds_a_max_code(fmt):
    x = to_cuda(inputs.random_matrix(1024, 2048, seed=5, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e3))
    top = oracle.top_code(fmt)
    for block in ((1, 128), (128, 128)):
        q, s = B.fp8_quantize_blockwise(x, block, fmt)
        br, bc = block
        mag = (q & 0x7F).view(q.shape[0] // br, br, q.shape[1] // bc, bc)
        assert bool((mag.amax(dim=(1, 3)) == top).all())
        assert bool((mag <= top).all())


# -- delayed scaling: history kernel --------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("window", [1, 3, 16, 33, 1024])
def test_history_update_matches_oracle(fmt, window):
    rng = np.random.default_rng(window + 10 * fmt)
    steps = window * 2 + 5
    amaxes = np.exp(rng.uniform(np.log(1e-14), np.log(1e4), size=steps)).astype(np.float32)
    amaxes[3 % steps] = 0.0
    h = torch.zeros(window, dtype=torch.float32, device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    sc = torch.ones(1, dtype=torch.float32, device="cuda")
    am = torch.empty(1, dtype=torch.float32, device="cuda")
    ref = oracle.AmaxHistory(window, fmt)
    for k in range(steps):
        am.fill_(float(amaxes[k]))
        B.fp8_amax_history_update(h, st, am, sc, fmt)
        ref.update(amaxes[k])
        torch.cuda.synchronize()
        assert_bytes_equal(sc, fp32_bits(ref.scale), f"scale step {k}")
        assert st.cpu().tolist() == ref.state.tolist()
        assert_bytes_equal(h, fp32_bits(ref.history), f"history step {k}")


def test_history_state_out_of_range_is_clamped():
    W = 8
    h = torch.arange(W, dtype=torch.float32, device="cuda")
    st = torch.tensor([-3, 999], dtype=torch.int32, device="cuda")
    sc = torch.ones(1, device="cuda")
    am = torch.tensor([100.0], device="cuda")
    B.fp8_amax_history_update(h, st, am, sc, B.E4M3)
    torch.cuda.synchronize()
    # pos -3 mod 8 = 5, count clamped to 8 (full) -> slot 5 takes 100, scale from max = 100
    ref = oracle.AmaxHistory(W, oracle.E4M3)
    ref.history[:] = np.arange(W, dtype=np.float32)
    ref.state[:] = [5, 8]
    ref.update(100.0)
    assert st.cpu().tolist() == ref.state.tolist()
    assert_bytes_equal(h, fp32_bits(ref.history), "history")
    assert_bytes_equal(sc, fp32_bits(ref.scale), "scale")


# -- boundary behaviour on the device ---------------------------------------------------

def test_misaligned_device_pointers_rejected():
    buf = torch.zeros(4096 + 64, dtype=torch.uint8, device="cuda")
    x = buf[1:1 + 2 * 1024].view(torch.uint8)
    L = B.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    q = torch.empty(1024, dtype=torch.uint8, device="cuda")
    s = torch.empty(8, dtype=torch.float32, device="cuda")
    assert L.fp8_quantize_blockwise(x.data_ptr(), 1, 8, 128, 1, 128, 0, q.data_ptr(), s.data_ptr(), stream) == -3
    assert L.fp8_dequantize(buf[3:].data_ptr(), 0, 8, 128, 1, 128, s.data_ptr(), q.data_ptr(), 1, stream) == -3


def test_runs_on_a_side_stream():
    x = to_cuda(inputs.random_matrix(512, 1024, seed=9, dtype=torch.bfloat16))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        q, s = B.fp8_quantize_blockwise(x, (1, 128), B.E4M3)
    side.synchronize()
    oq, os_ = oracle_blockwise(host_input(x.cpu()), 1, 128, oracle.E4M3)
    assert_bytes_equal(q, oq, "side-stream codes")
    assert_bytes_equal(s, fp32_bits(os_), "side-stream scales")


# -- fake quantization (fused round trip) ---------------------------------------------

def check_fake_quant(x_cpu, block, fmt, what, scale=None, in_place=False, want_scales=True):
    br, bc = block
    xh = host_input(x_cpu)
    oy, os_ = oracle.fake_quantize(xh, fmt, br, bc, scale=scale)
    x = to_cuda(x_cpu)
    s_in = None if scale is None else torch.tensor([scale], dtype=torch.float32, device="cuda")
    gs = None
    if want_scales and br != 0:
        R, C = x.shape
        gs = Guarded((math.ceil(R / br), math.ceil(C / bc)), torch.float32)
    if in_place:
        y = B.fp8_fake_quantize(x, block, fmt, scale_in=s_in, y=x, scales_out=None if gs is None else gs.t)
        assert y.data_ptr() == x.data_ptr()
    else:
        gy = Guarded(tuple(x.shape), x.dtype)
        y = B.fp8_fake_quantize(x, block, fmt, scale_in=s_in, y=gy.t, scales_out=None if gs is None else gs.t)
    torch.cuda.synchronize()
    if not in_place:
        gy.check()
    assert_bytes_equal(y, oy, f"{what} fake-quant values")
    if gs is not None:
        gs.check()
        assert_bytes_equal(gs.t, fp32_bits(os_), f"{what} fake-quant scales")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("block", [(1, 128), (128, 128)])
def test_fake_quant_blockwise(fmt, dtype, block):
    for i, (R, C) in enumerate(SHAPES):
        x = inputs.random_matrix(R, C, seed=3000 + i, dtype=dtype, outlier_frac=0.01, factor=1e3)
        check_fake_quant(x, block, fmt, f"{block} {R}x{C} {dtype}", want_scales=(i % 2 == 0))
        check_fake_quant(x, block, fmt, f"{block} {R}x{C} {dtype} in place", in_place=True)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fake_quant_per_tensor(fmt, dtype):
    for i, n in enumerate([1, 7, 8, 17, 4096, 4097, (1 << 20) + 3]):
        x = inputs.random_matrix(1, n, seed=4000 + i, dtype=dtype, outlier_frac=0.001, factor=1e3).reshape(-1)
        for scale in (1.0, 37.5, 1e-30, 3e30):
            check_fake_quant(x, (0, 0), fmt, f"per-tensor n={n} s={scale}", scale=scale)
        check_fake_quant(x, (0, 0), fmt, f"per-tensor n={n} in place", scale=2.5, in_place=True)


def test_fake_quant_edge_values():
    x = special_values().repeat(8)[:256].reshape(2, 128).contiguous()
    for fmt in FMTS:
        check_fake_quant(x, (1, 128), fmt, "special values 1x128")
        check_fake_quant(x, (0, 0), fmt, "special values per tensor", scale=1.0)


# -- amax and scale entry points (the pieces of sharded per-tensor scaling) -----------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_amax_and_scale_entry_points(dtype):
    for i, n in enumerate([0, 1, 9, 4097, (1 << 20) + 5]):
        x = inputs.random_matrix(1, max(n, 1), seed=5000 + i, dtype=dtype, outlier_frac=0.01, factor=1e3).reshape(-1)[:n]
        a = B.fp8_amax(to_cuda(x))
        oa = oracle.amax(host_input(x)) if n else np.float32(0)
        for fmt in FMTS:
            s = B.fp8_scale_from_amax(a, fmt)
            torch.cuda.synchronize()
            assert_bytes_equal(a, fp32_bits([oa]), f"amax n={n}")
            assert_bytes_equal(s, fp32_bits([oracle.scale_from_amax(oa, fmt)]), f"scale n={n}")


def test_sharded_per_tensor_single_rank_matches_unsharded():
    from fine_grained_block_b200 import sharded
    x = inputs.random_matrix(512, 1024, seed=91, dtype=torch.bfloat16, outlier_frac=0.001, factor=1e3)
    q, s, a = sharded.quantize_per_tensor_sharded(to_cuda(x), B.E5M2)
    oq, os_, oa = oracle_per_tensor(host_input(x), oracle.E5M2)
    torch.cuda.synchronize()
    assert_bytes_equal(q, oq, "sharded codes")
    assert_bytes_equal(s, fp32_bits([os_]), "sharded scale")
    assert_bytes_equal(a, fp32_bits([oa]), "sharded amax")


# -- one-pass per-tensor current scaling --------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fused_per_tensor_matches_two_pass_and_oracle(fmt, dtype):
    ws = B.fused_workspace()
    calls = 0  # one-pass calls so far
    for i, n in enumerate([1, 7, 8, 9, 1000, 4097, 1 << 16, (1 << 20) + 3, 1 << 22, 3 << 22, 1 << 24]):
        x_cpu = inputs.random_matrix(1, n, seed=6000 + i, dtype=dtype, outlier_frac=0.001, factor=1e3).reshape(-1)
        x = to_cuda(x_cpu)
        for rep in range(2):  # the workspace must come back ready for the next call
            gq = Guarded((n,), torch.uint8)
            q, s, a = B.fp8_quantize_per_tensor_fused(x, fmt, workspace=ws, q=gq.t)
            torch.cuda.synchronize()
            gq.check()
            oq, os_, oa = oracle_per_tensor(host_input(x_cpu), fmt)
            assert_bytes_equal(a, fp32_bits([oa]), f"fused amax n={n}")
            assert_bytes_equal(s, fp32_bits([os_]), f"fused scale n={n}")
            assert_bytes_equal(q, oq, f"fused codes n={n}")
            # arrivals and the running amax are back to zero; a one-pass call adds one to the call count
            # and leaves its amax beside it (larger tensors take two passes and leave the workspace alone;
            # up to 2^20 + 3 elements always fit)
            w = ws.cpu().tolist()
            assert w[0] == 0 and w[1] == 0, w
            assert w[3] in (calls, calls + 1), (w, calls)
            if n <= (1 << 20) + 3:
                assert w[3] == calls + 1, (w, calls, n)
            if w[3] == calls + 1:
                calls += 1
                assert (w[2] & 0xFFFFFFFF) == int(np.asarray(fp32_bits([oa])).view(np.uint32)[0]), \
                    f"result word amax n={n}"
    assert B.fp8_device_status() == 0


def test_fused_per_tensor_outlier_tensors():
    ws = B.fused_workspace()
    for factor, a_cpu in inputs.relerr_outlier_tensors():
        q, s, a = B.fp8_quantize_per_tensor_fused(to_cuda(a_cpu), B.E4M3, workspace=ws)
        oq, os_, oa = oracle.quantize_per_tensor(a_cpu.numpy(), oracle.E4M3)
        torch.cuda.synchronize()
        assert_bytes_equal(q, oq, f"fused x{factor}")
        assert_bytes_equal(s, fp32_bits([os_]), f"fused scale x{factor}")


# -- delayed scaling refinements: margin and moving average ------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("algo,alpha,margin,window", [(0, 1.0, 1.1, 16), (0, 1.0, 1.0, 5), (0, 1.0, 2.5, 33),
                                                      (1, 0.1, 1.0, 1), (1, 0.25, 1.1, 8), (1, 1.0, 1.0, 3),
                                                      (1, 0.0, 1.3, 2)])
def test_history_update_ex_matches_oracle(fmt, algo, alpha, margin, window):
    rng = np.random.default_rng(17 + window)
    amaxes = np.exp(rng.uniform(np.log(1e-14), np.log(1e4), size=3 * window + 10)).astype(np.float32)
    amaxes[2] = 0.0
    h = torch.zeros(window, dtype=torch.float32, device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    sc = torch.ones(1, dtype=torch.float32, device="cuda")
    am = torch.empty(1, dtype=torch.float32, device="cuda")
    ref = oracle.AmaxHistory(window, fmt, algo=algo, alpha=alpha, margin=margin)
    for k, a in enumerate(amaxes):
        am.fill_(float(a))
        B.fp8_amax_history_update_ex(h, st, am, sc, fmt, algo, alpha, margin)
        lib = oracle.lib()
        assert lib.orc_amax_history_update_ex(ref.history.ctypes.data, ref.state.ctypes.data, window, float(a), fmt,
                                              ref.scale.ctypes.data, algo, float(alpha), float(margin)) == 0
        torch.cuda.synchronize()
        assert_bytes_equal(sc, fp32_bits(ref.scale), f"scale step {k}")
        assert st.cpu().tolist()[1] == int(ref.state[1])
        if algo == 0:
            assert st.cpu().tolist()[0] == int(ref.state[0])
            assert_bytes_equal(h, fp32_bits(ref.history), f"history step {k}")
        else:
            assert_bytes_equal(h[:1], fp32_bits(ref.history[:1]), f"ema step {k}")


# -- MX: 1x32 blocks, power-of-two scales as E8M0 bytes ----------------------------------

def run_mx(x_cpu: torch.Tensor, fmt, rule):
    R, C = x_cpu.shape
    x = to_cuda(x_cpu)
    gq = Guarded((R, C), torch.uint8)
    ge = Guarded((R, math.ceil(C / 32)), torch.uint8)
    B.fp8_quantize_mx(x, fmt, rule, q=gq.t, e8m0=ge.t)
    torch.cuda.synchronize()
    gq.check()
    ge.check()
    return gq.t, ge.t


def check_mx(x_cpu, fmt, rule, what, nan_positions=None):
    xh = host_input(x_cpu)
    q, e = run_mx(x_cpu, fmt, rule)
    oq, oe = oracle_mx(xh, fmt, rule)
    assert_bytes_equal(e, oe, f"{what} e8m0")
    if nan_positions is not None:
        # a NaN element has several valid NaN codes: require a NaN code there,
        # exact bytes everywhere else
        qc = q.cpu().numpy()
        nan_codes = {oracle.E4M3: (0x7F,), oracle.E5M2: (0x7D, 0x7E, 0x7F)}[fmt]
        assert all((int(qc[i]) & 0x7F) in nan_codes for i in nan_positions), what
        for i in nan_positions:
            qc[i] = oq[i]
        q = torch.from_numpy(qc)
    assert_bytes_equal(q, oq, f"{what} codes")
    for out_dtype, oc in ((torch.float32, oracle.F32), (torch.bfloat16, oracle.BF16)):
        gy = Guarded(tuple(oq.shape), out_dtype)
        B.fp8_dequantize_mx(to_cuda(torch.from_numpy(oq)), e, fmt, out_dtype, y=gy.t)
        torch.cuda.synchronize()
        gy.check()
        assert_bytes_equal(gy.t, oracle_dequant_mx(oq, fmt, oe, oc), f"{what} dequant {out_dtype}")


MX_SHAPES = SHAPES + [(3, 32), (5, 33), (7, 95), (9, 64), (33, 160), (2, 31)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rule", [B.MX_FIT, B.MX_OCP])
def test_mx_ragged(fmt, dtype, rule):
    for i, (R, C) in enumerate(MX_SHAPES):
        x = inputs.random_matrix(R, C, seed=3000 + i, dtype=dtype, outlier_frac=0.01, factor=1e3)
        check_mx(x, fmt, rule, f"mx rule {rule} {R}x{C} {dtype}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rule", [B.MX_FIT, B.MX_OCP])
def test_mx_edge_values(fmt, rule):
    R, C = 16, 256
    x = inputs.random_matrix(R, C, seed=78, dtype=torch.float32)
    x[0, :32] = 0.0                          # all-zero block
    x[1, :32] = -0.0
    x[2, :32] = 1e-42                        # fp32 subnormals only
    x[3, :64] = torch.linspace(-1e-30, 1e-30, 64)
    x[4, 32:64] = 3.0e38                     # near fp32 max: k = -120 or so
    x[4, 64:96] = torch.finfo(torch.float32).max  # fp32 max: its dequant overflows to Inf
    x[5, :128] = torch.tensor([2.0 ** k for k in range(-64, 64)])
    x[6, :] = 1.0                            # every element hits the top of its binade
    x[7, :32] = 1.75 * 2.0 ** -8             # amax * 2^k exactly MAX under the fit rule
    x[7, 32:64] = 1.7500001
    x[8, 3] = float("inf")                   # blocks holding Inf: the NaN byte
    x[9, 40] = float("-inf")
    x[10, :32] = torch.linspace(-3.0, 3.0, 32) * 2.0 ** 100
    for dtype in (torch.float32, torch.bfloat16):
        check_mx(x.to(dtype), fmt, rule, f"mx edge {dtype}")
    x[11, 7] = float("nan")                  # NaN does not count toward amax
    check_mx(x, fmt, rule, "mx edge NaN", nan_positions=[(11, 7)])


@pytest.mark.parametrize("fmt", FMTS)
def test_mx_dequant_every_byte(fmt):
    """Every finite code against every E8M0 byte, 0 (the subnormal multiplier 2^-127) to 0xFF (NaN)."""
    top = oracle.top_code(fmt)
    codes = np.array([c for c in range(256) if (c & 0x7F) <= top], dtype=np.uint8)
    q = np.ascontiguousarray(np.tile(codes, (256, 1))[:, :224])   # 224 codes = 7 blocks per row
    e = np.tile(np.arange(256, dtype=np.uint8).reshape(256, 1), (1, 7))
    e[:, 3] = e[::-1, 0]
    qg, eg = to_cuda(torch.from_numpy(q)), to_cuda(torch.from_numpy(np.ascontiguousarray(e)))
    for out_dtype, oc in ((torch.float32, oracle.F32), (torch.bfloat16, oracle.BF16)):
        y = B.fp8_dequantize_mx(qg, eg, fmt, out_dtype)
        torch.cuda.synchronize()
        assert_bytes_equal(y, oracle.dequantize_mx(q, fmt, e, oc), f"mx dequant bytes {out_dtype}")
        y2 = B.fp8_dequantize_mx(qg[:, :200].contiguous(), eg, fmt, out_dtype)  # ragged: 200 = 6 blocks + 8
        torch.cuda.synchronize()
        assert_bytes_equal(y2, oracle.dequantize_mx(np.ascontiguousarray(q[:, :200]), fmt, e, oc),
                           f"mx dequant ragged {out_dtype}")


def test_mx_empty():
    q, e = B.fp8_quantize_mx(torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda"))
    assert q.numel() == 0 and e.numel() == 0
    y = B.fp8_dequantize_mx(torch.zeros(4, 0, dtype=torch.uint8, device="cuda"),
                            torch.zeros(4, 0, dtype=torch.uint8, device="cuda"))
    assert y.numel() == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mx_16_byte_aligned_buffers(fmt, dtype):
    """Input and output 16- but not 32-byte aligned: the 16-byte lane kernels."""
    R, C = 67, 320
    x_cpu = inputs.random_matrix(R, C, seed=3100, dtype=dtype, outlier_frac=0.01, factor=1e3)
    off = 16 // x_cpu.element_size()
    buf = torch.empty(R * C + off, dtype=dtype, device="cuda")
    x = buf[off:].view(R, C)
    x.copy_(x_cpu.to("cuda"))
    assert x.data_ptr() % 32 == 16
    q, e = B.fp8_quantize_mx(x, fmt, B.MX_FIT)
    torch.cuda.synchronize()
    oq, oe = oracle_mx(host_input(x_cpu), fmt, B.MX_FIT)
    assert_bytes_equal(e, oe, "e8m0")
    assert_bytes_equal(q, oq, "codes")
    for out_dtype, oc in ((torch.float32, oracle.F32), (torch.bfloat16, oracle.BF16)):
        esz = torch.empty(0, dtype=out_dtype).element_size()
        ybuf = torch.empty(R * C + 16 // esz, dtype=out_dtype, device="cuda")
        y = ybuf[16 // esz:].view(R, C)
        assert y.data_ptr() % 32 == 16
        B.fp8_dequantize_mx(q, e, fmt, out_dtype, y=y)
        torch.cuda.synchronize()
        assert_bytes_equal(y, oracle_dequant_mx(oq, fmt, oe, oc), f"dequant {out_dtype}")


# -- per-tensor with a transposed copy ---------------------------------------------------

def check_transpose(x_cpu, fmt, what, scale=None, with_q=True):
    R, C = x_cpu.shape
    x = to_cuda(x_cpu)
    gq = Guarded((R, C), torch.uint8) if with_q else None
    gt = Guarded((C, R), torch.uint8)
    s_in = None if scale is None else torch.tensor([scale], dtype=torch.float32, device="cuda")
    _, _, s, a = B.fp8_quantize_per_tensor_transpose(x, fmt, s_in, with_q=with_q, q=None if gq is None else gq.t,
                                                     qt=gt.t)
    torch.cuda.synchronize()
    gt.check()
    oq, oqt, os_, oa = oracle.quantize_per_tensor_transpose(host_input(x_cpu), fmt, scale)
    assert_bytes_equal(s, fp32_bits([os_]), f"{what} scale")
    assert_bytes_equal(a, fp32_bits([oa]), f"{what} amax")
    assert_bytes_equal(gt.t, oqt, f"{what} qt")
    if gq is not None:
        gq.check()
        assert_bytes_equal(gq.t, oq, f"{what} q")


TRANSPOSE_SHAPES = [(128, 128), (256, 384), (1024, 4096), (130, 384), (257, 640), (64, 100), (200, 77), (5, 1),
                    (1, 8), (16, 4096), (4096, 16), (48, 96)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_per_tensor_transpose(fmt, dtype):
    for i, (R, C) in enumerate(TRANSPOSE_SHAPES):
        x = inputs.random_matrix(R, C, seed=4000 + i, dtype=dtype, outlier_frac=0.01, factor=1e3)
        check_transpose(x, fmt, f"transpose {R}x{C} {dtype}")
        check_transpose(x, fmt, f"transpose delayed {R}x{C} {dtype}", scale=3.25)
    x = inputs.random_matrix(512, 256, seed=4100, dtype=dtype)
    check_transpose(x, fmt, "transpose qt only", with_q=False)
    check_transpose(x, fmt, "transpose qt only delayed", scale=0.5, with_q=False)


def test_per_tensor_transpose_16_byte_aligned_input():
    R, C = 256, 512
    x_cpu = inputs.random_matrix(R, C, seed=4200, dtype=torch.bfloat16, outlier_frac=0.01, factor=1e3)
    buf = torch.empty(R * C + 8, dtype=torch.bfloat16, device="cuda")
    x = buf[8:].view(R, C)
    x.copy_(x_cpu.to("cuda"))
    assert x.data_ptr() % 32 == 16
    q, qt, s, a = B.fp8_quantize_per_tensor_transpose(x, B.E4M3)
    torch.cuda.synchronize()
    oq, oqt, os_, oa = oracle.quantize_per_tensor_transpose(host_input(x_cpu), B.E4M3)
    assert_bytes_equal(qt, oqt, "qt")
    assert_bytes_equal(q, oq, "q")


# -- blockwise quantization of x and of x^T in one pass ------------------------------------------

BT_SHAPES = [(128, 128), (256, 384), (384, 128), (128, 1024), (1024, 4096)]


def check_blockwise_transpose(x_cpu, block, fmt, what, x=None):
    R, C = x_cpu.shape
    br, bc = block
    x = to_cuda(x_cpu) if x is None else x
    gq, gt = Guarded((R, C), torch.uint8), Guarded((C, R), torch.uint8)
    gs, gst = Guarded((R // br, C // bc), torch.float32), Guarded((C // br, R // bc), torch.float32)
    B.fp8_quantize_blockwise_transpose(x, block, fmt, q=gq.t, scales=gs.t, qt=gt.t, scales_t=gst.t)
    torch.cuda.synchronize()
    for g in (gq, gt, gs, gst):
        g.check()
    oq, os_, oqt, ost = oracle.quantize_blockwise_transpose(host_input(x_cpu), br, bc, fmt)
    assert_bytes_equal(gs.t, fp32_bits(os_), f"{what} scales")
    assert_bytes_equal(gq.t, oq, f"{what} q")
    assert_bytes_equal(gst.t, fp32_bits(ost), f"{what} scales_t")
    assert_bytes_equal(gt.t, oqt, f"{what} qt")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("block", [(1, 128), (128, 128)])
def test_blockwise_transpose(fmt, dtype, block):
    for i, (R, C) in enumerate(BT_SHAPES):
        x = inputs.random_matrix(R, C, seed=4300 + i, dtype=dtype, outlier_frac=0.01, factor=1e3)
        x[:, 3] = 0  # an all-zero column: its 1x128 column blocks get MAX / eps
        check_blockwise_transpose(x, block, fmt, f"{block} {R}x{C} {dtype}")


@pytest.mark.parametrize("fmt", FMTS)
def test_blockwise_transpose_many_tiles_per_cta(fmt):
    """bf16 1x128 with several times more tiles than resident CTAs, so each CTA of the persistent kernel
    reuses its shared-memory stages (both mbarrier parities) many times."""
    x = inputs.random_matrix(4096, 8192, seed=4350 + fmt, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e3)
    x[:, 130] = 0
    check_blockwise_transpose(x, (1, 128), fmt, "1x128 4096x8192 bf16")


@pytest.mark.parametrize("fmt", FMTS)
def test_blockwise_transpose_edge_values(fmt):
    """Special rows and columns through x and x^T at once: zero and negative-zero runs, fp32 subnormals,
    values near the type's maximum, a binade ladder, constant runs, an all-zero 128x128 tile, and columns
    of each kind, so that row blocks and column blocks both meet them (finite inputs, the contract)."""
    R, C = 256, 512
    x = inputs.random_matrix(R, C, seed=78, dtype=torch.float32)
    x[0, :128] = 0.0
    x[1, :128] = -0.0
    x[2, :128] = 1e-42
    x[3, :128] = torch.linspace(-1e-30, 1e-30, 128)
    x[4, 128:256] = 3.0e38
    x[5, 256:384] = torch.tensor([2.0 ** k for k in range(-64, 64)])
    x[6, :] = 1.0
    x[128:256, 384:512] = 0.0
    x[:128, 7] = -0.0                       # a column block of negative zeros
    x[:128, 8] = 1e-42                      # a column block of subnormals
    x[:, 9] = torch.tensor([2.0 ** (k % 128 - 64) for k in range(R)])  # binade ladders down a column
    x[128:, 10] = 2.5e38
    for dtype in (torch.float32, torch.bfloat16):
        xd = x.to(dtype)
        for block in ((1, 128), (128, 128)):
            check_blockwise_transpose(xd, block, fmt, f"edge {block} {dtype}")


def test_blockwise_transpose_16_byte_aligned_input():
    R, C = 256, 512
    x_cpu = inputs.random_matrix(R, C, seed=4400, dtype=torch.bfloat16, outlier_frac=0.01, factor=1e3)
    buf = torch.empty(R * C + 8, dtype=torch.bfloat16, device="cuda")
    x = buf[8:].view(R, C)
    x.copy_(x_cpu.to("cuda"))
    assert x.data_ptr() % 32 == 16
    for block in ((1, 128), (128, 128)):
        check_blockwise_transpose(x_cpu, block, B.E4M3, f"16-byte aligned {block}", x=x)


# -- one delayed-scaling step in one launch ---------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("algo,alpha,margin,window", [(0, 1.0, 1.0, 4), (0, 1.0, 1.1, 3), (1, 0.25, 1.0, 2)])
def test_delayed_step_matches_oracle_and_two_calls(fmt, dtype, algo, alpha, margin, window):
    """fp8_quantize_delayed_step == delayed cast + history update: codes, scale used, amax, next scale,
    history and state, step after step, against the oracle and against the two separate calls."""
    sizes = [0, 7, 4097, (1 << 20) + 3, 1 << 22]
    fused = B.DelayedScaler(window=window, fmt=fmt, algo=algo, alpha=alpha, margin=margin, fused=True)
    split = B.DelayedScaler(window=window, fmt=fmt, algo=algo, alpha=alpha, margin=margin, fused=False)
    ref = oracle.AmaxHistory(window, fmt, algo=algo, alpha=alpha, margin=margin)
    for k in range(2 * window + 4):
        n = sizes[k % len(sizes)]
        x_cpu = inputs.random_matrix(1, max(n, 1), seed=6000 + k, dtype=dtype, outlier_frac=1e-3,
                                     factor=10.0 ** (k % 5)).reshape(-1)[:n]
        x = to_cuda(x_cpu)
        s_ref = float(ref.scale[0])
        q1, s1 = fused.step(x)
        q2, s2 = split.step(x)
        oq, _, oa = oracle.quantize_per_tensor(host_input(x_cpu), fmt, scale=s_ref)
        ref.update(oa)
        torch.cuda.synchronize()
        assert_bytes_equal(q1, oq, f"step {k} codes")
        assert_bytes_equal(q1, q2.cpu().numpy(), f"step {k} codes vs two calls")
        assert_bytes_equal(s1, fp32_bits([s_ref]), f"step {k} scale used")
        assert_bytes_equal(fused.amax, fp32_bits([oa]), f"step {k} amax")
        assert_bytes_equal(fused.scale, fp32_bits(ref.scale), f"step {k} next scale")
        assert_bytes_equal(fused.scale, split.scale.cpu().numpy().view(np.uint32), f"step {k} next scale vs two calls")
        assert fused.state.cpu().tolist() == split.state.cpu().tolist()
        assert_bytes_equal(fused.history, split.history.cpu().numpy().view(np.uint32), f"step {k} history")
    assert int(fused.workspace.abs().sum().item()) == 0  # left zero for the next call


# -- grouped blockwise quantization ---------------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("block", [(1, 128), (128, 128)])
def test_grouped_matches_oracle(fmt, dtype, block):
    shapes = [(128, 128), (300, 256), (1, 128), (0, 128), (129, 384), (1024, 1024), (7, 128), (256, 0)]
    shapes += [(64 + (i % 5), 128 * (1 + i % 3)) for i in range(140)]  # more than one launch's worth
    xs_cpu = [inputs.random_matrix(max(R, 1), max(C, 1), seed=7000 + i, dtype=dtype, outlier_frac=0.01,
                                   factor=1e3)[:R, :C].contiguous() for i, (R, C) in enumerate(shapes)]
    xs = [to_cuda(x) for x in xs_cpu]
    # one tensor 16- but not 32-byte aligned: the whole group takes 16-byte lanes
    esz = xs_cpu[1].element_size()
    buf = torch.empty(xs_cpu[1].numel() + 16 // esz, dtype=dtype, device="cuda")
    xs[1] = buf[16 // esz:].view(xs_cpu[1].shape)
    xs[1].copy_(xs_cpu[1].to("cuda"))
    for lanes in ("16-byte", "32-byte"):
        group = xs if lanes == "16-byte" else [xs[0], to_cuda(xs_cpu[1])] + xs[2:]
        qs, ss = B.fp8_quantize_blockwise_grouped(group, block, fmt)
        torch.cuda.synchronize()
        for i, (x_cpu, q, s) in enumerate(zip(xs_cpu, qs, ss)):
            if x_cpu.numel() == 0:
                continue
            oq, os_ = oracle.quantize_blockwise(host_input(x_cpu), *block, fmt)
            assert_bytes_equal(s, fp32_bits(os_), f"{lanes} tensor {i} scales")
            assert_bytes_equal(q, oq, f"{lanes} tensor {i} codes")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_grouped_current_scaling_matches_oracle(fmt, dtype):
    """fp8_quantize_per_tensor_grouped over 140 tensors (more than one launch of 128; empty, one-element,
    ragged and multi-chunk ones; outlier magnitudes that differ per tensor) == the oracle's current scaling
    of each tensor on its own, codes, scale and amax bit for bit, twice in a row (the amax outputs are
    cleared by the call, whatever they held), with 16- and 32-byte lanes."""
    sizes = [0, 1, 7, 4097, 1 << 16, (1 << 20) + 3] + [1000 * (i + 1) + (i % 9) for i in range(134)]
    xs_cpu = [inputs.random_matrix(1, max(n, 1), seed=9500 + i, dtype=dtype, outlier_frac=1e-3,
                                   factor=10.0 ** (i % 5)).reshape(-1)[:n] for i, n in enumerate(sizes)]
    refs = [oracle.quantize_per_tensor(host_input(x), fmt) for x in xs_cpu]
    xs = [to_cuda(x) for x in xs_cpu]
    # one tensor 16- but not 32-byte aligned: the whole group takes 16-byte lanes
    esz = xs_cpu[4].element_size()
    buf = torch.empty(xs_cpu[4].numel() + 16 // esz, dtype=dtype, device="cuda")
    x16 = buf[16 // esz:]
    x16.copy_(xs_cpu[4].to("cuda"))
    for lanes, group in (("32-byte", xs), ("16-byte", xs[:4] + [x16] + xs[5:])):
        amaxes = [torch.full((1,), 1e30, dtype=torch.float32, device="cuda") for _ in xs]  # stale values
        for call in range(2):
            qs, ss, aa = B.fp8_quantize_per_tensor_grouped(group, fmt, amaxes=amaxes)
            torch.cuda.synchronize()
            for i, (oq, os_, oa) in enumerate(refs):
                what = f"{lanes} call {call} tensor {i}"
                assert_bytes_equal(aa[i], fp32_bits([oa]), what + " amax")
                assert_bytes_equal(ss[i], fp32_bits([os_]), what + " scale")
                assert_bytes_equal(qs[i], oq, what + " codes")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("algo,alpha,margin,window", [(0, 1.0, 1.0, 3), (1, 0.5, 1.1, 2)])
def test_grouped_delayed_steps_match_single_calls_and_oracle(fmt, dtype, algo, alpha, margin, window):
    """fp8_quantize_delayed_step_grouped over 140 tensors (more than one launch of 128, with empty and ragged
    ones) == each tensor's own DelayedScaler, and the oracle, step after step."""
    sizes = [0, 1, 7, 4097, 1 << 16, (1 << 18) + 3] + [1000 * (i + 1) + (i % 9) for i in range(134)]
    kw = dict(window=window, fmt=fmt, algo=algo, alpha=alpha, margin=margin)
    grouped = [B.DelayedScaler(**kw) for _ in sizes]
    single = [B.DelayedScaler(**kw) for _ in sizes]
    refs = [oracle.AmaxHistory(window, fmt, algo=algo, alpha=alpha, margin=margin) for _ in sizes]
    ws = torch.zeros(len(sizes) * B.FUSED_WORKSPACE_BYTES // 4, dtype=torch.int32, device="cuda")
    for k in range(window + 2):
        xs_cpu = [inputs.random_matrix(1, max(n, 1), seed=9000 + 131 * k + i, dtype=dtype, outlier_frac=1e-3,
                                       factor=10.0 ** (i % 4)).reshape(-1)[:n] for i, n in enumerate(sizes)]
        xs = [to_cuda(x) for x in xs_cpu]
        s_refs = [float(r.scale[0]) for r in refs]
        qg = B.fp8_quantize_delayed_step_grouped(xs, grouped, workspace=ws)
        qs = [sc.step(x)[0] for sc, x in zip(single, xs)]
        torch.cuda.synchronize()
        for i, (x_cpu, r) in enumerate(zip(xs_cpu, refs)):
            oq, _, oa = oracle.quantize_per_tensor(host_input(x_cpu), fmt, scale=s_refs[i])
            r.update(oa)
            assert_bytes_equal(qg[i], oq, f"step {k} tensor {i} codes")
            assert_bytes_equal(qg[i], qs[i].cpu().numpy(), f"step {k} tensor {i} codes vs single")
            assert_bytes_equal(grouped[i].scale_used, fp32_bits([s_refs[i]]), f"step {k} tensor {i} scale used")
            assert_bytes_equal(grouped[i].amax, fp32_bits([oa]), f"step {k} tensor {i} amax")
            assert_bytes_equal(grouped[i].scale, fp32_bits(r.scale), f"step {k} tensor {i} next scale")
            assert grouped[i].state.cpu().tolist() == single[i].state.cpu().tolist()
    assert int(ws.abs().sum().item()) == 0
