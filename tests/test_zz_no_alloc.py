"""The entry point for callers that cannot allocate device memory.

fp8_quantize_per_tensor_fused_noalloc is fp8_quantize_per_tensor_fused
without the workspace argument.  It serves code that may not call cudaMalloc
(for instance a plugin of an inference runtime that hands out no workspace,
or a C caller whose device memory all belongs to another framework's
allocator): its workspace is a fixed array in the library's own device
memory.  This test calls it through the C ABI twice in a row on each input
and requires the same bytes as the existing workspace-taking entry point and
as the oracle, the same bit-exact bar as every other parity test here.  It
also finds the largest size the entry point accepts, for each element type
and input alignment, and checks it against the limit the header states.  It
depends on no state left by other tests, so it passes alone in a fresh
process or after them.
"""
import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs
from parity_util import host_input

pytestmark = pytest.mark.gpu

DT = {torch.float32: B.F32, torch.bfloat16: B.BF16}
FP8_ERR_TOO_LARGE = -8


def _bits(t):
    t = t.detach().cpu()
    return t.view(torch.int32).numpy() if t.dtype == torch.float32 else t.numpy()


@pytest.mark.parametrize("fmt", [B.E4M3, B.E5M2])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_no_alloc_matches_workspace_entry_point_two_calls_in_a_row(fmt, dtype):
    L = B.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    for i, n in enumerate([1, 9, 4097, (1 << 20) + 3, 1 << 22]):
        x = inputs.random_matrix(1, n, seed=7000 + i, dtype=dtype, outlier_frac=1e-3, factor=1e3,
                                 device="cuda").reshape(-1)
        # the existing entry point, with a workspace of its own
        q_ref, s_ref, a_ref = B.fp8_quantize_per_tensor_fused(x, fmt, workspace=B.fused_workspace())
        torch.cuda.synchronize()
        # and the oracle, directly: current scaling over the whole tensor
        oq, os_, oa = oracle.quantize_per_tensor(host_input(x.cpu()), fmt)
        assert np.array_equal(_bits(q_ref), oq), n
        assert np.array_equal(_bits(s_ref), np.array([os_], np.float32).view(np.int32)), n
        assert np.array_equal(_bits(a_ref), np.array([oa], np.float32).view(np.int32)), n
        for call in range(2):
            q = torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda")
            s = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
            a = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
            rc = L.fp8_quantize_per_tensor_fused_noalloc(x.data_ptr(), DT[dtype], n, fmt, q.data_ptr(),
                                                         s.data_ptr(), a.data_ptr(), stream)
            assert rc == 0, B.fp8_status_string(rc)
            torch.cuda.synchronize()
            assert np.array_equal(_bits(q), _bits(q_ref)), (n, call)
            assert np.array_equal(_bits(s), _bits(s_ref)), (n, call)
            assert np.array_equal(_bits(a), _bits(a_ref)), (n, call)


def test_no_alloc_rejects_tensors_beyond_its_limit():
    L = B.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    n = 1 << 27  # 256 MiB of bf16: far beyond what one pass holds on chip
    x = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    a = torch.empty(1, dtype=torch.float32, device="cuda")
    rc = L.fp8_quantize_per_tensor_fused_noalloc(x.data_ptr(), B.BF16, n, B.E4M3, q.data_ptr(), s.data_ptr(),
                                                 a.data_ptr(), stream)
    assert rc == FP8_ERR_TOO_LARGE
    assert "too large" in B.fp8_status_string(rc)


# The limit the header states: n <= C * 1024 * E + (E - 1), E elements per lane vector (16 or 8 for bf16,
# 8 or 4 for fp32, at a 32- or only 16-byte-aligned x), C co-resident CTAs; on a 148-SM B200, C = 592 with
# 32-byte lanes and 740 with 16-byte lanes.
B200_LIMIT = {(torch.bfloat16, 32): 9_699_343, (torch.bfloat16, 16): 6_062_087,
              (torch.float32, 32): 4_849_671, (torch.float32, 16): 3_031_043}


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_no_alloc_limit_by_alignment(dtype):
    """The largest accepted n, found by bisection on the return code (a refused call enqueues nothing), is one
    full lane vector per thread of every co-resident CTA plus a tail; one more element is refused.  An x that
    is only 16-byte aligned takes 16-byte lanes, so a size just above that limit is refused there and
    accepted at a 32-byte-aligned address."""
    L = B.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    cap = 1 << 24
    esz = torch.empty(0, dtype=dtype).element_size()
    buf = torch.zeros(cap * esz + 64, dtype=torch.uint8, device="cuda")
    q = torch.empty(cap + 64, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    a = torch.empty(1, dtype=torch.float32, device="cuda")
    base = buf.data_ptr()
    assert base % 256 == 0

    def call(x_ptr, n):
        return L.fp8_quantize_per_tensor_fused_noalloc(x_ptr, DT[dtype], n, B.E4M3, q.data_ptr(), s.data_ptr(),
                                                       a.data_ptr(), stream)

    limits = {}
    for lane, ptr in ((32, base), (16, base + 16)):
        lo, hi = 1, cap  # call(lo) accepted, call(hi) refused
        assert call(ptr, lo) == 0 and call(ptr, hi) == FP8_ERR_TOO_LARGE
        while hi - lo > 1:
            mid = (lo + hi) // 2
            rc = call(ptr, mid)
            assert rc in (0, FP8_ERR_TOO_LARGE), B.fp8_status_string(rc)
            lo, hi = (mid, hi) if rc == 0 else (lo, mid)
        torch.cuda.synchronize()
        limits[lane] = lo
        elems = lane // esz
        # a whole number of CTAs of 1024 lane vectors, plus a tail of elems - 1
        assert (lo - (elems - 1)) % (1024 * elems) == 0, lo
    assert limits[32] > limits[16]
    # just above the 16-byte-lane limit: refused at base + 16, accepted at the 32-byte-aligned base
    n = limits[16] + 1
    assert call(base + 16, n) == FP8_ERR_TOO_LARGE
    assert call(base, n) == 0
    torch.cuda.synchronize()
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert limits[32] == B200_LIMIT[(dtype, 32)] and limits[16] == B200_LIMIT[(dtype, 16)], limits
