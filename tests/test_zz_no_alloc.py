"""The entry point for callers that cannot allocate device memory.

fp8_quantize_per_tensor_fused_noalloc is fp8_quantize_per_tensor_fused
without the workspace argument.  It serves code that may not call cudaMalloc
(for instance a plugin of an inference runtime that hands out no workspace,
or a C caller whose device memory all belongs to another framework's
allocator): its workspace is a fixed array in the library's own device
memory.  This test calls it through the C ABI twice in a row on each input
and requires the same bytes as the existing workspace-taking entry point, the
same bit-exact bar as every other parity test here.  It depends on no state
left by other tests, so it passes alone in a fresh process or after them.
"""
import numpy as np
import pytest
import torch

from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs

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
