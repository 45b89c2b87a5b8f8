"""Bounded waits and the device status word (no GPU fault involved).

The one-pass per-tensor kernel's grid barrier never waits forever: a wait that
runs out sets a bit in the library's device status word and the kernel
returns.  The self-test kernel runs the same wait on a word that nothing
changes, so its wait must run out; real calls must never set the bit."""
import pytest
import torch

from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs

pytestmark = pytest.mark.gpu


def test_selftest_wait_times_out_and_is_reported():
    B.fp8_device_status(clear=True)
    B.fp8_selftest_wait_timeout(2000)  # 2 ms
    torch.cuda.synchronize()
    assert B.fp8_device_status(clear=True) & B.DEVICE_STATUS_WAIT_TIMEOUT
    assert B.fp8_device_status() == 0
    # the device is still usable
    x = torch.ones(256, 256, dtype=torch.bfloat16, device="cuda")
    q, s = B.fp8_quantize_blockwise(x, (128, 128), B.E4M3)
    torch.cuda.synchronize()
    assert bool((q == 0x7E).all()) and bool((s == 448.0).all())


def test_one_pass_barrier_never_times_out():
    B.fp8_device_status(clear=True)
    ws = B.fused_workspace()
    for n in (1, 4096, 1 << 20, 3 << 21):
        x = inputs.random_matrix(1, n, seed=n, device="cuda").reshape(-1)
        for fmt in (B.E4M3, B.E5M2):
            for _ in range(3):
                B.fp8_quantize_per_tensor_fused(x, fmt, workspace=ws)
    torch.cuda.synchronize()
    assert B.fp8_device_status() == 0
