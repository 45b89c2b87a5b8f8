"""Bounded waits and the device status word (no GPU fault involved).

The TMA pipelines never wait forever: a wait that runs out sets a bit in the
library's device status word and the kernel returns.  The self-test kernel
waits on a barrier that nothing completes, so its wait must run out; the real
pipelines must never set the bit."""
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


def test_tile_pipeline_never_times_out():
    B.fp8_device_status(clear=True)
    for rows, cols in ((128, 128), (4096, 4096), (130, 384), (1, 128), (16384, 7168)):
        x = inputs.random_matrix(rows, cols, seed=rows + cols, device="cuda")
        for fmt in (B.E4M3, B.E5M2):
            B.fp8_quantize_blockwise(x, (128, 128), fmt)
    torch.cuda.synchronize()
    assert B.fp8_device_status() == 0
