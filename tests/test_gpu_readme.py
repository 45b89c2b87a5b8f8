"""The usage example of the top-level guide runs as written, and its results agree with the oracle on a sample."""
import os
import re

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_bytes_equal, fp32_bits, host_input

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GUIDE = "README.md"  # the file that holds the one python usage example


def test_usage_example_runs():
    text = open(os.path.join(ROOT, GUIDE)).read()
    blocks = re.findall(r"```python\n(.*?)```", text, flags=re.S)
    assert len(blocks) == 1
    env = {}
    exec(compile(blocks[0], "usage-example", "exec"), env)
    torch.cuda.synchronize()
    x, qx, sx = env["x"], env["qx"], env["sx"]
    assert tuple(env["y"].shape) == (16384, 4096) and env["y"].dtype == torch.bfloat16
    oq, os_ = oracle.quantize_blockwise(host_input(x[:256].cpu()), 1, 128, oracle.E4M3)
    assert_bytes_equal(qx[:256], oq, "usage example 1x128 codes")
    assert_bytes_equal(sx[:256], fp32_bits(os_), "usage example 1x128 scales")
    assert bool(torch.isfinite(env["x_hat"].float()).all()) and float(env["scale_used"].item()) == 1.0
