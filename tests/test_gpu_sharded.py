"""The sharded wrappers with the library's kernels on one GPU (world size 1: no exchange); the
multi-rank exchange itself is covered on gloo ranks in test_dist_gloo.py."""
import numpy as np
import pytest
import torch

import oracle
from fine_grained_block_b200 import binding as B
from fine_grained_block_b200 import inputs, sharded
from parity_util import assert_bytes_equal, fp32_bits, host_input, to_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("algo,alpha,margin", [(0, 1.0, 1.0), (1, 0.5, 1.1)])
def test_sharded_delayed_scaler_single_rank(algo, alpha, margin):
    sc = sharded.ShardedDelayedScaler(window=3, fmt=B.E5M2, algo=algo, alpha=alpha, margin=margin)
    ref = oracle.AmaxHistory(3, oracle.E5M2, algo=algo, alpha=alpha, margin=margin)
    for k in range(7):
        x = inputs.random_matrix(257, 384, seed=9700 + k, dtype=torch.bfloat16, outlier_frac=1e-3,
                                 factor=10.0 ** (k % 3))
        s_ref = float(ref.scale[0])
        q = sc.step(to_cuda(x))
        oq, _, oa = oracle.quantize_per_tensor(host_input(x), oracle.E5M2, scale=s_ref)
        ref.update(oa)
        torch.cuda.synchronize()
        assert_bytes_equal(q, oq, f"step {k} codes")
        assert_bytes_equal(sc.scale, fp32_bits(ref.scale), f"step {k} next scale")


def test_sharded_per_tensor_and_blockwise_single_rank():
    x = inputs.random_matrix(384, 512, seed=9800, dtype=torch.bfloat16, outlier_frac=1e-3, factor=1e3)
    q, s, a = sharded.quantize_per_tensor_sharded(to_cuda(x), B.E4M3)
    oq, os_, oa = oracle.quantize_per_tensor(host_input(x), oracle.E4M3)
    assert_bytes_equal(q, oq, "per-tensor codes")
    assert_bytes_equal(s, fp32_bits([os_]), "per-tensor scale")
    qb, sb = sharded.quantize_blockwise_sharded(to_cuda(x), (128, 128), B.E4M3)
    oqb, osb = oracle.quantize_blockwise(host_input(x), 128, 128, oracle.E4M3)
    assert_bytes_equal(qb, oqb, "blockwise codes")
    assert_bytes_equal(sb, fp32_bits(osb), "blockwise scales")
