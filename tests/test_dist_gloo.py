"""The multi-rank paths on CPU with the gloo backend (world size 2).

- per-tensor current scaling of a row-sharded tensor: the shards' amax is
  all-reduced (MAX), so every rank casts with the scale of the whole tensor;
  the gathered codes equal the unsharded result.  The per-shard compute is the
  CPU oracle here (the library's kernels need a GPU); what is under test is
  the exchange.
- blockwise quantization of row shards needs no exchange and reproduces the
  unsharded result when shard edges fall on block edges.
- the benchmark's max-over-ranks reduction of timings.
"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from fine_grained_block_b200 import inputs, sharded

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_ops():
    def amax(x):
        return torch.tensor([float(oracle.amax(inputs.bf16_bits(x)))], dtype=torch.float32)

    def scale(a, fmt):
        return torch.tensor([float(oracle.scale_from_amax(float(a.item()), fmt))], dtype=torch.float32)

    def cast(x, fmt, s):
        q, _, _ = oracle.quantize_per_tensor(inputs.bf16_bits(x), fmt, scale=float(s.item()))
        return torch.from_numpy(q)

    def blockwise(x, block, fmt):
        q, s = oracle.quantize_blockwise(inputs.bf16_bits(x), block[0], block[1], fmt)
        return torch.from_numpy(q), torch.from_numpy(s)

    return sharded.ShardOps(amax=amax, scale_from_amax=scale, cast=cast, blockwise=blockwise)


class OracleDelayedState:
    """A rank's delayed-scaling state kept by the oracle's AmaxHistory."""

    def __init__(self, window, fmt, algo, alpha, margin):
        self.fmt = fmt
        self.h = oracle.AmaxHistory(window, fmt, algo=algo, alpha=alpha, margin=margin)

    @property
    def scale(self):
        return torch.from_numpy(self.h.scale.copy())


def oracle_delayed_ops():
    def cast_amax(x, st):
        q, _, a = oracle.quantize_per_tensor(inputs.bf16_bits(x), st.fmt, scale=float(st.h.scale[0]))
        return torch.from_numpy(q), torch.tensor([float(a)], dtype=torch.float32)

    return sharded.DelayedOps(new_state=lambda w, f, al, a, m, d: OracleDelayedState(w, f, al, a, m),
                              cast_amax=cast_amax, update=lambda st, amax: st.h.update(float(amax.item())))


DELAYED_STEPS, DELAYED_WINDOW = 6, 3


def delayed_input(k):
    """Step k's tensor: the largest element sits in rank (k % 2)'s rows."""
    x = inputs.random_matrix(300, 256, seed=90 + k, dtype=torch.bfloat16, outlier_frac=0.002, factor=1e2)
    x[10 if k % 2 == 0 else 250, 3] = torch.tensor(3e3 * (k + 1), dtype=torch.bfloat16)
    return x


def _worker(rank, port, outdir, case):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        x = inputs.random_matrix(300, 256, seed=77, dtype=torch.bfloat16, outlier_frac=0.002, factor=1e3)
        if case == "per_tensor":
            # put the largest value in rank 1's rows so rank 0 must learn it through the exchange
            x[250, 7] = torch.tensor(5e4, dtype=torch.bfloat16)
            r0, r1 = sharded.row_shard(300, WORLD, rank, multiple=1)
            q, s, a = sharded.quantize_per_tensor_sharded(x[r0:r1].contiguous(), oracle.E5M2, ops=oracle_ops())
            np.save(os.path.join(outdir, f"q{rank}.npy"), q.numpy())
            np.save(os.path.join(outdir, f"s{rank}.npy"), np.array([s.item(), a.item()], dtype=np.float32))
        elif case == "blockwise":
            for block in ((1, 128), (128, 128)):
                r0, r1 = sharded.row_shard(300, WORLD, rank, multiple=block[0])
                q, s = sharded.quantize_blockwise_sharded(x[r0:r1].contiguous(), block, oracle.E4M3, ops=oracle_ops())
                np.save(os.path.join(outdir, f"b{block[0]}_q{rank}.npy"), q.numpy())
                np.save(os.path.join(outdir, f"b{block[0]}_s{rank}.npy"), s.numpy())
        elif case == "delayed":
            r0, r1 = sharded.row_shard(300, WORLD, rank, multiple=1)
            sc = sharded.ShardedDelayedScaler(window=DELAYED_WINDOW, fmt=oracle.E5M2, ops=oracle_delayed_ops(),
                                              device="cpu")
            for k in range(DELAYED_STEPS):
                scale_used = float(sc.scale.item())
                q = sc.step(delayed_input(k)[r0:r1].contiguous())
                np.save(os.path.join(outdir, f"d{k}_q{rank}.npy"), q.numpy())
                np.save(os.path.join(outdir, f"d{k}_s{rank}.npy"),
                        np.array([scale_used, float(sc.scale.item())], dtype=np.float32))
        elif case == "timing":
            import importlib.util
            root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
            spec = importlib.util.spec_from_file_location("bench", os.path.join(root, "bench.py"))
            bench = importlib.util.module_from_spec(spec)
            spec.loader.exec_module(bench)
            local = [1.0 + rank, 5.0 - 3 * rank, 0.25 * (rank + 1)]
            out = bench.max_over_ranks(local, WORLD, device="cpu")
            np.save(os.path.join(outdir, f"t{rank}.npy"), np.array(out))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(case):
    with tempfile.TemporaryDirectory() as d:
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_worker, args=(r, PORT[0], d, case)) for r in range(WORLD)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        return {f: np.load(os.path.join(d, f)) for f in os.listdir(d)}


PORT = [0]


@pytest.fixture(autouse=True)
def _port():
    PORT[0] = _free_port()


def test_row_shard_covers_rows_on_block_edges():
    for rows in (1, 127, 128, 129, 300, 4096, 16384 + 5):
        for world in (1, 2, 3, 8):
            for m in (1, 128):
                spans = [sharded.row_shard(rows, world, r, m) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == rows
                for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                    assert a1 == b0
                for a0, a1 in spans:
                    # every boundary inside the tensor falls on a block edge
                    assert (a0 % m == 0 or a0 == rows) and (a1 % m == 0 or a1 == rows)


def test_per_tensor_sharded_matches_unsharded():
    out = _run("per_tensor")
    x = inputs.random_matrix(300, 256, seed=77, dtype=torch.bfloat16, outlier_frac=0.002, factor=1e3)
    x[250, 7] = torch.tensor(5e4, dtype=torch.bfloat16)
    q, s, a = oracle.quantize_per_tensor(inputs.bf16_bits(x), oracle.E5M2)
    s0, s1 = out["s0.npy"], out["s1.npy"]
    assert s0[0] == s1[0] == s and s0[1] == s1[1] == a
    assert np.array_equal(np.concatenate([out["q0.npy"], out["q1.npy"]]), q)


def test_blockwise_sharded_matches_unsharded():
    out = _run("blockwise")
    x = inputs.random_matrix(300, 256, seed=77, dtype=torch.bfloat16, outlier_frac=0.002, factor=1e3)
    for br in (1, 128):
        q, s = oracle.quantize_blockwise(inputs.bf16_bits(x), br, 128, oracle.E4M3)
        assert np.array_equal(np.concatenate([out[f"b{br}_q0.npy"], out[f"b{br}_q1.npy"]]), q)
        assert np.array_equal(np.concatenate([out[f"b{br}_s0.npy"], out[f"b{br}_s1.npy"]]), s)


def test_bench_timing_is_max_over_ranks():
    out = _run("timing")
    want = [2.0, 5.0, 0.5]
    assert out["t0.npy"].tolist() == want and out["t1.npy"].tolist() == want


def test_delayed_scaling_sharded_matches_unsharded():
    """Each rank casts its rows with the shared scale, then the ranks all-reduce the amax for the history
    update: codes, scales used and next scales equal the whole tensor's on one device, step after step,
    although the largest element alternates between the ranks."""
    out = _run("delayed")
    ref = oracle.AmaxHistory(DELAYED_WINDOW, oracle.E5M2)
    for k in range(DELAYED_STEPS):
        xh = inputs.bf16_bits(delayed_input(k))
        s_ref = float(ref.scale[0])
        oq, _, oa = oracle.quantize_per_tensor(xh, oracle.E5M2, scale=s_ref)
        ref.update(oa)
        q = np.concatenate([out[f"d{k}_q{r}.npy"].reshape(-1, 256) for r in range(WORLD)])
        assert np.array_equal(q, oq.reshape(q.shape)), k
        for r in range(WORLD):
            used, nxt = out[f"d{k}_s{r}.npy"]
            assert np.float32(used) == np.float32(s_ref) and np.float32(nxt) == ref.scale[0], (k, r)
    assert float(ref.scale[0]) != 1.0  # the window filled and the scale moved off its initial value
