"""Helpers for the GPU parity tests.

- Guard-band buffers: outputs are views into a larger buffer whose margins are
  filled with 0xA5 and checked after the call, to catch out-of-bounds writes.
- Threaded oracle: the oracle is single-threaded C and ctypes releases the GIL,
  so large cases split rows into independent chunks (block rows stay whole)
  and run the oracle on them in parallel.  The chunking is by rows only; every
  chunk is the oracle's own computation on that part of the tensor.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from fine_grained_block_b200 import inputs

NTHREADS = max(1, min(32, len(os.sched_getaffinity(0))))
_pool = ThreadPoolExecutor(max_workers=NTHREADS)

TORCH_OF = {oracle.E4M3: torch.float8_e4m3fn, oracle.E5M2: torch.float8_e5m2}


class Guarded:
    """A CUDA tensor view with 0xA5 guard bands on both sides."""
    PAD = 4096

    def __init__(self, shape, dtype, device="cuda"):
        esize = torch.empty(0, dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * esize
        self.buf = torch.full((self.PAD + self.n + self.PAD,), 0xA5, dtype=torch.uint8, device=device)
        self.t = self.buf[self.PAD:self.PAD + self.n].view(dtype).view(shape)

    def check(self):
        head = self.buf[:self.PAD]
        tail = self.buf[self.PAD + self.n:]
        assert bool((head == 0xA5).all()) and bool((tail == 0xA5).all()), "write outside the output buffer"


def host_input(t: torch.Tensor) -> np.ndarray:
    """The oracle's view of a CPU tensor: float32 array or bf16 bit patterns."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def _row_chunks(rows: int, br: int):
    per = max(br, math.ceil(rows / (NTHREADS * 4) / br) * br)
    return [(r, min(rows, r + per)) for r in range(0, rows, per)]


def oracle_blockwise(x: np.ndarray, br: int, bc: int, fmt: int):
    R, C = x.shape
    chunks = _row_chunks(R, br)
    parts = list(_pool.map(lambda rc: oracle.quantize_blockwise(x[rc[0]:rc[1]], br, bc, fmt), chunks))
    if not parts:
        return np.zeros((R, C), np.uint8), np.zeros((0, math.ceil(C / bc)), np.float32)
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def oracle_amax(x: np.ndarray) -> np.float32:
    flat = x.reshape(-1)
    step = max(1, math.ceil(flat.size / (NTHREADS * 4)))
    parts = list(_pool.map(lambda i: oracle.amax(flat[i:i + step]), range(0, flat.size, step)))
    return np.float32(max(parts)) if parts else np.float32(0)


def oracle_per_tensor(x: np.ndarray, fmt: int, scale=None):
    """Returns (codes, scale used, amax) exactly as oracle.quantize_per_tensor, computed in row chunks."""
    a = oracle_amax(x)
    s = oracle.scale_from_amax(a, fmt) if scale is None else np.float32(scale)
    flat = x.reshape(-1)
    step = max(1, math.ceil(flat.size / (NTHREADS * 4)))
    parts = list(_pool.map(lambda i: oracle.quantize_per_tensor(flat[i:i + step], fmt, scale=float(s))[0],
                           range(0, flat.size, step)))
    q = np.concatenate(parts).reshape(x.shape) if parts else np.zeros(x.shape, np.uint8)
    return q, s, a


def oracle_cast(x: np.ndarray, fmt: int, scale) -> np.ndarray:
    """oracle.quantize_per_tensor's codes for a given scale, in chunks (no amax pass)."""
    flat = x.reshape(-1)
    step = max(1, math.ceil(flat.size / (NTHREADS * 4)))
    parts = list(_pool.map(lambda i: oracle.quantize_per_tensor(flat[i:i + step], fmt, scale=float(scale))[0],
                           range(0, flat.size, step)))
    return np.concatenate(parts).reshape(x.shape) if parts else np.zeros(x.shape, np.uint8)


def oracle_dequant(q: np.ndarray, fmt: int, scales: np.ndarray, br: int, bc: int, out_dtype: int):
    if q.ndim == 1:
        q = q.reshape(1, -1)
    R, C = q.shape
    if br == 0:
        chunks = _row_chunks(R, 1)
        parts = list(_pool.map(lambda rc: oracle.dequantize(q[rc[0]:rc[1]], fmt, scales, 0, 0, out_dtype), chunks))
    else:
        chunks = _row_chunks(R, br)
        parts = list(_pool.map(
            lambda rc: oracle.dequantize(q[rc[0]:rc[1]], fmt, scales[rc[0] // br:math.ceil(rc[1] / br)], br, bc,
                                         out_dtype), chunks))
    return np.concatenate(parts)


def oracle_gemm(qa, sa, a_fmt, qb, sb, b_fmt, b_block=128):
    """oracle.gemm_blockwise over row chunks of A in parallel (each chunk's rows are the oracle's own
    computation)."""
    M = qa.shape[0]
    per = max(1, math.ceil(M / (NTHREADS * 2)))
    parts = list(_pool.map(lambda r: oracle.gemm_blockwise(qa[r:r + per], sa[r:r + per], a_fmt, qb, sb, b_fmt,
                                                           b_block=b_block), range(0, M, per)))
    return np.concatenate(parts)


def oracle_mx(x: np.ndarray, fmt: int, rule: int):
    """oracle.quantize_mx in row chunks: (codes, e8m0)."""
    R, C = x.shape
    chunks = _row_chunks(R, 1)
    parts = list(_pool.map(lambda rc: oracle.quantize_mx(x[rc[0]:rc[1]], fmt, rule), chunks))
    if not parts:
        return np.zeros((R, C), np.uint8), np.zeros((0, math.ceil(C / 32)), np.uint8)
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def oracle_dequant_mx(q: np.ndarray, fmt: int, e8m0: np.ndarray, out_dtype: int):
    chunks = _row_chunks(q.shape[0], 1)
    parts = list(_pool.map(lambda rc: oracle.dequantize_mx(q[rc[0]:rc[1]], fmt, e8m0[rc[0]:rc[1]], out_dtype),
                           chunks))
    return np.concatenate(parts)


def _nan_mask(bits: np.ndarray, kind: str) -> np.ndarray:
    if kind == "f32":
        return ((bits & 0x7F800000) == 0x7F800000) & ((bits & 0x007FFFFF) != 0)
    return ((bits & 0x7F80) == 0x7F80) & ((bits & 0x007F) != 0)


def assert_bytes_equal(got: torch.Tensor, want: np.ndarray, what: str):
    """Bit-for-bit equality.  For fp32 / bf16 values, two NaNs count as equal whatever their payload
    (the contract fixes NaN-ness, not the NaN bit pattern)."""
    g = got.detach().cpu().contiguous()
    kind = None
    if g.dtype == torch.bfloat16:
        g = g.view(torch.int16).numpy().view(np.uint16)
        kind = "bf16"
    elif g.dtype == torch.float32:
        g = g.numpy().view(np.uint32)
        want = want.view(np.uint32) if want.dtype == np.float32 else want
        kind = "f32"
    else:
        g = g.numpy()
    want = np.asarray(want).reshape(g.shape)
    diff = g != want
    if kind is not None:
        diff &= ~(_nan_mask(g, kind) & _nan_mask(want, kind))
    if diff.any():
        bad = np.argwhere(diff)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches; first at {i}: got {g[i]!r} want {want[i]!r}")


def to_cuda(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().to("cuda")


def fp32_bits(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).view(np.uint32)
