"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws numbers.  It holds none of the quantization
arithmetic, imports neither the CUDA binding nor the oracle, and is the one
piece both sides share: every test and benchmark input comes from here.

Every generator draws with a seeded ``torch.Generator`` (CPU by default, so
the bytes are the same on every machine; ``device="cuda"`` draws with a seeded
CUDA generator for sizes where the CPU draw is too slow), in fp32, and casts
to bf16 with torch's round-to-nearest-even where the workload is bf16.

Workloads (the page passages they follow):
  * ``relerr_outlier_tensors`` -- the "FP8 training" experiment of the
    mixed-precision handbook page: seed 0, a fresh ``randn(256, 1024)`` per
    outlier factor in (1e2, 1e4, 3e4), columns 0-3 multiplied by the factor.
  * ``scalar_values`` -- the scalar experiment of the PyTorch-FP8 page, s2.2.
  * ``weight_4096`` -- a bf16 weight, N(0, 0.02^2), for 128x128 blocks.
  * ``activation_outlier_channels`` -- bf16 activations N(0, 1) with a few
    channels scaled by 1e3 (outlier channels, handbook "FP8 training").
  * ``gradient_steps`` -- bf16 gradients with |g| log-uniform in [1e-6, 1e-2]
    and random sign, re-scaled each step by (1 + 0.1 sin k), for delayed
    scaling over an amax history (PyTorch-FP8 page, s4.2; s1.2 on gradient
    magnitudes from 1e-2 down to 1e-6).
  * ``sweep_tensor`` -- bf16 N(0, 1) of 2^n elements with 0.1% of the
    entries scaled by 1e3, shaped [2^n / 4096, 4096].
"""
from __future__ import annotations

import math

import torch

SCALAR_VALUES = (1.0, 1.5, 1.25, 1.125, 1.1, 0.1, 448.0, 449.0, 0.015625, 0.0001)
OUTLIER_FACTORS = (1e2, 1e4, 3e4)


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def scalar_values() -> torch.Tensor:
    """The ten scalars of the scalar experiment, fp32."""
    return torch.tensor(SCALAR_VALUES, dtype=torch.float32)


def relerr_outlier_tensors(seed: int = 0, rows: int = 256, cols: int = 1024):
    """Yield (factor, fp32 [rows, cols]) in the handbook's draw order: one generator, a fresh draw per factor."""
    g = _gen(seed)
    out = []
    for factor in OUTLIER_FACTORS:
        a = torch.randn(rows, cols, generator=g, dtype=torch.float32)
        a[:, :4] *= factor
        out.append((factor, a))
    return out


def weight_4096(seed: int = 1, rows: int = 4096, cols: int = 4096, std: float = 0.02,
                device: str = "cpu") -> torch.Tensor:
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, dtype=torch.float32, device=device) * std
    return w.to(torch.bfloat16)


def activation_outlier_channels(seed: int = 2, rows: int = 16384, cols: int = 7168,
                                n_outlier: int = 8, factor: float = 1e3,
                                device: str = "cpu") -> torch.Tensor:
    g = _gen(seed, device)
    a = torch.randn(rows, cols, generator=g, dtype=torch.float32, device=device)
    ch = torch.randperm(cols, generator=g, device=device)[:n_outlier]
    a[:, ch] *= factor
    return a.to(torch.bfloat16)


def gradient_base(seed: int = 3, rows: int = 8192, cols: int = 8192,
                  lo: float = 1e-6, hi: float = 1e-2, device: str = "cpu") -> torch.Tensor:
    """fp32 gradient with log-uniform magnitude in [lo, hi] and a random sign."""
    g = _gen(seed, device)
    u = torch.rand(rows, cols, generator=g, dtype=torch.float32, device=device)
    mag = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    sign = torch.randint(0, 2, (rows, cols), generator=g, device=device).to(torch.float32) * 2 - 1
    return mag * sign


def gradient_step(base: torch.Tensor, k: int) -> torch.Tensor:
    """Step k's bf16 gradient: base * fp32(1 + 0.1 sin k)."""
    f = torch.tensor(1.0 + 0.1 * math.sin(k), dtype=torch.float32)
    return (base * f.to(base.device)).to(torch.bfloat16)


def sweep_tensor(log2_n: int, seed: int = 4, cols: int = 4096, outlier_frac: float = 1e-3,
                 factor: float = 1e3, device: str = "cpu") -> torch.Tensor:
    n = 1 << log2_n
    cols = min(cols, n)
    g = _gen(seed, device)
    x = torch.randn(n, generator=g, dtype=torch.float32, device=device)
    mask = torch.rand(n, generator=g, dtype=torch.float32, device=device) < outlier_frac
    x[mask] *= factor
    return x.view(n // cols, cols).to(torch.bfloat16)


def random_matrix(rows: int, cols: int, seed: int, dtype=torch.bfloat16, scale: float = 1.0,
                  outlier_frac: float = 0.0, factor: float = 1.0, device: str = "cpu") -> torch.Tensor:
    """Generic N(0, scale^2) matrix with optional sparse outliers, for shape and edge-case tests."""
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, dtype=torch.float32, device=device) * scale
    if outlier_frac > 0:
        mask = torch.rand(rows, cols, generator=g, dtype=torch.float32, device=device) < outlier_frac
        x[mask] *= factor
    return x.to(dtype)


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
