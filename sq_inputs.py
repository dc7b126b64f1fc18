"""Seeded synthetic inputs for the SmoothQuant W8A8 linear layer.

This module only draws random numbers: it holds none of the method's arithmetic.
Both the CUDA path and the CPU oracle are fed the very same bytes it produces.

Recipe (after the activation-outlier description in "4.2 W8A8 量化与 SmoothQuant",
sec. 1.1: about 1% of channels, about 100x larger, the same channels for every
token).  Draw order from ``numpy.random.default_rng(seed)`` (PCG64):

1. outlier channel indices: ``rng.choice(K, round(frac * K), replace=False)``
2. per-outlier multipliers: a fixed factor, or log-uniform on [lo, hi]
   (``exp(rng.uniform(ln lo, ln hi, n))``)
3. X ~ N(0, 1) float32 of shape [M, K]; the outlier columns are multiplied
4. W ~ N(0, w_std) float32 of shape [K, N] (row j = input channel j)
5. LayerNorm gamma ~ U(0.5, 1.5), beta = 0 (or ~ N(0, beta_std) when asked)

bfloat16 tensors are produced by round-to-nearest-even casting (torch) and are
returned as ``numpy.uint16`` bit patterns.  ``torch_case`` draws the same recipe
with a seeded ``torch.Generator`` directly on a device, for full-size workloads
whose values the oracle then reads back from the device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass
class LinearCase:
    M: int
    K: int
    N: int
    x: np.ndarray            # [M, K] float32, or uint16 bf16 bits
    W: np.ndarray            # [K, N] float32, or uint16 bf16 bits
    gamma: np.ndarray        # [K] float32
    beta: np.ndarray | None  # [K] float32 or None
    outlier_idx: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (round to nearest even, via torch)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _multipliers(rng, n, outlier_mult):
    if isinstance(outlier_mult, tuple):
        lo, hi = outlier_mult
        return np.exp(rng.uniform(math.log(lo), math.log(hi), n)).astype(np.float32)
    return np.full(n, float(outlier_mult), np.float32)


def make_case(M: int, K: int, N: int, seed: int, *, x_dtype: str = "bf16", w_dtype: str = "bf16",
              w_std: float = 0.02, outlier_frac: float = 0.01, outlier_mult=100.0,
              beta_std: float = 0.0) -> LinearCase:
    rng = np.random.default_rng(seed)
    n_out = int(round(outlier_frac * K))
    idx = np.sort(rng.choice(K, n_out, replace=False)) if n_out > 0 else np.zeros(0, np.int64)
    mult = _multipliers(rng, n_out, outlier_mult)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if n_out:
        x[:, idx] *= mult[None, :]
    W = rng.normal(0.0, w_std, (K, N)).astype(np.float32)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32)
    beta = rng.normal(0.0, beta_std, K).astype(np.float32) if beta_std > 0 else None
    if x_dtype == "bf16":
        x = to_bf16_bits(x)
    if w_dtype == "bf16":
        W = to_bf16_bits(W)
    return LinearCase(M, K, N, x, W, gamma, beta, idx)


def tiny_case() -> LinearCase:
    """16 tokens x K=256 -> N=256, fp32, 3 fixed outlier channels x100, W ~ N(0, 0.02), seed 0."""
    return make_case(16, 256, 256, 0, x_dtype="f32", w_dtype="f32", w_std=0.02, outlier_mult=100.0)


def torch_case(M: int, K: int, N: int, seed: int, device, *, w_std: float = 0.02,
               outlier_frac: float = 0.01, outlier_mult=100.0, with_weights: bool = True):
    """Same recipe drawn on ``device`` with a seeded torch.Generator (bf16 X and W).

    Returns (x [M, K] bf16, W [K, N] bf16 or None, gamma [K] f32, outlier index tensor)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    n_out = int(round(outlier_frac * K))
    idx = torch.randperm(K, generator=g, device=device)[:n_out].sort().values
    if isinstance(outlier_mult, tuple):
        lo, hi = outlier_mult
        u = torch.rand(n_out, generator=g, device=device)
        mult = torch.exp(math.log(lo) + (math.log(hi) - math.log(lo)) * u)
    else:
        mult = torch.full((n_out,), float(outlier_mult), device=device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if n_out:
        x[:, idx] *= mult[None, :]
    x = x.to(torch.bfloat16)
    W = None
    if with_weights:
        W = (torch.randn(K, N, generator=g, device=device, dtype=torch.float32) * w_std).to(torch.bfloat16)
    gamma = 0.5 + torch.rand(K, generator=g, device=device, dtype=torch.float32)
    return x, W, gamma, idx
