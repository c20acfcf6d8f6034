"""Seeded synthetic inputs: BF16 weight matrices and activations.

This module only draws random numbers.  It holds none of the compression
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (the same for every workload):
  * weights: ``torch.Generator('cpu').manual_seed(seed)``, then
    ``randn(n*k, float32) * sigma``; then ``randperm(n*k)[:round(frac*n*k)]``
    from the same generator picks outlier positions, whose values are
    replaced by ``randn(count) * outlier_sigma``; finally ``.to(bfloat16)``
    (round to nearest even) and the raw 16-bit patterns are returned.
  * activations: a separate generator seeded ``10_000 + seed``, ``randn(m, k)``
    rounded to BF16.

The weight shapes are those of the Llama MLP projections (gate/up [F, H],
down [H, F]); no trained weights are used.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


def weights_bf16(n: int, k: int, sigma: float = 0.02, outlier_frac: float = 0.0,
                 outlier_sigma: float = 1.0, seed: int = 0) -> np.ndarray:
    """uint16[n, k] BF16 bit patterns of N(0, sigma^2) weights with outliers."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    w = torch.randn(n * k, generator=g, dtype=torch.float32) * sigma
    count = int(round(outlier_frac * n * k))
    if count:
        idx = torch.randperm(n * k, generator=g)[:count]
        w[idx] = torch.randn(count, generator=g, dtype=torch.float32) * outlier_sigma
    bits = w.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return bits.reshape(n, k).copy()


def activations_bf16(m: int, k: int, seed: int = 0) -> np.ndarray:
    """uint16[m, k] BF16 bit patterns of N(0, 1) activations (seed 10000+seed)."""
    g = torch.Generator("cpu").manual_seed(10_000 + int(seed))
    x = torch.randn(m, k, generator=g, dtype=torch.float32)
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """Plain reinterpretation helper for reports (uint16 -> float32)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Projection:
    name: str
    n: int
    k: int


# Llama-3.1-8B MLP (hidden 4096, intermediate 14336) and Llama-70B MLP
# (hidden 8192, intermediate 28672); W is [out, in] so that Y = X W^T.
LLAMA8B = (Projection("gate", 14336, 4096), Projection("up", 14336, 4096),
           Projection("down", 4096, 14336))
LLAMA70B = (Projection("gate", 28672, 8192), Projection("up", 28672, 8192),
            Projection("down", 8192, 28672))


def small_matrix(seed: int = 0) -> np.ndarray:
    """1024 x 1024, N(0, 0.02^2), 0.1% N(0, 2^2) outliers."""
    return weights_bf16(1024, 1024, 0.02, 0.001, 2.0, seed)


def llama8b_layer(seed_base: int = 1, sigma: float = 0.02, frac: float = 0.0005):
    """The three 8B MLP matrices with seeds seed_base, seed_base+1, seed_base+2."""
    return {p.name: weights_bf16(p.n, p.k, sigma, frac, 1.0, seed_base + i)
            for i, p in enumerate(LLAMA8B)}
