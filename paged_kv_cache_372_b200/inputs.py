"""Seeded synthetic random draws shared by the tests, the benchmark and the oracle runs.

This module holds random number generation only: no step of the attention,
cache-write or copy arithmetic lives here. Everything is drawn on the CPU from
a ``torch.Generator`` so that a seed gives the same inputs on any machine.
"""
from __future__ import annotations

import math

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, dtype: str, gen: torch.Generator, chunk: int = 1 << 26) -> torch.Tensor:
    """N(0, 1) in fp32, cast round-to-nearest-even to ``dtype`` (CPU tensor)."""
    out = torch.empty(shape, dtype=DTYPES[dtype])
    flat = out.view(-1)
    for start in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - start)
        flat[start:start + n] = torch.randn(n, generator=gen, dtype=torch.float32)
    return out


def uniform_int(lo: int, hi: int, n: int, gen: torch.Generator) -> list[int]:
    """n integers uniform on the closed range [lo, hi]."""
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


def lognormal_int(median: float, sigma: float, lo: int, hi: int, n: int,
                  gen: torch.Generator) -> list[int]:
    """round(exp(N(ln median, sigma))) clipped to [lo, hi]."""
    z = torch.randn(n, generator=gen, dtype=torch.float64)
    x = torch.exp(math.log(median) + sigma * z).round().clamp(lo, hi)
    return [int(v) for v in x.tolist()]


def permutation(n: int, gen: torch.Generator) -> list[int]:
    return torch.randperm(n, generator=gen).tolist()


def choice(n: int, k: int, gen: torch.Generator) -> list[int]:
    """k distinct integers from range(n), in random order."""
    return torch.randperm(n, generator=gen)[:k].tolist()
