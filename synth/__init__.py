"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers; it holds none of the quantization or
product arithmetic, and it imports neither the oracle nor the CUDA binding.
Both sides receive the same bytes: a caller draws once and hands copies of the
one tensor to the oracle and to the CUDA path.

Distributions follow the workloads of the pages' decode setting:
  * ``gaussian_weights``: N(0, std^2) entries with a Bernoulli(frac) mask that
    multiplies the selected entries by ``mult`` (0.1 % of entries x10 by
    default), the heavy-tailed "few large weights" picture of the Q4_0
    chapter's section 4.1.1 and 4.5.
  * ``logstd_weights``: every run of 32 consecutive weights along a row gets its
    own std drawn log-uniformly from [lo, hi], so block scales vary the way the
    K-quants post's eight sub-scales (0.08 .. 0.18) do.
  * ``activations``: N(0, 1) in the requested dtype.
"""
from __future__ import annotations

import math

import torch

__all__ = ["gaussian_weights", "logstd_weights", "activations", "generator"]


def generator(seed: int, device: str | torch.device = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_weights(M: int, K: int, seed: int, std: float = 0.02,
                     frac: float = 0.001, mult: float = 10.0,
                     device: str | torch.device = "cpu") -> torch.Tensor:
    """fp32 [M, K]: N(0, std^2) with a Bernoulli(frac) set of entries scaled by mult."""
    g = generator(seed, device)
    w = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    w.mul_(std)
    if frac > 0.0:
        u = torch.rand((M, K), generator=g, device=device, dtype=torch.float32)
        w = torch.where(u < frac, w * mult, w)
    return w


def logstd_weights(M: int, K: int, seed: int, lo: float = 0.005, hi: float = 0.05,
                   group: int = 32, device: str | torch.device = "cpu") -> torch.Tensor:
    """fp32 [M, K]: each run of ``group`` weights along a row has its own std,
    drawn log-uniformly in [lo, hi]; entries are std * N(0, 1)."""
    assert K % group == 0
    g = generator(seed, device)
    u = torch.rand((M, K // group, 1), generator=g, device=device, dtype=torch.float32)
    std = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    w = torch.randn((M, K // group, group), generator=g, device=device, dtype=torch.float32)
    return (w * std).reshape(M, K)


def activations(B: int, K: int, seed: int, dtype: torch.dtype = torch.float16,
                device: str | torch.device = "cpu") -> torch.Tensor:
    """[B, K] N(0, 1) activations, drawn in fp32 and cast to ``dtype``."""
    g = generator(seed, device)
    return torch.randn((B, K), generator=g, device=device, dtype=torch.float32).to(dtype)
