"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and shapes them; it holds none of the
quantization or matmul arithmetic.  Every tensor is generated on the CPU with
``torch.Generator('cpu')`` (``randn`` in fp32, scaled, then cast with
round-to-nearest-even), so the CUDA path and the oracle consume the same bits.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, seed: int, std: float = 1.0, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from ``seed``, then cast to ``dtype``."""
    t = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        t = t * std
    return t.to(dtype)


def with_outliers(shape, seed: int, std: float = 0.02, frac: float = 0.01,
                  factor: float = 20.0, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) weight with ``frac`` of its entries (chosen uniformly without
    replacement) multiplied by ``factor``."""
    g = _gen(seed)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32) * std
    n = t.numel()
    k = int(round(frac * n))
    idx = torch.randperm(n, generator=g)[:k]
    flat = t.view(-1)
    flat[idx] = flat[idx] * factor
    return t.to(dtype)


def zipf_experts(n: int, n_experts: int, s: float, seed: int) -> torch.Tensor:
    """``n`` expert ids (int32) with P(expert k-1) proportional to k^-s."""
    p = torch.arange(1, n_experts + 1, dtype=torch.float64) ** (-s)
    idx = torch.multinomial(p / p.sum(), n, replacement=True, generator=_gen(seed))
    return idx.to(torch.int32)


def iota(shape, dtype=torch.float32) -> torch.Tensor:
    """0, 1, 2, ... laid out row-major in ``shape`` (Nx.iota)."""
    n = 1
    for d in shape:
        n *= d
    return torch.arange(n, dtype=torch.float64).reshape(tuple(shape)).to(dtype)


# ---------------------------------------------------------------------------
# The workloads, by name.  Sizes are those of the configurations the library is
# measured on; ``seed`` defaults follow "seed 0 for the tiny case, the
# configuration's position otherwise".
# ---------------------------------------------------------------------------

@dataclass
class QmmCase:
    name: str
    x: torch.Tensor            # [M, K] (or [batch, M, K] for gather)
    w: torch.Tensor            # dense weight before quantization
    group_size: int
    bits: int
    transpose: bool
    rhs_indices: Optional[torch.Tensor] = None
    lhs_indices: Optional[torch.Tensor] = None


def tiny_case(seed: int = 0) -> QmmCase:
    """f32 W [64, 128] ~ N(0,1), x f32 [2, 128] ~ N(0,1); int4, gs 64, transpose."""
    w = normal((64, 128), seed, 1.0, torch.float32)
    x = normal((2, 128), seed + 1, 1.0, torch.float32)
    return QmmCase("tiny_f32_int4_gs64", x, w, 64, 4, True)


def decode_case(m: int, seed: int = 1, n: int = 14336, k: int = 4096, bits: int = 4,
                group_size: int = 64) -> QmmCase:
    """x bf16 [m, 4096] ~ N(0,1); W bf16 [14336, 4096] ~ N(0, 0.02^2)."""
    w = normal((n, k), seed, 0.02, torch.bfloat16)
    x = normal((m, k), seed + 1000 + m, 1.0, torch.bfloat16)
    return QmmCase(f"decode_m{m}_int{bits}_gs{group_size}", x, w, group_size, bits, True)


def prefill_case(bits: int, m: int = 2048, seed: int = 2, n: int = 14336,
                 k: int = 4096, group_size: int = 64) -> QmmCase:
    """x bf16 [2048, 4096] ~ N(0,1); W bf16 [14336, 4096] ~ N(0, 0.02^2)."""
    w = normal((n, k), seed, 0.02, torch.bfloat16)
    x = normal((m, k), seed + 1000, 1.0, torch.bfloat16)
    return QmmCase(f"prefill_m{m}_int{bits}_gs{group_size}", x, w, group_size, bits, True)


def sweep_weight(seed: int = 3, n: int = 4096, k: int = 4096) -> torch.Tensor:
    """W bf16 [4096, 4096] ~ N(0, 0.02^2) with 1% of entries x20."""
    return with_outliers((n, k), seed, 0.02, 0.01, 20.0, torch.bfloat16)


def sweep_x(m: int, seed: int = 3, k: int = 4096) -> torch.Tensor:
    return normal((m, k), seed + 1000 + m, 1.0, torch.bfloat16)


def moe_case(seed: int = 4, n_experts: int = 8, n: int = 14336, k: int = 4096,
             tokens: int = 512, zipf_s: float = 1.2) -> QmmCase:
    """8 stacked experts W bf16 [8, 14336, 4096] ~ N(0, 0.02^2); x bf16
    [512, 1, 4096] ~ N(0,1); rhs_indices int32 [512] ~ Zipf(1.2) over experts."""
    w = normal((n_experts, n, k), seed, 0.02, torch.bfloat16)
    x = normal((tokens, 1, k), seed + 1000, 1.0, torch.bfloat16)
    rhs = zipf_experts(tokens, n_experts, zipf_s, seed + 2000)
    return QmmCase("moe_e8_t512_int4_gs64", x, w, 64, 4, True, rhs_indices=rhs)
