"""Seeded synthetic BF16 weight tensors for the decode workloads.

This module is shared by the oracle tests, the GPU parity tests and the
benchmark. It holds no codec arithmetic: only random draws, fp32 -> BF16
rounding (torch, round to nearest even) and the tensor shapes of the models
the workloads imitate. No real checkpoints or datasets are used; these
tensors stand in for the LLM weights the DFloat11 page ("70% Size, 100%
Accuracy", section "Przelom: DFloat11") and the codebook pages talk about.

Every generator takes an integer seed and a torch device. The same seed on the
same device always gives the same bytes; CPU and CUDA generators give
different (but individually deterministic) streams, so callers that compare
two implementations hand both of them the same tensor.
"""
from __future__ import annotations

from typing import Iterator

import numpy as np
import torch

# Llama-3-8B decoder-layer linear weights: (name, rows, cols).
LLAMA3_8B_LAYER = (
    ("q", 4096, 4096),
    ("k", 1024, 4096),
    ("v", 1024, 4096),
    ("o", 4096, 4096),
    ("gate", 14336, 4096),
    ("up", 14336, 4096),
    ("down", 4096, 14336),
)
LLAMA3_8B_LAYERS = 32
LLAMA3_8B_HIDDEN = 4096

# Llama-3-70B: hidden 8192, FFN 28672, 64 query / 8 KV heads of dim 128.
LLAMA3_70B_LAYER = (
    ("q", 8192, 8192),
    ("k", 1024, 8192),
    ("v", 1024, 8192),
    ("o", 8192, 8192),
    ("gate", 28672, 8192),
    ("up", 28672, 8192),
    ("down", 8192, 28672),
)
LLAMA3_70B_LAYERS = 80
LLAMA3_70B_HIDDEN = 8192

VOCAB = 128256

EMBED_SEED = 900000
LM_HEAD_SEED = 900001
SEED_70B_OFFSET = 1_000_000


def tensor_seed(layer: int, t: int, offset: int = 0) -> int:
    """Seed of tensor t (q,k,v,o,gate,up,down = 0..6) of a decoder layer."""
    return offset + 1000 * layer + t


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, seed: int, sigma: float | None = None,
                sigma_range: tuple[float, float] | None = None,
                outlier_frac: float = 0.0, outlier_scale: float = 20.0,
                device="cpu") -> torch.Tensor:
    """N(0, sigma) weights rounded to BF16.

    If ``sigma`` is None it is the first draw of the tensor's generator,
    uniform in ``sigma_range``. A fraction ``outlier_frac`` of the entries
    (chosen by a second uniform draw per entry) is multiplied by
    ``outlier_scale`` before rounding.
    """
    g = _gen(seed, device)
    if sigma is None:
        lo, hi = sigma_range
        sigma = lo + (hi - lo) * float(torch.rand((), generator=g, device=device, dtype=torch.float64))
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    x.mul_(sigma)
    if outlier_frac > 0.0:
        mask = torch.rand(shape, generator=g, device=device, dtype=torch.float32) < outlier_frac
        x[mask] *= outlier_scale
        del mask
    return x.to(torch.bfloat16)


def normal_fp16(shape, seed: int, sigma: float, outlier_frac: float = 0.0, outlier_scale: float = 20.0,
                device="cpu") -> torch.Tensor:
    """N(0, sigma) weights rounded to FP16 (same draws as normal_bf16 with a
    fixed sigma, different rounding): the FP16 proof-of-concept workload of
    the codebook pages, as 16-bit patterns for either codec."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    x.mul_(sigma)
    if outlier_frac > 0.0:
        mask = torch.rand(shape, generator=g, device=device, dtype=torch.float32) < outlier_frac
        x[mask] *= outlier_scale
        del mask
    return x.to(torch.float16)


def activations_bf16(M: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    """M activation rows of width cols for a linear layer: i.i.d. N(0, 1) with
    0.1 % outliers x20 (the scale of normalised hidden states), BF16."""
    return normal_bf16((M, cols), seed, sigma=1.0, outlier_frac=1e-3, outlier_scale=20.0, device=device)


def small_square(seed: int = 0, device="cpu") -> torch.Tensor:
    """1024 x 1024 weights, i.i.d. N(0, 0.02), BF16."""
    return normal_bf16((1024, 1024), seed, sigma=0.02, device=device)


def llama_layer_tensors(layer: int, shapes=LLAMA3_8B_LAYER, sigma_range=(0.01, 0.04),
                        seed_offset: int = 0, device="cpu") -> Iterator[tuple[str, torch.Tensor]]:
    """The seven linear weights of one decoder layer, N(0, sigma) + 0.1 % outliers x20."""
    for t, (name, rows, cols) in enumerate(shapes):
        yield name, normal_bf16((rows, cols), tensor_seed(layer, t, seed_offset),
                                sigma_range=sigma_range, outlier_frac=1e-3,
                                outlier_scale=20.0, device=device)


def llama_embedding(which: str, hidden: int, sigma_range=(0.01, 0.04), seed_offset: int = 0,
                    device="cpu") -> torch.Tensor:
    """Embedding or LM-head matrix (VOCAB x hidden), same value distribution."""
    seed = seed_offset + (EMBED_SEED if which == "embed" else LM_HEAD_SEED)
    return normal_bf16((VOCAB, hidden), seed, sigma_range=sigma_range, outlier_frac=1e-3,
                       outlier_scale=20.0, device=device)


def _bf16_bits(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16).view(torch.int16).to(torch.int32) & 0xFFFF


def codebook_table(U: int, seed: int, device="cpu") -> torch.Tensor:
    """U distinct BF16 bit patterns (int32 in [0, 65536)).

    Entries are N(0, 0.02) draws rounded to BF16 and de-duplicated in draw
    order, until U are found or 64*U values have been drawn. Any shortfall is
    filled with distinct unused patterns chosen uniformly at random. U = 65536
    is every pattern, in a seeded random order.
    """
    if not 1 <= U <= 65536:
        raise ValueError("U must be in [1, 65536]")
    g = _gen(seed, "cpu")
    if U == 65536:
        return torch.randperm(65536, generator=g).to(torch.int32).to(device)
    seen = np.zeros(65536, dtype=bool)
    order: list[int] = []
    drawn = 0
    while len(order) < U and drawn < 64 * U:
        batch = max(1024, U)
        bits = _bf16_bits(torch.randn(batch, generator=g, dtype=torch.float32) * 0.02).numpy()
        drawn += batch
        for b in bits.tolist():
            if not seen[b]:
                seen[b] = True
                order.append(b)
                if len(order) == U:
                    break
    if len(order) < U:
        unused = np.flatnonzero(~seen)
        pick = torch.randperm(len(unused), generator=g)[: U - len(order)].numpy()
        order.extend(unused[pick].tolist())
    return torch.tensor(order, dtype=torch.int32, device=device)


def codebook_stress(U: int, n: int, seed: int, s: float = 1.1, device="cpu") -> torch.Tensor:
    """n BF16 values drawn from a U-entry table with Zipf(s) entry frequencies.

    The table comes from ``codebook_table``; a seeded permutation assigns Zipf
    ranks to its entries (p(rank r) proportional to r^-s), and the n indices
    are sampled by inverse CDF on float64 uniforms.
    """
    table = codebook_table(U, seed, device="cpu")
    g = _gen(seed + 1, "cpu")
    rank_of = torch.randperm(U, generator=g)
    p = torch.arange(1, U + 1, dtype=torch.float64).pow(-s)
    cdf = torch.cumsum(p, 0)
    cdf /= cdf[-1].clone()
    cdf[-1] = 1.0
    cdf = cdf.to(device)
    gd = _gen(seed + 2, device)
    out = torch.empty(n, dtype=torch.int16, device=device)
    step = 1 << 26
    by_rank = table[rank_of].to(device)
    for i0 in range(0, n, step):
        m = min(step, n - i0)
        u = torch.rand(m, generator=gd, device=device, dtype=torch.float64)
        r = torch.searchsorted(cdf, u).clamp_(max=U - 1)
        out[i0:i0 + m] = by_rank[r].to(torch.int16)
    return out.view(torch.bfloat16)


def uniform_patterns(n: int, seed: int, device="cpu") -> torch.Tensor:
    """n uniformly random 16-bit patterns: sign, exponent and mantissa all
    uniform (Inf, NaN and subnormal patterns included)."""
    g = _gen(seed, device)
    return torch.randint(-32768, 32768, (n,), generator=g, device=device,
                         dtype=torch.int16).view(torch.bfloat16)


def equal_exponents(n: int, bits: int, seed: int, first: int | None = None, step: int = 1,
                    device="cpu") -> torch.Tensor:
    """n patterns whose exponents take 2^bits values first, first + step, ...
    (by default consecutive and centred on 127) in equal numbers (n // 2^bits
    of each, the remainder from the first values), in random order, with
    uniform sign and mantissa bits: exponent frequencies as flat as they can
    be."""
    m = 1 << bits
    first = (128 - step * m // 2) if first is None else first
    assert 0 <= first and first + step * (m - 1) <= 255
    g = _gen(seed, device)
    e = (torch.arange(n, device=device, dtype=torch.int32) % m) * step + first
    e = e[torch.randperm(n, generator=g, device=device)]
    sm = torch.randint(0, 256, (n,), generator=g, device=device, dtype=torch.int32)
    u = ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)
    return u.to(torch.int16).view(torch.bfloat16)


def all_patterns() -> torch.Tensor:
    """Every 16-bit pattern once, ascending."""
    return torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)


def random_patterns_from(alphabet, n: int, seed: int) -> torch.Tensor:
    """n patterns drawn uniformly from a given list of 16-bit patterns."""
    g = _gen(seed, "cpu")
    a = torch.tensor([int(v) & 0xFFFF for v in alphabet], dtype=torch.int32)
    idx = torch.randint(0, len(a), (n,), generator=g)
    return a[idx].to(torch.int16).view(torch.bfloat16)


def as_u16(x: torch.Tensor) -> np.ndarray:
    """Host numpy view (uint16) of a BF16/int16 tensor's bit patterns."""
    x = x.detach()
    if x.device.type != "cpu":
        x = x.cpu()
    return x.contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def describe(n: int) -> str:
    return f"{n:,} weights ({2 * n / 1e6:.1f} MB BF16)"


__all__ = [
    "LLAMA3_8B_LAYER", "LLAMA3_70B_LAYER", "VOCAB", "tensor_seed", "normal_bf16",
    "small_square", "llama_layer_tensors", "llama_embedding", "codebook_table",
    "codebook_stress", "uniform_patterns", "all_patterns", "random_patterns_from",
    "as_u16", "describe",
]
