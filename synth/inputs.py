"""Seeded synthetic tensors with the shapes and value distributions of the
QLoRA workloads (LLaMA-shaped linears, N(0, 0.02^2) pretrained-like weights,
N(0, 1) activations and output gradients, LoRA factors initialised as
L1 ~ N(0, 1/in), L2 ~ N(0, 0.01^2)).

Host tensors come from NumPy's PCG64 generator; large tensors can be drawn
directly on a CUDA device with a seeded ``torch.Generator`` (same recipe,
different stream of random numbers).  bfloat16 tensors are produced by
rounding float32 draws with torch's own conversion.
"""

from __future__ import annotations

import numpy as np
import torch

WEIGHT_STD = 0.02
L2_STD = 0.01


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_f32(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    return (g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32 NumPy array -> bfloat16 CPU tensor (torch's round-to-nearest-even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal_bf16(g: np.random.Generator, shape, std: float = 1.0) -> torch.Tensor:
    return to_bf16(normal_f32(g, shape, std))


def weight_f32(g: np.random.Generator, n_out: int, k_in: int, std: float = WEIGHT_STD) -> np.ndarray:
    return normal_f32(g, (n_out, k_in), std)


def weight_bf16_with_outliers(g: np.random.Generator, n_out: int, k_in: int,
                              std: float = WEIGHT_STD, frac: float = 1e-3,
                              sigmas: float = 10.0) -> torch.Tensor:
    """bf16 N(0, std^2) weights with exactly round(frac * numel) positions,
    drawn uniformly without replacement, set to +/- sigmas * std (random sign)."""
    w = normal_f32(g, (n_out, k_in), std).reshape(-1)
    n_out_lier = int(round(frac * w.size))
    pos = g.choice(w.size, size=n_out_lier, replace=False)
    sign = np.where(g.random(n_out_lier) < 0.5, -1.0, 1.0).astype(np.float32)
    w[pos] = sign * np.float32(sigmas * std)
    return to_bf16(w.reshape(n_out, k_in))


def lora_factors(g: np.random.Generator, k_in: int, n_out: int, r: int):
    """(L1 [k_in, r] ~ N(0, 1/k_in), L2 [r, n_out] ~ N(0, 0.01^2)) as bf16."""
    L1 = normal_bf16(g, (k_in, r), 1.0 / np.sqrt(k_in))
    L2 = normal_bf16(g, (r, n_out), L2_STD)
    return L1, L2


def device_normal(shape, std: float, seed: int, device, dtype=torch.float32) -> torch.Tensor:
    """Large seeded N(0, std^2) tensor drawn on ``device`` (float32, then cast)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    t.mul_(std)
    return t if dtype == torch.float32 else t.to(dtype)


def device_weight_with_outliers(n_out: int, k_in: int, seed: int, device,
                                std: float = WEIGHT_STD, frac: float = 1e-3,
                                sigmas: float = 10.0) -> torch.Tensor:
    """Device version of ``weight_bf16_with_outliers`` (bf16)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    w = torch.randn(n_out * k_in, generator=gen, device=device, dtype=torch.float32).mul_(std)
    n_out_lier = int(round(frac * w.numel()))
    pos = torch.randperm(w.numel(), generator=gen, device=device)[:n_out_lier]
    sign = torch.where(torch.rand(n_out_lier, generator=gen, device=device) < 0.5, -1.0, 1.0)
    w[pos] = sign * (sigmas * std)
    return w.view(n_out, k_in).to(torch.bfloat16)


def dropout_mask(g: np.random.Generator, M: int, K: int, p: float) -> np.ndarray:
    """Keep mask of LoRA dropout, bit-packed: uint32 [M, K/32], bit b of word w
    of row i keeps element (i, 32 w + b); each element is kept with
    probability 1 - p, independently.  K must be a multiple of 32."""
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    keep = g.random((M, K), dtype=np.float32) >= np.float32(p)
    return pack_mask(keep)


def pack_mask(keep: np.ndarray) -> np.ndarray:
    """bool [M, K] -> uint32 [M, K/32] (element 32 w + b in bit b of word w)."""
    M, K = keep.shape
    bits = keep.reshape(M, K // 32, 32).astype(np.uint64) << np.arange(32, dtype=np.uint64)
    return bits.sum(axis=-1).astype(np.uint32)


def unpack_mask(words: np.ndarray, K: int) -> np.ndarray:
    """uint32 [M, K/32] -> bool [M, K], the inverse of pack_mask."""
    w = np.asarray(words, dtype=np.uint32)
    return ((w[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool).reshape(w.shape[0], K)
