"""Array plumbing shared by the GPU tests (numpy <-> torch device tensors)."""
from __future__ import annotations

import numpy as np
import torch

from group_wise_affine_qlinear_b200 import synthetic as S

# Tokens per tile of the fused tensor-core kernel (its dispatch record says "... x 192t ..."); sampled
# rows include both sides of every boundary between such tiles.
FUSED_TILE_TOKENS = 192


def to_dev_codes(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes).view(np.int32)).cuda()


def to_dev_f16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float16)).cuda()


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def random_layer(rng: np.random.Generator, M: int, K: int, N: int):
    """Small random layer with the synthetic recipe's distributions (codes, scales, biases, x bits)."""
    codes = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint32)
    s = np.exp(rng.uniform(np.log(1e-3), np.log(2e-2), size=(N, K // 64))).astype(np.float16)
    b = (-7.5 * s.astype(np.float64) + 0.1 * s.astype(np.float64) * rng.standard_normal(s.shape)).astype(np.float16)
    sigma = np.exp(rng.standard_normal(K)).astype(np.float32)
    x = S.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) * sigma[None, :])
    return x, codes, s, b


def random_layer8(rng: np.random.Generator, M: int, K: int, N: int):
    """Small random layer with 8-bit codes, drawn as in the synthetic module's 8-bit recipe."""
    codes = rng.integers(0, 1 << 32, size=(N, K // 4), dtype=np.uint32)
    s = (np.exp(rng.uniform(np.log(1e-3), np.log(2e-2), size=(N, K // 64))) / 17.0).astype(np.float16)
    b = (-127.5 * s.astype(np.float64) + 1.7 * s.astype(np.float64) * rng.standard_normal(s.shape)).astype(np.float16)
    sigma = np.exp(rng.standard_normal(K)).astype(np.float32)
    x = S.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) * sigma[None, :])
    return x, codes, s, b


def sample_rows(M: int, n_random: int = 64, seed: int = 0, tile: int = 128) -> np.ndarray:
    """Row 0, row M-1, both sides of every tile boundary, and random rows."""
    rows = {0, M - 1}
    for t in range(tile, M, tile):
        rows.update((t - 1, t))
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, M, size=min(n_random, M)).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < M))
