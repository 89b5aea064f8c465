"""Seeded synthetic workloads for the group-wise affine W4 g64 quantized linear.

Input generation only.  This module draws packed 4-bit codes, f16 group scales
and biases, and bf16 activations with the shapes and value distributions of the
Ideogram 4 DiT projections (aimarketly "Ideogram-4-IQ4_M": f16 scale + f16 bias
per 64 weights; jimmysue "Ideogram 4" notes, sec. 2.8 spec table: hidden 4608,
13 x 4096 = 53248 text features, 4096 image tokens at 1024^2).  It holds none of
the layer's arithmetic: no dequantization, no quantization fit and no matmul.
The CPU oracle and the CUDA path both consume exactly the arrays returned here.

Random streams are numpy's Philox4x64 (a published counter-based generator),
keyed by (seed, tensor id), so every array is reproducible on any host and can
be regenerated block by block.

Recipe (shared by every workload):
  * codes: uniform random 32-bit words; each word holds 8 codes, low nibble
    first, so every code is an independent uniform integer in [0, 15];
  * scale s = RN_f16(exp(U(ln 1e-3, ln 2e-2)));
  * bias  b = RN_f16(-7.5 * s + N(0, (0.1 * s)^2)) computed in float64 from the
    stored f16 scale;
  * activations x[m][j] = RN_bf16(z * sigma_j), z ~ N(0, 1), sigma_j = exp(N(mu_j, 1)),
    mu_j = 0, except the long-K text projection, whose 13 channel blocks of
    4096 get mu = -1.5 + 0.25 * block to mimic 13 concatenated encoder layers.

8-bit workloads (the Q8 pack of huggingface "SceneWorks/ideogram-4-mlx",
Versions; aimarketly "Ideogram-4-IQ4_M", Conversion, keeps the conditioning
projection at 8 bits): codes uint32 [N][K/4], each word 4 uniform codes in
[0, 255], low byte first; scale s = RN_f16(exp(U(ln 1e-3, ln 2e-2)) / 17) and
bias b = RN_f16(-127.5 * s + N(0, (1.7 * s)^2)), so a group spans the same
range of weights as a 4-bit group (255 s = 15 * 17 s).
"""
from __future__ import annotations

import dataclasses
import hashlib

import numpy as np

GROUP = 64
ROW_BLOCK = 128          # activation rows drawn per Philox stream

# Tensor ids (upper 32 bits of the Philox key's second word).
_TID_CODES = 1
_TID_SCALES = 2
_TID_BIASES = 3
_TID_X = 4
_TID_SIGMA = 5
_TID_DENSE_W = 6


def _rng(seed: int, tid: int, sub: int) -> np.random.Generator:
    key = np.array([seed, (tid << 32) | sub], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bit patterns.

    Used only to store generated activations in the bf16 input format.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def weights(seed: int, widx: int, N: int, K: int):
    """Packed codes uint32 [N][K/8], scales float16 [N][K/64], biases float16 [N][K/64]."""
    assert K % GROUP == 0
    G = K // GROUP
    codes = _rng(seed, _TID_CODES, widx).integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint32)
    lo, hi = np.log(1e-3), np.log(2e-2)
    s = np.exp(_rng(seed, _TID_SCALES, widx).uniform(lo, hi, size=(N, G))).astype(np.float16)
    s64 = s.astype(np.float64)
    noise = _rng(seed, _TID_BIASES, widx).standard_normal(size=(N, G))
    b = (-7.5 * s64 + noise * (0.1 * s64)).astype(np.float16)
    return codes, s, b


def weights8(seed: int, widx: int, N: int, K: int):
    """8-bit packed codes uint32 [N][K/4], scales float16 [N][K/64], biases float16 [N][K/64]."""
    assert K % GROUP == 0
    G = K // GROUP
    codes = _rng(seed, _TID_CODES, widx).integers(0, 1 << 32, size=(N, K // 4), dtype=np.uint32)
    lo, hi = np.log(1e-3), np.log(2e-2)
    s = (np.exp(_rng(seed, _TID_SCALES, widx).uniform(lo, hi, size=(N, G))) / 17.0).astype(np.float16)
    s64 = s.astype(np.float64)
    noise = _rng(seed, _TID_BIASES, widx).standard_normal(size=(N, G))
    b = (-127.5 * s64 + noise * (1.7 * s64)).astype(np.float16)
    return codes, s, b


def channel_sigma(seed: int, xidx: int, K: int, block_means: bool = False) -> np.ndarray:
    z = _rng(seed, _TID_SIGMA, xidx).standard_normal(size=K)
    mu = np.zeros(K)
    if block_means:
        mu = -1.5 + 0.25 * (np.arange(K) // 4096)
    return np.exp(mu + z).astype(np.float32)


def activations(seed: int, xidx: int, M: int, K: int, block_means: bool = False,
                out: np.ndarray | None = None) -> np.ndarray:
    """bf16 activations as uint16 bit patterns [M][K], drawn in blocks of ROW_BLOCK rows.

    Row r always comes from stream (seed, x, xidx, r // ROW_BLOCK), so the first M
    rows of a larger draw equal a draw of M rows.
    """
    sigma = channel_sigma(seed, xidx, K, block_means)
    x = out if out is not None else np.empty((M, K), dtype=np.uint16)
    for blk in range((M + ROW_BLOCK - 1) // ROW_BLOCK):
        r0 = blk * ROW_BLOCK
        r1 = min(M, r0 + ROW_BLOCK)
        z = _rng(seed, _TID_X, (xidx << 24) | blk).standard_normal(size=(ROW_BLOCK, K), dtype=np.float32)
        x[r0:r1] = f32_to_bf16_bits(z[: r1 - r0] * sigma[None, :])
    return x


def dense_weight(seed: int, widx: int, N: int, K: int, std: float) -> np.ndarray:
    """Unquantized float32 weights N(0, std^2), the input of a quantization fit."""
    z = _rng(seed, _TID_DENSE_W, widx).standard_normal(size=(N, K), dtype=np.float32)
    return (z * np.float32(std)).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One linear layer y[M][N] = x[M][K] . W[N][K]^T of the synthetic suite."""
    name: str
    M: int
    K: int
    N: int
    seed: int
    widx: int = 0
    xidx: int = 0
    block_means: bool = False
    fitted_rows: int = 0          # leading rows of W that come from an imatrix fit of dense floats
    bits: int = 4                 # code width: 4 (W4 g64) or 8 (W8 g64)
    note: str = ""

    @property
    def flops(self) -> float:
        return 2.0 * self.M * self.K * self.N

    @property
    def weight_bytes(self) -> int:
        return self.N * self.K * self.bits // 8 + 4 * self.N * (self.K // GROUP)

    def x(self, M: int | None = None) -> np.ndarray:
        return activations(self.seed, self.xidx, self.M if M is None else M, self.K, self.block_means)

    def w(self):
        if self.bits == 8:
            return weights8(self.seed, self.widx, self.N, self.K)
        return weights(self.seed, self.widx, self.N, self.K)

    def w_pair(self):
        """Gate and up weights of a SwiGLU pair, [N][K] each: weight indices widx and widx + 1."""
        return weights(self.seed, self.widx, self.N, self.K), weights(self.seed, self.widx + 1, self.N, self.K)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny", 16, 256, 256, seed=0, note="tiny parity case"),
        Workload("qkv", 4608, 4608, 13824, seed=1,
                 note="DiT attention QKV projection, 1024^2 canvas: 4096 image + 512 text tokens"),
        Workload("mlp_up_gate", 4608, 4608, 36864, seed=2, widx=0, xidx=0, fitted_rows=4608,
                 note="DiT SwiGLU up/gate pair (2 x 18432), first 4608 rows imatrix-fitted"),
        Workload("mlp_down", 4608, 18432, 4608, seed=2, widx=1, xidx=1,
                 note="DiT SwiGLU down projection"),
        Workload("mlp_gate_up_12288", 4608, 4608, 12288, seed=2, widx=2, xidx=0,
                 note="SwiGLU gate and up projections at the pages' intermediate size 12288 (N = I per weight)"),
        Workload("text_proj", 512, 53248, 4608, seed=3, block_means=True,
                 note="llm_cond_proj 53248->4608; M swept over 1, 8, 32, 512 (leading rows)"),
        Workload("text_proj_w8", 512, 53248, 4608, seed=3, widx=1, block_means=True, bits=8,
                 note="llm_cond_proj 53248->4608 at 8 bits; M swept over 1, 8, 32, 512 (leading rows)"),
        Workload("canvas2048_n4608", 33792, 4608, 4608, seed=4, widx=0,
                 note="2048^2 canvas, two packed samples"),
        Workload("canvas2048_n13824", 33792, 4608, 13824, seed=4, widx=1,
                 note="2048^2 canvas, two packed samples, QKV width"),
    ]
}

TEXT_PROJ_M = (1, 8, 32, 512)


def digest(*arrays: np.ndarray) -> str:
    """Short content hash of generated arrays (reproducibility record)."""
    h = hashlib.sha256()
    for a in arrays:
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()[:16]
