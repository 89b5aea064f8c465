"""Tensor parallelism for the packed layer: column- and row-parallel shards and their forward passes.

A two-GPU tensor-parallel layout of the Ideogram 4 DiT is a validated configuration on B200
(docs.sglang.io Ideogram4 cookbook, "Tensor and sequence parallelism"). That page replicates its
bitsandbytes NF4 text encoder instead of sharding it, because NF4's quantization state does not split
along the input dimension. A group-wise affine g64 weight does split: each (scale, bias) covers 64
consecutive inputs of one output row. So any range of rows is itself a packed weight, and so is any K
range that starts and ends on a multiple of 64.

Column-parallel (split N). A rank holds a set of rows of W: a row slice of codes, scales and biases,
which is a view for one block and a copy for several (e.g. the Q, K and V blocks of a fused QKV weight).
Its output is its own columns of y, and nothing is exchanged; a following row-parallel layer takes that
slice as its K shard.

Row-parallel (split K). Rank r of W holds the K range [r K/W, (r+1) K/W) of every row, a multiple of
64, and the matching columns of x. Each rank computes an fp32 partial of the whole y. The partials are
gathered in rank order over the process group (NCCL on GPUs), and qlinear_reduce_partials sums them in
that order and rounds once. Every rank therefore holds the same bytes, and the result differs from a
single-GPU fp32 accumulation only in where the additions fall.

Weights are sharded once, at load time (torch slicing). Every arithmetic step of a forward pass runs in
the library's kernels; the collective only moves bytes.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib as L

GROUP = 64


def column_ranges(N: int, rank: int, world: int, parts: int = 1) -> list[tuple[int, int]]:
    """Rows [start, stop) of W [N][K] held by `rank`: N is `parts` equal blocks, each split evenly."""
    if parts < 1 or N % parts:
        raise ValueError(f"N = {N} is not {parts} equal blocks")
    blk = N // parts
    if blk % world or (blk // world) % 8:
        raise ValueError(f"a block of {blk} rows does not split into {world} shards of a multiple of 8 rows")
    per = blk // world
    return [(p * blk + rank * per, p * blk + (rank + 1) * per) for p in range(parts)]


def row_range(K: int, rank: int, world: int) -> tuple[int, int]:
    """Inputs [k0, k1) of the row-parallel shard of `rank`: whole 64-groups only."""
    if K % (world * GROUP):
        raise ValueError(f"K = {K} does not split into {world} shards of whole {GROUP}-groups")
    per = K // world
    return rank * per, (rank + 1) * per


def column_shard(codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, rank: int, world: int,
                 parts: int = 1):
    """(codes, scales, biases) of the rows `rank` holds in a column-parallel layout."""
    rngs = column_ranges(codes.shape[0], rank, world, parts)

    def take(t):
        if len(rngs) == 1:
            return t[rngs[0][0]:rngs[0][1]]
        return torch.cat([t[a:b] for a, b in rngs]).contiguous()

    return take(codes), take(scales), take(biases)


def row_shard(codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, rank: int, world: int,
              bits: int = 4):
    """(codes, scales, biases) of the K range `rank` holds in a row-parallel layout (contiguous copies)."""
    K = codes.shape[1] * (32 // bits)
    k0, k1 = row_range(K, rank, world)
    w0, w1 = k0 * bits // 32, k1 * bits // 32
    g0, g1 = k0 // GROUP, k1 // GROUP
    return codes[:, w0:w1].contiguous(), scales[:, g0:g1].contiguous(), biases[:, g0:g1].contiguous()


def input_shard(x: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """Columns of x [M][K] that meet the row-parallel shard of `rank`."""
    k0, k1 = row_range(x.shape[1], rank, world)
    return x[:, k0:k1].contiguous()


def _world(group) -> int:
    if not dist.is_available() or not dist.is_initialized():
        return 1
    return dist.get_world_size(group)


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's partial [M][N], stacked in rank order: [world][M][N] (one all-gather)."""
    world = _world(group)
    if world == 1:
        return partial.unsqueeze(0)
    out = torch.empty((world * partial.shape[0], *partial.shape[1:]), dtype=partial.dtype, device=partial.device)
    dist.all_gather_into_tensor(out, partial.contiguous(), group=group)
    return out.view(world, *partial.shape)


def column_parallel_forward(x: torch.Tensor, shard, bits: int = 4, **kw) -> torch.Tensor:
    """This rank's columns of y = x . W^T (no exchange)."""
    fwd = L.forward if bits == 4 else L.forward8
    return fwd(x, *shard, **kw)


def row_parallel_forward(x_shard: torch.Tensor, shard, bits: int = 4, group=None, out: torch.Tensor | None = None,
                         out_dtype=torch.bfloat16) -> torch.Tensor:
    """y = x . W^T from this rank's K shard: fp32 partial, all-gather in rank order, ordered sum, one rounding."""
    fwd = L.forward if bits == 4 else L.forward8
    partial = fwd(x_shard, *shard, out_dtype=torch.float32)
    return L.reduce_partials(gather_partials(partial, group), out=out, out_dtype=out_dtype)
