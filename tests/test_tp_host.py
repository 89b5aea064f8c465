"""Tensor-parallel sharding on the host (no GPU): shard bookkeeping, and that the shards of a packed
weight are packed weights whose layers add up (row-parallel) or concatenate (column-parallel) to the
whole layer, checked with the oracle."""
import numpy as np
import pytest
import torch

from group_wise_affine_qlinear_b200 import tp
from oracle import qlinear_oracle as O

from ._helpers import random_layer, random_layer8


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a))


def _np(shard):
    c, s, b = shard
    return c.numpy().view(np.uint32), s.numpy(), b.numpy()


def test_column_ranges():
    assert tp.column_ranges(13824, 0, 2, parts=3) == [(0, 2304), (4608, 6912), (9216, 11520)]
    assert tp.column_ranges(13824, 1, 2, parts=3) == [(2304, 4608), (6912, 9216), (11520, 13824)]
    assert tp.column_ranges(256, 1, 2) == [(128, 256)]
    with pytest.raises(ValueError):
        tp.column_ranges(264, 0, 2, parts=2)     # 132 rows per block: not 2 shards of a multiple of 8
    with pytest.raises(ValueError):
        tp.column_ranges(100, 0, 1, parts=3)


def test_row_range_needs_whole_groups():
    assert tp.row_range(4608, 1, 2) == (2304, 4608)
    assert tp.row_range(4608, 3, 4) == (3456, 4608)
    with pytest.raises(ValueError):
        tp.row_range(192, 0, 2)                  # 96 inputs per shard: a group would straddle the boundary


@pytest.mark.parametrize("bits", [4, 8])
def test_row_shards_are_column_slices_of_the_weight(bits):
    rng = np.random.default_rng(70 + bits)
    x, codes, s, b = (random_layer if bits == 4 else random_layer8)(rng, 3, 512, 24)
    deq = O.dequant_exact if bits == 4 else O.dequant8_exact
    full = deq(codes, s, b)
    for r in range(4):
        sh = _np(tp.row_shard(_t(codes.view(np.int32)), _t(s), _t(b), r, 4, bits=bits))
        k0, k1 = tp.row_range(512, r, 4)
        assert np.array_equal(deq(*sh), full[:, k0:k1])


def test_column_shards_are_rows_of_the_weight():
    rng = np.random.default_rng(72)
    _, codes, s, b = random_layer(rng, 1, 256, 48)
    full = O.dequant_exact(codes, s, b)
    for r in range(2):
        sh = _np(tp.column_shard(_t(codes.view(np.int32)), _t(s), _t(b), r, 2, parts=3))
        rows = np.concatenate([np.arange(a, c) for a, c in tp.column_ranges(48, r, 2, parts=3)])
        assert np.array_equal(O.dequant_exact(*sh), full[rows])


@pytest.mark.parametrize("bits", [4, 8])
def test_row_parallel_partials_add_up_to_the_layer(bits):
    """sum_r x[:, K_r] . W[:, K_r]^T = x . W^T: the K split at group boundaries loses nothing (float64)."""
    rng = np.random.default_rng(73 + bits)
    x, codes, s, b = (random_layer if bits == 4 else random_layer8)(rng, 5, 1024, 40)
    fwd = O.forward_ref if bits == 4 else O.forward8_ref
    y = fwd(x, codes, s, b)
    tot = np.zeros_like(y)
    for r in range(2):
        sh = _np(tp.row_shard(_t(codes.view(np.int32)), _t(s), _t(b), r, 2, bits=bits))
        xr = tp.input_shard(_t(x.view(np.int16)), r, 2).numpy().view(np.uint16)
        tot += fwd(xr, *sh)
    scale = np.abs(O.decode_bf16(x)) @ np.abs((O.dequant_f32 if bits == 4 else O.dequant8_f32)(codes, s, b)).T
    assert np.all(np.abs(tot - y) <= 1e-12 * scale + 1e-300)
