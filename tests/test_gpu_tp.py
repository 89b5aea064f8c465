"""Tensor-parallel layouts on one GPU: both ranks' shards run one after the other (no rank waits on
another), and the combination step runs in qlinear_reduce_partials.  Row-parallel y and column-parallel
slices against the oracle (reading R5); the ordered reduction bit-exact against numpy's float32 sums."""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import tp
from oracle import qlinear_oracle as O

from ._helpers import bf16_bits, random_layer, random_layer8, to_dev_bf16, to_dev_codes, to_dev_f16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required for -m gpu tests")
    ql.lib()
    yield
    assert ql.device_status() == 0


def _dev(codes, s, b):
    return to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)


def test_reduce_partials_bitexact():
    rng = np.random.default_rng(95)
    p = (rng.standard_normal((3, 40, 264)) * np.exp(rng.uniform(-8, 8, (3, 40, 264)))).astype(np.float32)
    ref32 = (p[0] + p[1]) + p[2]                        # float32, in partial order
    pd = torch.from_numpy(p).cuda()
    y32 = ql.reduce_partials(pd, out_dtype=torch.float32)
    assert np.array_equal(y32.cpu().numpy().view(np.uint32), ref32.view(np.uint32))
    y16 = ql.reduce_partials(pd)
    assert np.array_equal(bf16_bits(y16), O.round_bf16(ref32.astype(np.float64)))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M", [8, 300])
def test_row_parallel_two_ranks(bits, M):
    rng = np.random.default_rng(96 + bits + M)
    x, codes, s, b = (random_layer if bits == 4 else random_layer8)(rng, M, 1024, 264)
    xd, full = to_dev_bf16(x), _dev(codes, s, b)
    fwd = ql.forward if bits == 4 else ql.forward8
    parts = [fwd(tp.input_shard(xd, r, 2), *tp.row_shard(*full, r, 2, bits=bits), out_dtype=torch.float32)
             for r in range(2)]
    y = ql.reduce_partials(torch.stack(parts))
    ref = (O.forward_ref if bits == 4 else O.forward8_ref)(x, codes, s, b)
    t = O.tolerance(O.decode_bf16(bf16_bits(y)), ref)
    assert t["ok"], t
    # one rank, no process group: the same call path with a single partial
    y1 = tp.row_parallel_forward(xd, full, bits=bits)
    assert O.tolerance(O.decode_bf16(bf16_bits(y1)), ref)["ok"]


def test_column_parallel_fused_qkv_two_ranks():
    """Q, K and V blocks each split between two ranks: every rank's output columns are the oracle's."""
    rng = np.random.default_rng(98)
    x, codes, s, b = random_layer(rng, 200, 512, 3 * 256)
    xd, full = to_dev_bf16(x), _dev(codes, s, b)
    ref = O.forward_ref(x, codes, s, b)
    for r in range(2):
        y = tp.column_parallel_forward(xd, tp.column_shard(*full, r, 2, parts=3))
        cols = np.concatenate([np.arange(a, c) for a, c in tp.column_ranges(768, r, 2, parts=3)])
        t = O.tolerance(O.decode_bf16(bf16_bits(y)), ref[:, cols])
        assert t["ok"], (r, t)
