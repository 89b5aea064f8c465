"""GPU parity of the fused tensor-core path with its K-steps split (qlinear_forward_config with
QL_PATH_TC_FUSED and split_k > 1): every slice of every tile is its own work unit, writes an fp32
partial, and the partials are summed in slice order and rounded once.  Against the oracle within
reading R5, for 4- and 8-bit codes, and on sampled rows of the text projection at M = 512, the shape
with fewer tiles than SMs that the split is for.

The file sorts after the paths already validated on a B200, so a run stopping at its first failure
has checked those first.
"""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import synthetic as S
from oracle import qlinear_oracle as O

from ._helpers import FUSED_TILE_TOKENS, bf16_bits, random_layer, random_layer8, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16

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


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("split", [2, 3, 7])
@pytest.mark.parametrize("K,N", [(448, 264), (1024, 520)])
def test_fused_split_k(bits, split, K, N):
    rng = np.random.default_rng(bits * 100 + split * 10 + K + N)
    fwd = ql.forward if bits == 4 else ql.forward8
    ref_fn = O.forward_ref if bits == 4 else O.forward8_ref
    for M in (1, 100, 193, 400):
        x, codes, s, b = (random_layer if bits == 4 else random_layer8)(rng, M, K, N)
        for dt in (torch.bfloat16, torch.float32):
            y = fwd(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_FUSED, split_k=split, out_dtype=dt)
            got = O.decode_bf16(bf16_bits(y)) if dt == torch.bfloat16 else y.double().cpu().numpy()
            t = O.tolerance(got, ref_fn(x, codes, s, b), bf16_output=(dt == torch.bfloat16))
            assert t["ok"], (M, dt, t)
    assert f"splitk={split}" in ql.last_dispatch()


def test_fused_split_k_one_group_per_slice_and_determinism():
    rng = np.random.default_rng(101)
    x, codes, s, b = random_layer(rng, 250, 640, 264)            # 10 groups, 10 slices
    args = (to_dev_bf16(x), *_dev(codes, s, b))
    y = ql.forward(*args, path=ql.PATH_TC_FUSED, split_k=10)
    t = O.tolerance(O.decode_bf16(bf16_bits(y)), O.forward_ref(x, codes, s, b))
    assert t["ok"], t
    assert np.array_equal(bf16_bits(y), bf16_bits(ql.forward(*args, path=ql.PATH_TC_FUSED, split_k=10)))


def test_fused_split_k_text_proj_m512():
    """llm_cond_proj at M = 512: 54 output tiles, split 8 ways into 432 units on 148 SMs."""
    w = S.WORKLOADS["text_proj"]
    x = w.x(512)
    codes, s, b = w.w()
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_FUSED, split_k=8)
    rows = sample_rows(512, n_random=32, seed=512, tile=FUSED_TILE_TOKENS)
    t = O.tolerance(O.decode_bf16(bf16_bits(y)[rows]), O.forward_rows(x, codes, s, b, rows))
    assert t["ok"], t
