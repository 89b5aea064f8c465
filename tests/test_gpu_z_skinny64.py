"""GPU parity of the weight-streaming tensor-core path at 64 tokens (NT = 64: MMA N = 64, for
32 < M <= 64, reached through qlinear_forward_config with QL_PATH_TC_SKINNY), for 4- and 8-bit codes.
Within reading R5 at stream-K shapes and on sampled rows of the text projection at M = 64; one-hot
rows bit-exact (RN_bf16 of the f16 weight operand).

The file sorts after the paths already validated on a B200, so a run stopping at its first failure
has checked those first.
"""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import synthetic as S
from oracle import qlinear_oracle as O

from ._helpers import bf16_bits, random_layer, random_layer8, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16

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
@pytest.mark.parametrize("M", [33, 48, 64])
@pytest.mark.parametrize("K,N", [(64, 8), (4096, 264), (8192, 1032), (4160, 200)])
def test_skinny64_shapes(bits, M, K, N):
    rng = np.random.default_rng(bits * 1000 + M * 7 + K + N)
    x, codes, s, b = (random_layer if bits == 4 else random_layer8)(rng, M, K, N)
    fwd = ql.forward if bits == 4 else ql.forward8
    for dt in (torch.bfloat16, torch.float32):
        y = fwd(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_SKINNY, out_dtype=dt)
        got = O.decode_bf16(bf16_bits(y)) if dt == torch.bfloat16 else y.double().cpu().numpy()
        ref = (O.forward_ref if bits == 4 else O.forward8_ref)(x, codes, s, b)
        t = O.tolerance(got, ref, bf16_output=(dt == torch.bfloat16))
        assert t["ok"], (dt, t)
    assert "nt=64" in ql.last_dispatch()


@pytest.mark.parametrize("bits", [4, 8])
def test_skinny64_one_hot_bitexact(bits):
    rng = np.random.default_rng(102 + bits)
    K, N = 320, 264
    _, codes, s, b = (random_layer if bits == 4 else random_layer8)(rng, 1, K, N)
    ks = np.array(list(range(0, 320, 5)))[:64]
    x = np.zeros((ks.size, K), dtype=np.uint16)
    x[np.arange(ks.size), ks] = 0x3F80
    fwd = ql.forward if bits == 4 else ql.forward8
    y = fwd(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_SKINNY)
    deq16 = (O.dequant_f16 if bits == 4 else O.dequant8_f16)(codes, s, b)
    assert np.array_equal(bf16_bits(y), O.round_bf16(deq16.astype(np.float64))[:, ks].T)


def test_skinny64_text_proj():
    w = S.WORKLOADS["text_proj"]
    x = w.x(64)
    codes, s, b = w.w()
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_SKINNY)
    rows = sample_rows(64, n_random=16, seed=64, tile=16)
    t = O.tolerance(O.decode_bf16(bf16_bits(y)[rows]), O.forward_rows(x, codes, s, b, rows))
    assert t["ok"], t
