"""GPU parity of the fused SwiGLU up/gate pair (reading R10) against the oracle, within reading R11.

h = silu(x . W_gate^T) * (x . W_up^T) from one call that runs both projections in one tensor-core
GEMM and gates in its epilogue.  Small ragged shapes against the full oracle, one-hot rows that pin
the pairing of gate and up rows to one bf16 ulp, and sampled rows of the pages' MLP width
(K = 4608, I = 12288, M = 4608).

The file sorts after the other GPU parity files, so that a run stopping at its first failure has
already checked every older path.
"""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import synthetic as S
from oracle import qlinear_oracle as O

from ._helpers import FUSED_TILE_TOKENS, bf16_bits, random_layer, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16

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


def _pair(rng, M, K, I):
    x, gc, gs, gb = random_layer(rng, M, K, I)
    _, uc, us, ub = random_layer(rng, 1, K, I)
    return x, (gc, gs, gb), (uc, us, ub)


def _check(h_dev, x, gate, up, rows=None, bf16=True):
    g, u = O.swiglu_linears(x, gate, up, rows)
    h = h_dev if rows is None else h_dev[torch.from_numpy(rows).to(h_dev.device)]
    hv = O.decode_bf16(bf16_bits(h)) if bf16 else h.double().cpu().numpy()
    t = O.swiglu_tolerance(hv, g, u, bf16_output=bf16)
    assert t["ok"], t
    return t


@pytest.mark.parametrize("K,I", [(64, 8), (320, 136), (1024, 264), (2048, 520)])
def test_swiglu_ragged(K, I):
    rng = np.random.default_rng(K + I)
    for M in (1, 7, 33, 191, 193, 400):
        x, gate, up = _pair(rng, M, K, I)
        h = ql.swiglu(to_dev_bf16(x), _dev(*gate), _dev(*up))
        _check(h, x, gate, up)
    assert ql.last_dispatch().startswith("path=tc_fused_swiglu")


def test_swiglu_fp32_output():
    rng = np.random.default_rng(90)
    x, gate, up = _pair(rng, 200, 1024, 264)
    h = ql.swiglu(to_dev_bf16(x), _dev(*gate), _dev(*up), out_dtype=torch.float32)
    _check(h, x, gate, up, bf16=False)


def test_swiglu_one_hot_pairs_gate_and_up_rows():
    """x = e_k: g = RN_f16(w_g(n, k)) and u = RN_f16(w_u(n, k)) exactly, so h is silu(g) * u computed in
    fp32 and rounded to bf16: within one bf16 unit of the same value formed in float64.  A gate row
    paired with the wrong up row, or a wrong column, would be far off."""
    rng = np.random.default_rng(91)
    K, I = 320, 264
    _, gate, up = _pair(rng, 1, K, I)
    ks = np.array([0, 1, 4, 7, 8, 63, 64, 65, 130, 200, 255, 256, 319])
    x = np.zeros((ks.size, K), dtype=np.uint16)
    x[np.arange(ks.size), ks] = 0x3F80
    h = O.decode_bf16(bf16_bits(ql.swiglu(to_dev_bf16(x), _dev(*gate), _dev(*up))))
    g = O.dequant_f16(*gate).astype(np.float64)[:, ks].T
    u = O.dequant_f16(*up).astype(np.float64)[:, ks].T
    ref = O.silu(g) * u
    ulp = 2.0 * O.half_ulp_bf16(np.maximum(np.abs(ref), 1e-30))
    assert np.all(np.abs(h - ref) <= ulp + 1e-30)


def test_swiglu_zero_rows_and_scaled_rows():
    """A zero activation row gives h = 0 exactly; rows scaled by powers of two far from 1 meet R11."""
    rng = np.random.default_rng(92)
    K, I = 1024, 264
    _, gate, up = _pair(rng, 1, K, I)
    base = rng.standard_normal((4, K))
    rows = np.stack([base[0], np.zeros(K), base[2] * 2.0 ** -20, base[3] * 2.0 ** 6])
    x = S.f32_to_bf16_bits(rows.astype(np.float32))
    h = ql.swiglu(to_dev_bf16(x), _dev(*gate), _dev(*up))
    hv = O.decode_bf16(bf16_bits(h))
    assert np.all(hv[1] == 0.0)
    for t in (0, 2, 3):
        g, u = O.swiglu_linears(x[t:t + 1], gate, up)
        tol = O.swiglu_tolerance(hv[t:t + 1], g, u)
        assert tol["ok"], (t, tol)


def test_swiglu_deterministic():
    rng = np.random.default_rng(93)
    x, gate, up = _pair(rng, 300, 1024, 520)
    args = (to_dev_bf16(x), _dev(*gate), _dev(*up))
    assert np.array_equal(bf16_bits(ql.swiglu(*args)), bf16_bits(ql.swiglu(*args)))


def test_swiglu_full_mlp_width():
    """The pages' MLP: K = 4608, I = 12288, 4608 tokens; sampled rows (both sides of every fused-tile boundary)."""
    w = S.WORKLOADS["mlp_gate_up_12288"]
    x = w.x()
    gate, up = w.w_pair()
    h = ql.swiglu(to_dev_bf16(x), _dev(*gate), _dev(*up))
    rows = sample_rows(w.M, n_random=24, seed=5, tile=FUSED_TILE_TOKENS)
    _check(h, x, gate, up, rows=rows)
