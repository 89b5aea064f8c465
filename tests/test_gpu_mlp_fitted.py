"""The MLP up/gate projection with importance-fitted rows, as the 1024^2 SwiGLU workload defines it.

M = 4608 tokens, K = 4608, N = 2 x 18432.  Rows 0..4607 of the weight are dense N(0, 0.02^2) floats
packed by the importance-weighted fit, the importance being E[x^2] of this workload's own activations
(aimarketly "Ideogram-4-IQ4_M", "What IQ4 means here": every quantized weight is fitted with E[x^2]
statistics); the other rows follow the synthetic recipe.  So the forward path meets fitted groups,
whose scales and biases come from least squares rather than from the synthetic draw.

The oracle packs the fitted rows (over worker processes), the device fit packs the same rows and must
give the same bytes, and the forward pass through the dispatcher is checked on sampled rows.
"""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import synthetic as S
from oracle import qlinear_oracle as O

from ._helpers import FUSED_TILE_TOKENS, bf16_bits, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16
from ._oracle_pool import pack_imatrix_parallel

pytestmark = pytest.mark.gpu


def test_mlp_up_gate_with_fitted_rows():
    w = S.WORKLOADS["mlp_up_gate"]
    R = w.fitted_rows
    assert R == 4608 and w.N == 36864
    x = w.x()
    imp32 = O.imatrix_from_x(x).astype(np.float32)              # E[x^2] of this workload's activations
    dense = S.dense_weight(w.seed, w.widx, R, w.K, 0.02)
    rc, rs, rb = pack_imatrix_parallel(dense, imp32.astype(np.float64))      # the oracle's fit
    dc, ds, db = ql.pack(torch.from_numpy(dense).cuda(), imatrix=torch.from_numpy(imp32).cuda())
    assert ql.device_status() == 0
    assert np.array_equal(dc.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(ds.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(db.cpu().numpy().view(np.uint16), rb.view(np.uint16))
    # the pages' guarantee on this weight: never worse than RTN on the weighted objective, group by group
    imp = imp32.astype(np.float64)
    imp = imp + 1e-6 * imp.mean()
    e_fit = O.group_weighted_error(dense, rc, rs, rb, imp)
    e_rtn = O.group_weighted_error(dense, *O.pack_rtn(dense), imp)
    assert np.all(e_fit <= e_rtn * (1 + 1e-12)) and e_fit.sum() < e_rtn.sum()

    codes, s, b = w.w()
    codes, s, b = codes.copy(), s.copy(), b.copy()
    codes[:R], s[:R], b[:R] = rc, rs, rb
    y = ql.forward(to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b))
    assert ql.last_dispatch().startswith("path=tc_fused")
    rows = sample_rows(w.M, n_random=48, seed=2, tile=FUSED_TILE_TOKENS)
    y_ref = O.forward_rows(x, codes, s, b, rows)
    got = O.decode_bf16(bf16_bits(y)[rows])
    t = O.tolerance(got, y_ref)
    assert t["ok"], t
    # the fitted columns (output features 0..4607) on their own, whose weights are the fitted groups
    t = O.tolerance(got[:, :R], y_ref[:, :R])
    assert t["ok"], t
    assert ql.device_status() == 0
