"""Race detection for the tensor-core pipelines by shaking their timing (checked build).

qlinear_test_delay holds back one role of the kernels (activation producer, code producer, dequantizers,
MMA issuers, epilogue/drain warps), or all of them, at its start by a different time in every CTA and warp,
so that each hand-off between roles (TMA rings, tensor-memory stages, the accumulators, split-K partials,
stream-K segments) meets other orders of arrival.  Every result must be the same bytes as the undelayed
call's, and within the oracle's tolerance.  Shapes give CTAs several units: the fused path with several
tiles per CTA and with split-K units, and the weight-streaming path with two tile segments per CTA.
"""
import ctypes

import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from oracle import qlinear_oracle as O

from ._helpers import FUSED_TILE_TOKENS, bf16_bits, random_layer, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16

pytestmark = pytest.mark.gpu

ROLES = [1, 2, 4, 8, 16, 31]          # activations, codes, dequantizers, MMA, epilogue, all of them
CASES = [  # (M, K, N, path, split)
    (1152, 2048, 9216, ql.PATH_TC_FUSED, 1),     # 6 x 36 = 216 tiles on 148 CTAs
    (256, 8192, 2048, ql.PATH_TC_FUSED, 4),      # 16 tiles x 4 K slices
    (24, 16384, 4608, ql.PATH_TC_SKINNY, 0),     # stream-K runs over two tile segments
]


def _checked_library():
    from group_wise_affine_qlinear_b200 import build as qb
    return ql.load_library(qb.build(bounds_check=True))


@pytest.mark.parametrize("M,K,N,path,split", CASES)
def test_outputs_do_not_depend_on_role_timing(M, K, N, path, split):
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required for -m gpu tests")
    Lc = _checked_library()
    rng = np.random.default_rng(M * 7 + K)
    x, codes, s, b = random_layer(rng, M, K, N)
    xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws_bytes = Lc.qlinear_workspace_size_config(M, K, N, 64, path, split)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        y.fill_(float("nan"))
        assert Lc.qlinear_forward_config(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                                         1, M, K, N, 64, path, split, ws.data_ptr(), ws.numel(), st) == 0
        assert Lc.qlinear_get_device_status(st) == 0
        return bf16_bits(y)

    assert Lc.qlinear_test_delay(0, 0) == 0
    ref = call()
    rows = sample_rows(M, n_random=16, seed=M, tile=FUSED_TILE_TOKENS)
    t = O.tolerance(O.decode_bf16(ref[rows]), O.forward_rows(x, codes, s, b, rows))
    assert t["ok"], t
    try:
        for role in ROLES:
            assert Lc.qlinear_test_delay(role, 20_000) == 0        # up to 20 us per role
            for _ in range(2):
                got = call()
                diff = np.flatnonzero(got != ref)
                assert diff.size == 0, (role, diff.size, diff[:8])
    finally:
        assert Lc.qlinear_test_delay(0, 0) == 0


def test_delay_hook_rejects_bad_arguments():
    Lc = _checked_library()
    assert Lc.qlinear_test_delay(32, 1000) == 1                  # QL_ERR_INVALID_ARG: unknown bit
    assert Lc.qlinear_test_delay(1, 2_000_000) == 1              # above 1 ms
    assert Lc.qlinear_test_delay(0, 0) == 0
