"""Ring-depth stress of the fused tensor-core kernel (4-bit codes, bf16 output).

The checked build (libqlinear_bounds.so) can launch the kernel with other ring depths through
qlinear_test_ring_depth: 2 to 6 activation stages, 1 to 3 code stages (each 4 K-steps), one or two
epilogue staging blocks per warp.  Every ring position is a function of the step count alone and the
MMAs accumulate in the same K order, so every variant must write the same bytes; the shipped
configuration's output must also match the oracle.  The shapes give CTAs more than one tile, K-step
counts that leave a partial last code stage (K = 448: 4 + 3 steps), and ragged edges in M and N.
"""
import ctypes

import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from oracle import qlinear_oracle as O

from ._helpers import FUSED_TILE_TOKENS, bf16_bits, random_layer, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16

pytestmark = pytest.mark.gpu

VARIANTS = 7                  # QL_TEST_RING_VARIANTS
SHAPES = [(400, 1024, 15256), (200, 448, 4000), (192, 4608, 512), (77, 320, 1000)]


def _checked_library():
    from group_wise_affine_qlinear_b200 import build as qb
    return ql.load_library(qb.build(bounds_check=True))


def _last_dispatch(L) -> str:
    buf = ctypes.create_string_buffer(256)
    assert L.qlinear_last_dispatch(buf, 256) == 0
    return buf.value.decode()


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_every_ring_depth_writes_the_same_bytes(M, K, N):
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required for -m gpu tests")
    Lc = _checked_library()
    rng = np.random.default_rng(M + K + N)
    x, codes, s, b = random_layer(rng, M, K, N)
    xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws_bytes = Lc.qlinear_workspace_size_config(M, K, N, 64, ql.PATH_TC_FUSED, 1)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    try:
        for v in range(VARIANTS):
            assert Lc.qlinear_test_ring_depth(v) == 0
            y.fill_(float("nan"))
            assert Lc.qlinear_forward_config(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                                             1, M, K, N, 64, ql.PATH_TC_FUSED, 1, ws.data_ptr(), ws.numel(), st) == 0
            assert Lc.qlinear_get_device_status(st) == 0
            d = _last_dispatch(Lc)
            assert d.startswith("path=tc_fused "), d
            assert (f"ring_variant={v} " in d) == (v > 0), d
            outs.append(bf16_bits(y))
    finally:
        assert Lc.qlinear_test_ring_depth(0) == 0
    for v in range(1, VARIANTS):
        diff = np.flatnonzero(outs[v] != outs[0])
        assert diff.size == 0, (v, diff[:8])
    rows = sample_rows(M, n_random=24, seed=M, tile=FUSED_TILE_TOKENS)
    t = O.tolerance(O.decode_bf16(outs[0][rows]), O.forward_rows(x, codes, s, b, rows))
    assert t["ok"], t


def test_ring_depth_hook_rejects_unknown_variants():
    Lc = _checked_library()
    assert Lc.qlinear_test_ring_depth(-1) == 1          # QL_ERR_INVALID_ARG
    assert Lc.qlinear_test_ring_depth(VARIANTS) == 1
    from group_wise_affine_qlinear_b200 import build as qb
    shipped = ql.load_library(qb.build())               # by path: QL_LIBRARY may select the checked build
    assert shipped.qlinear_test_ring_depth(1) == 3      # the shipped library: QL_ERR_UNSUPPORTED
