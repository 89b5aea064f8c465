"""The allocation-free forward, qlinear_forward_noalloc, called through the C ABI.

It serves callers that cannot allocate device memory where they run the layer
(an engine plugin confined to someone else's memory pool, a serving loop that
must not allocate after start-up, a runtime that supplies no workspace): its
split-K scratch is a fixed array inside the library.  The tests pass in any
order, and alone in a fresh process, where the first call performs the
per-device set-up of the array's address.
"""
import ctypes

import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from oracle import qlinear_oracle as O

from ._helpers import bf16_bits, random_layer, to_dev_bf16, to_dev_codes, to_dev_f16

pytestmark = pytest.mark.gpu


def _call_noalloc(L, x, c, s, b, y, M, K, N, group=64):
    st = torch.cuda.current_stream().cuda_stream
    return L.qlinear_forward_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(c.data_ptr()),
                                     ctypes.c_void_p(s.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                     ctypes.c_void_p(y.data_ptr()), M, K, N, group, ctypes.c_void_p(st))


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required")
    L = ql.lib()
    rng = np.random.default_rng(2024)
    # two different shapes, both split along K (so both use the library's scratch array)
    for M, K, N in [(8, 53248, 4608), (32, 16384, 1024)]:
        x, codes, s, b = random_layer(rng, M, K, N)
        xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
        y_ref = ql.forward(xd, cd, sd, bd, path=ql.PATH_GEMV)          # existing entry, caller workspace
        assert "splitk=1 " not in ql.last_dispatch()
        ref = O.decode_bf16(bf16_bits(y_ref))
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(L, xd, cd, sd, bd, y, M, K, N) == 0
        got = O.decode_bf16(bf16_bits(y))
        t = O.tolerance(got, ref)
        assert t["ok"], t
        assert ql.device_status() == 0


def test_noalloc_rejects_out_of_range_sizes():
    L = ql.lib()
    rng = np.random.default_rng(5)
    x, codes, s, b = random_layer(rng, 65, 256, 64)
    xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
    y = torch.empty((65, 64), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(L, xd, cd, sd, bd, y, 65, 256, 64) == 3          # M above QL_NOALLOC_MAX_M
    assert _call_noalloc(L, xd, cd, sd, bd, y, 64, 256, 64, group=32) == 3
    assert _call_noalloc(L, xd, cd, sd, bd, y, 64, 250, 64) == 1
