"""The allocation-free forward, qlinear_forward_noalloc, called through the C ABI.

Some callers cannot allocate device memory at the point where they run the
layer: an engine plugin confined to another runtime's fixed memory pool, a
serving loop that is not allowed to allocate once it has started, or a host
that hands the layer only its inputs and outputs and no workspace.  This entry
point serves them by taking its split-K scratch from a fixed array compiled
into the library.

Its output is checked three ways on two calls in a row: bit for bit against
the workspace entry point's CUDA-core path (same arithmetic, same split), within
the layer's tolerance against the default entry point, and within the same
tolerance against the CPU oracle.  The file sorts last so that a run stopping
at its first failure has run every other test first; it also passes alone in
a fresh process, where its first call performs the per-device look-up of the
array's address.
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


# (M, K, N): split 2 and 4 along K (scratch array used), the maximum M = 64 (split 4), and a shape the
# split rule leaves whole (the kernel writes y directly)
SHAPES = [(8, 8192, 1024), (32, 16384, 1024), (64, 16384, 512), (4, 512, 8192)]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_noalloc_matches_existing_entry_and_oracle_two_calls_in_a_row(M, K, N):
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required")
    L = ql.lib()
    rng = np.random.default_rng(2024 + M)
    x, codes, s, b = random_layer(rng, M, K, N)
    xd, cd, sd, bd = to_dev_bf16(x), to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)
    y_ref = O.forward_ref(x, codes, s, b)
    y_gemv = bf16_bits(ql.forward(xd, cd, sd, bd, path=ql.PATH_GEMV))       # workspace entry, same path
    split = ql.last_dispatch()
    y_auto = O.decode_bf16(bf16_bits(ql.forward(xd, cd, sd, bd)))            # default entry point
    assert (M, K, N) != SHAPES[-1] or "splitk=1 " in split
    assert (M, K, N) == SHAPES[-1] or "splitk=1 " not in split
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(L, xd, cd, sd, bd, y, M, K, N) == 0, f"call {call}"
        got_bits = bf16_bits(y)
        assert np.array_equal(got_bits, y_gemv), f"call {call}: differs from the workspace entry's bytes"
        got = O.decode_bf16(got_bits)
        t = O.tolerance(got, y_ref)
        assert t["ok"], (call, t)
        t = O.tolerance(got, y_auto)
        assert t["ok"], (call, t)
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
