"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, and rejects bad arguments before any
launch."""
import ctypes
import os
import re

import pytest

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import build as qb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    qb.build()
    return ql.lib()


def _declared():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            txt = open(os.path.join(inc, f)).read()
            names += re.findall(r"QL_API\s+[\w\s\*]+?\b(qlinear8?_\w+)\s*\(", txt)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = _declared()
    for n in ("qlinear_forward", "qlinear_dequant", "qlinear_pack", "qlinear_workspace_size",
              "qlinear8_forward", "qlinear8_forward_config", "qlinear8_dequant", "qlinear8_pack",
              "qlinear8_workspace_size", "qlinear8_workspace_size_config"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in _declared():
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert ql.version() == 100
    for code, name in ql.STATUS.items():
        assert L.qlinear_status_string(code).decode() == name
    assert L.qlinear_status_string(99).decode() == "QL_ERR_UNKNOWN"


def test_last_dispatch_buffer_checks(L):
    assert L.qlinear_last_dispatch(None, 10) == 1
    buf = ctypes.create_string_buffer(4)
    assert L.qlinear_last_dispatch(buf, 4) == 0
    assert len(buf.value) <= 3


FAKE = 0x10000000          # never dereferenced: validation rejects before any launch


def _fwd(L, x=FAKE, c=FAKE + (1 << 24), s=FAKE + (2 << 24), b=FAKE + (3 << 24), y=FAKE + (4 << 24),
         M=16, K=256, N=256, group=64):
    return L.qlinear_forward(x, c, s, b, y, M, K, N, group, None, 0, None)


def test_forward_rejects_bad_shapes(L):
    assert _fwd(L, group=32) == 3
    assert _fwd(L, group=128) == 3
    assert _fwd(L, K=100) == 1
    assert _fwd(L, K=0) == 1
    assert _fwd(L, N=12) == 1
    assert _fwd(L, M=0) == 1
    assert _fwd(L, M=-3) == 1


def test_forward_rejects_null_and_misaligned(L):
    assert _fwd(L, x=0) == 1
    assert _fwd(L, y=0) == 1
    assert _fwd(L, c=FAKE + (1 << 24) + 4) == 2
    assert _fwd(L, x=FAKE + 2) == 2


def test_forward_rejects_output_aliasing(L):
    assert _fwd(L, y=FAKE) == 1                     # y over x
    assert _fwd(L, y=FAKE + (1 << 24) + 64) == 1    # y inside codes


def test_forward_config_rejects_bad_path(L):
    r = L.qlinear_forward_config(FAKE, FAKE + (1 << 24), FAKE + (2 << 24), FAKE + (3 << 24), FAKE + (4 << 24),
                                 1, 16, 256, 256, 64, 9, 0, None, 0, None)
    assert r == 1


def test_dequant_and_pack_validation(L):
    assert L.qlinear_dequant(FAKE, FAKE + (1 << 24), FAKE + (2 << 24), 256, 256, 32, FAKE + (3 << 24), 0, None) == 3
    assert L.qlinear_dequant(FAKE, FAKE + (1 << 24), FAKE + (2 << 24), 256, 256, 64, FAKE, 0, None) == 1
    assert L.qlinear_dequant(FAKE + 8, FAKE + (1 << 24), FAKE + (2 << 24), 256, 256, 64, FAKE + (3 << 24), 0, None) == 2
    # an importance vector overlapping an output is rejected before any launch
    assert L.qlinear_pack(FAKE, FAKE + (1 << 24), 256, 256, 64, FAKE + (1 << 24), FAKE + (2 << 24), FAKE + (3 << 24), None) == 1
    assert L.qlinear_pack(FAKE, None, 256, 256, 64, FAKE, FAKE + (2 << 24), FAKE + (3 << 24), None) == 1


def test_workspace_size_values(L):
    # fused path: f16 activations + row scales + transposed (scale, bias) pairs, 256-byte aligned pieces
    M, K, N = 4608, 4608, 13824
    ws = ql.workspace_size(M, K, N, ql.PATH_TC_FUSED)
    assert ws == M * K * 2 + M * 4 + (K // 64) * N * 4
    assert ql.workspace_size(1, 4096, 64, ql.PATH_GEMV, 1) == 0
    assert ql.workspace_size(2, 4096, 64, ql.PATH_GEMV, 4) == 4 * 2 * 64 * 4
    assert L.qlinear_workspace_size(16, 100, 256, 64) == ctypes.c_size_t(-1).value


# The dispatcher's choice, read through the workspace it asks for (the library assumes a B200's 148
# SMs when no GPU is present).  Expected choices are the fastest forced configurations measured on a
# B200 for these shapes (or within 5% of it): the weight-streaming kernel up to 64 tokens, then the
# fused kernel split so that ceil(tiles * S / SMs) waves of ceil(G / S) K-steps are fewest.
DISPATCH_TABLE = [
    # (M, K, N, path, split) -- text projection 53248 -> 4608, QKV 4608 -> 13824, MLP down 18432 -> 4608
    (1, 53248, 4608, ql.PATH_TC_SKINNY, 0), (32, 53248, 4608, ql.PATH_TC_SKINNY, 0),
    (33, 53248, 4608, ql.PATH_TC_SKINNY, 0), (64, 53248, 4608, ql.PATH_TC_SKINNY, 0),
    (65, 53248, 4608, ql.PATH_TC_FUSED, 8), (128, 53248, 4608, ql.PATH_TC_FUSED, 8),
    (192, 53248, 4608, ql.PATH_TC_FUSED, 8), (256, 53248, 4608, ql.PATH_TC_FUSED, 4),
    (384, 53248, 4608, ql.PATH_TC_FUSED, 4), (512, 53248, 4608, ql.PATH_TC_FUSED, 5),
    (128, 4608, 13824, ql.PATH_TC_FUSED, 2), (256, 4608, 13824, ql.PATH_TC_FUSED, 1),
    (512, 4608, 13824, ql.PATH_TC_FUSED, 1), (1024, 4608, 13824, ql.PATH_TC_FUSED, 1),
    (4608, 4608, 13824, ql.PATH_TC_FUSED, 1),
    (128, 18432, 4608, ql.PATH_TC_FUSED, 8), (512, 18432, 4608, ql.PATH_TC_FUSED, 5),
    (4608, 18432, 4608, ql.PATH_TC_FUSED, 1),
]


@pytest.mark.parametrize("M,K,N,path,split", DISPATCH_TABLE)
def test_dispatcher_table(L, M, K, N, path, split):
    auto = ql.workspace_size(M, K, N)
    assert auto == ql.workspace_size(M, K, N, path, split)
    if path == ql.PATH_TC_FUSED:
        for other in (1, 2, 4, 8, 12, 16):
            if other != split:
                assert ql.workspace_size(M, K, N, path, other) != auto


def test_profile_events_pairing(L):
    assert L.qlinear_set_profile_events(FAKE, None) == 1
    assert L.qlinear_set_profile_events(None, None) == 0


# ---------------------------------------------------------------- 8-bit codes (codes [N][K/4])

def _fwd8(L, x=FAKE, c=FAKE + (1 << 24), s=FAKE + (2 << 24), b=FAKE + (3 << 24), y=FAKE + (4 << 24),
          M=16, K=256, N=256, group=64):
    return L.qlinear8_forward(x, c, s, b, y, M, K, N, group, None, 0, None)


def test_forward8_rejects_bad_arguments(L):
    assert _fwd8(L, group=32) == 3
    assert _fwd8(L, K=100) == 1
    assert _fwd8(L, N=12) == 1
    assert _fwd8(L, M=0) == 1
    assert _fwd8(L, x=0) == 1
    assert _fwd8(L, c=FAKE + (1 << 24) + 4) == 2
    assert _fwd8(L, y=FAKE) == 1


def test_forward8_counts_one_byte_per_code(L):
    # 256 x 256 8-bit codes span 64 KiB: a y starting 40000 bytes in lies inside them (it would not
    # for 4-bit codes, which span 32 KiB)
    assert _fwd8(L, y=FAKE + (1 << 24) + 40000) == 1
    assert L.qlinear8_dequant(FAKE, FAKE + (1 << 24), FAKE + (2 << 24), 256, 256, 64, FAKE + 40000, 0, None) == 1


def test_pack8_validation(L):
    # the importance-weighted fit is built for 4-bit codes only
    assert L.qlinear8_pack(FAKE, FAKE + (4 << 24), 256, 256, 64, FAKE + (1 << 24), FAKE + (2 << 24),
                           FAKE + (3 << 24), None) == 3
    assert L.qlinear8_pack(FAKE, None, 256, 256, 32, FAKE + (1 << 24), FAKE + (2 << 24), FAKE + (3 << 24), None) == 3
    # codes (64 KiB) running into the scales
    assert L.qlinear8_pack(FAKE, None, 256, 256, 64, FAKE + (1 << 24), FAKE + (1 << 24) + 40000, FAKE + (3 << 24),
                           None) == 1


def test_workspace_size8_values(L):
    M, K, N = 4608, 4608, 13824
    assert ql.workspace_size8(M, K, N, ql.PATH_TC_FUSED) == M * K * 2 + M * 4 + (K // 64) * N * 4
    assert ql.workspace_size8(2, 4096, 64, ql.PATH_GEMV, 4) == 4 * 2 * 64 * 4
    assert L.qlinear8_workspace_size(16, 100, 256, 64) == ctypes.c_size_t(-1).value


# ---------------------------------------------------------------- SwiGLU pair

def _sw(L, x=FAKE, gc=FAKE + (1 << 24), gs=FAKE + (2 << 24), gb=FAKE + (3 << 24), uc=FAKE + (5 << 24),
        us=FAKE + (6 << 24), ub=FAKE + (7 << 24), h=FAKE + (4 << 24), dt=1, M=16, K=256, I=256, group=64,
        ws=FAKE + (8 << 24), ws_bytes=1 << 24):
    return L.qlinear_swiglu_forward(x, gc, gs, gb, uc, us, ub, h, dt, M, K, I, group, ws, ws_bytes, None)


def test_swiglu_rejects_bad_arguments(L):
    assert _sw(L, group=32) == 3
    assert _sw(L, K=100) == 1
    assert _sw(L, I=12) == 1
    assert _sw(L, M=0) == 1
    assert _sw(L, uc=0) == 1
    assert _sw(L, dt=7) == 1
    assert _sw(L, ub=FAKE + (7 << 24) + 2) == 2
    assert _sw(L, h=FAKE + (5 << 24) + 64) == 1          # h inside the up codes
    assert _sw(L, ws=None, ws_bytes=0) == 4
    assert _sw(L, ws_bytes=100) == 4
    assert _sw(L, ws=FAKE + (4 << 24)) == 1              # workspace over h


def test_swiglu_workspace_size(L):
    M, K, I = 4608, 4608, 12288
    # f16 activations, row scales, and (scale, bias) pairs of 256 interleaved rows per 128-column tile
    assert ql.swiglu_workspace_size(M, K, I) == M * K * 2 + M * 4 + (K // 64) * ((I + 127) // 128) * 256 * 4
    assert L.qlinear_swiglu_workspace_size(16, 100, 256, 64) == ctypes.c_size_t(-1).value


def test_reduce_partials_validation(L):
    assert L.qlinear_reduce_partials(None, 2, 64, FAKE, 1, None) == 1
    assert L.qlinear_reduce_partials(FAKE, 0, 64, FAKE + (1 << 24), 1, None) == 1
    assert L.qlinear_reduce_partials(FAKE, 2, 66, FAKE + (1 << 24), 1, None) == 1     # not a multiple of 4
    assert L.qlinear_reduce_partials(FAKE, 2, 64, FAKE + (1 << 24), 5, None) == 1
    assert L.qlinear_reduce_partials(FAKE + 4, 2, 64, FAKE + (1 << 24), 1, None) == 2
    assert L.qlinear_reduce_partials(FAKE, 2, 64, FAKE + 256, 1, None) == 1           # y inside the partials


def test_fused_split_k_workspace(L):
    """The fused path's split-K adds fp32 partials [S][M][N] to its workspace; more slices than groups is an error."""
    M, K, N = 512, 53248, 4608
    base = ql.workspace_size(M, K, N, ql.PATH_TC_FUSED, 1)
    assert ql.workspace_size(M, K, N, ql.PATH_TC_FUSED, 8) == base + 8 * M * N * 4
    assert L.qlinear_workspace_size_config(16, 256, 256, 64, ql.PATH_TC_FUSED, 5) == ctypes.c_size_t(-1).value


def test_bounds_checked_build_exports_every_declared_symbol():
    """The index-checked variant (QL_BOUNDS_CHECK, selected at run time by QL_LIBRARY) builds and exports the ABI."""
    Lb = ctypes.CDLL(qb.build(bounds_check=True))
    for n in _declared():
        assert hasattr(Lb, n), n


def test_test_hooks_are_inert_in_the_shipped_library(L):
    """The checked build's hooks (held-back producers, ring depths) change nothing in the shipped library."""
    assert L.qlinear_test_stall(1, 20_000_000) == 3              # QL_ERR_UNSUPPORTED
    assert L.qlinear_test_ring_depth(1) == 3
    assert L.qlinear_test_ring_depth(0) == 3
    assert L.qlinear_test_delay(31, 10_000) == 3
