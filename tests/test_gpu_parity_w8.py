"""GPU parity of the W8 g64 variant (8-bit codes, uint32 [N][K/4], low byte first) against the oracle.

The same bars as the 4-bit path: bit-exact dequant, RTN pack and one-hot forward; the tolerance of
reading R5 for the forward pass on every kernel path, at small shapes with ragged edges and on
sampled rows of the full conditioning projection (K = 53248, N = 4608), which the pages keep at
8 bits.
"""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import synthetic as S
from oracle import qlinear_oracle as O

from ._helpers import FUSED_TILE_TOKENS, bf16_bits, random_layer8, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16

pytestmark = pytest.mark.gpu

PATHS = {"gemv": ql.PATH_GEMV, "tc_fused": ql.PATH_TC_FUSED, "tc_skinny": ql.PATH_TC_SKINNY}
MAX_M = {"gemv": 129, "tc_fused": 1 << 30, "tc_skinny": 32}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required for -m gpu tests")
    ql.lib()
    yield
    assert ql.device_status() == 0


def _dev(codes, s, b):
    return to_dev_codes(codes), to_dev_f16(s), to_dev_f16(b)


def _check_tol(y_dev, y_ref, bf16=True):
    y = O.decode_bf16(bf16_bits(y_dev)) if bf16 else y_dev.double().cpu().numpy()
    t = O.tolerance(y, y_ref, bf16_output=bf16)
    assert t["relF"] <= 4e-3 and t["max_gate"] <= 1.5e-2, t
    return t


# ------------------------------------------------------------------ dequant

@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_dequant8_bitexact(dt):
    rng = np.random.default_rng(80)
    _, codes, s, b = random_layer8(rng, 1, 1024, 264)
    out = ql.dequant8(*_dev(codes, s, b), out_dtype=dt)
    if dt == torch.float32:
        assert np.array_equal(out.cpu().numpy().view(np.uint32), O.dequant8_f32(codes, s, b).view(np.uint32))
    else:
        assert np.array_equal(bf16_bits(out), O.dequant8_bf16(codes, s, b))


def test_dequant8_all_codes_edge_values_bitexact():
    """All 256 codes x f16 edge values (zeros, subnormals, max normal, negatives) for scale and bias."""
    e = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x0400, 0x3C00, 0xBC00, 0x7BFF, 0xFBFF,
                  0x1400, 0x2E66, 0xC000, 0x3555, 0x0200, 0x8200], dtype=np.uint16)
    S_, B_ = np.meshgrid(e, e, indexing="ij")
    N = S_.size
    s = np.repeat(S_.reshape(N, 1), 4, axis=1).view(np.float16)
    b = np.repeat(B_.reshape(N, 1), 4, axis=1).view(np.float16)
    q = np.tile(np.arange(256), 1)[None, :].repeat(N, 0)          # one row = 4 groups = codes 0..255
    codes = O.pack_codes8(q)
    for dt in (torch.float32, torch.bfloat16):
        out = ql.dequant8(*_dev(codes, s, b), out_dtype=dt)
        if dt == torch.float32:
            got = out.cpu().numpy()
            ref = O.dequant8_f32(codes, s, b)
            both_nan = np.isnan(got) & np.isnan(ref)
            assert np.array_equal(got.view(np.uint32)[~both_nan], ref.view(np.uint32)[~both_nan])
        else:
            assert np.array_equal(bf16_bits(out), O.dequant8_bf16(codes, s, b))


# ------------------------------------------------------------------ pack

def test_pack8_rtn_bitexact():
    rng = np.random.default_rng(81)
    w = (rng.standard_normal((96, 512)) * 0.02).astype(np.float32)
    w[3, :64] = 0.125                        # constant group
    w[4, 64:128] = np.float32(-65504.0)      # extreme but packable
    w[4, 70] = 65504.0
    w[5, :64] = rng.standard_normal(64).astype(np.float32) * 1e-7   # scale rounds to an f16 subnormal or zero
    w[6, :] = np.round(w[6, :] * 1000) / 1000
    c, s, b = ql.pack8(torch.from_numpy(w).cuda())
    rc, rs, rb = O.pack8_rtn(w)
    assert np.array_equal(c.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(b.cpu().numpy().view(np.uint16), rb.view(np.uint16))
    assert ql.device_status() == 0


def test_pack8_rtn_bitexact_dit_weight():
    w = S.dense_weight(2, 0, 256, 4608, 0.02)
    c, s, b = ql.pack8(torch.from_numpy(w).cuda())
    rc, rs, rb = O.pack8_rtn(w)
    assert np.array_equal(c.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(b.cpu().numpy().view(np.uint16), rb.view(np.uint16))


def test_pack8_nonfinite_reports_status():
    w = np.zeros((8, 128), dtype=np.float32)
    w[2, 5] = np.nan
    w[5, 100] = 1e6
    c, s, b = ql.pack8(torch.from_numpy(w).cuda())
    assert ql.device_status() == 1          # QL_ERR_INVALID_ARG
    cs = c.cpu().numpy()
    assert np.all(cs[2, :16] == 0) and np.all(cs[5, 16:] == 0)


def test_pack8_then_forward8_matches_oracle():
    """Quantize on the device, run the layer on the device, compare with the oracle on the packed result."""
    w = S.dense_weight(5, 0, 264, 1024, 0.02)
    c, s, b = ql.pack8(torch.from_numpy(w).cuda())
    x = random_layer8(np.random.default_rng(82), 24, 1024, 8)[0]
    codes, sn, bn = c.cpu().numpy().view(np.uint32), s.cpu().numpy(), b.cpu().numpy()
    for path in PATHS.values():
        y = ql.forward8(to_dev_bf16(x), c, s, b, path=path)
        _check_tol(y, O.forward8_ref(x, codes, sn, bn))


# ------------------------------------------------------------------ forward, small shapes

@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_forward8_small(path, out):
    rng = np.random.default_rng(83)
    x, codes, s, b = random_layer8(rng, 16, 256, 256)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    y = ql.forward8(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path], out_dtype=dt)
    _check_tol(y, O.forward8_ref(x, codes, s, b), bf16=(out == "bf16"))
    assert ql.last_dispatch().startswith(f"path={path} bits=8")


@pytest.mark.parametrize("path", list(PATHS))
def test_forward8_one_hot_bitexact(path):
    """x rows = unit vectors select single weights: exact results.

    CUDA-core path (exact codes, fp32 scale and bias): y = RN_bf16(fp32 dequant).
    Tensor-core paths (weights dequantized to an f16 operand): y = RN_bf16(RN_f16(w)).
    Every position of a code word and both halves of a 64-group are hit.
    """
    rng = np.random.default_rng(84)
    K, N = 320, 264
    _, codes, s, b = random_layer8(rng, 1, K, N)
    ks = np.array([0, 1, 2, 3, 4, 5, 6, 7, 8, 15, 16, 31, 32, 63, 64, 65, 66, 67, 130, 200, 255, 256, 257, 258,
                   259, 318, 319] + list(range(9, 320, 37)))
    if path == "tc_skinny":
        ks = ks[:32]
    x = np.zeros((ks.size, K), dtype=np.uint16)
    x[np.arange(ks.size), ks] = 0x3F80
    y = ql.forward8(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path])
    got = bf16_bits(y)
    if path == "gemv":
        ref = O.dequant8_bf16(codes, s, b)[:, ks].T
    else:
        ref = O.round_bf16(O.dequant8_f16(codes, s, b).astype(np.float64))[:, ks].T
    assert np.array_equal(got, ref)


RAGGED_M = [1, 2, 3, 7, 8, 31, 32, 33, 127, 129, 255, 257, 513]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("K,N", [(64, 8), (320, 264), (1024, 520)])
def test_forward8_ragged(path, K, N):
    rng = np.random.default_rng(K + N + 85)
    for M in RAGGED_M:
        if M > MAX_M[path]:
            continue
        x, codes, s, b = random_layer8(rng, M, K, N)
        y = ql.forward8(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path])
        _check_tol(y, O.forward8_ref(x, codes, s, b))


@pytest.mark.parametrize("M", [1, 8, 17, 32])
@pytest.mark.parametrize("K,N", [(64, 8), (128, 4608), (4096, 264), (65536, 128), (4160, 200), (4352, 136)])
def test_skinny8_stream_k_shapes(M, K, N):
    """Stream-K runs of 4-group chunks: runs that start and end inside tiles, one tile shared by many
    CTAs, parameter boxes of 8 groups read by two chunks each (4096, 65536), a group count that is no
    whole number of chunks (4160 = 65 groups), and whole chunks with direct parameter loads (4352 = 68
    groups, no whole number of 8-group boxes)."""
    rng = np.random.default_rng(M * 7 + K + N + 86)
    x, codes, s, b = random_layer8(rng, M, K, N)
    y = ql.forward8(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_SKINNY)
    _check_tol(y, O.forward8_ref(x, codes, s, b))


@pytest.mark.parametrize("path", list(PATHS))
def test_forward8_activation_dynamic_range(path):
    rng = np.random.default_rng(87)
    K, N = 1024, 264
    _, codes, s, b = random_layer8(rng, 6, K, N)
    base = rng.standard_normal((6, K))
    rows = np.empty((6, K))
    rows[0] = base[0]
    rows[1] = 0.0
    rows[2] = base[2] * 1e30
    rows[3] = base[3] * 1e-30
    rows[4] = np.sign(base[4]) * np.exp2(rng.uniform(-40, 40, K))
    rows[5] = 1e-6 * base[5]
    rows[5, 17] = 1e4
    x = S.f32_to_bf16_bits(rows.astype(np.float32))
    y = ql.forward8(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path])
    ref = O.forward8_ref(x, codes, s, b)
    got = O.decode_bf16(bf16_bits(y))
    assert np.all(got[1] == 0.0)
    for t in (0, 2, 3, 4, 5):
        tol = O.tolerance(got[t:t + 1], ref[t:t + 1], bf16_output=True)
        assert tol["relF"] <= 4e-3 and tol["max_gate"] <= 1.5e-2, (t, tol)


@pytest.mark.parametrize("split", [1, 3, 16])
def test_gemv8_split_k(split):
    rng = np.random.default_rng(88 + split)
    x, codes, s, b = random_layer8(rng, 4, 1024, 64)
    y = ql.forward8(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_GEMV, split_k=split)
    _check_tol(y, O.forward8_ref(x, codes, s, b))


def test_forward8_deterministic():
    rng = np.random.default_rng(89)
    x, codes, s, b = random_layer8(rng, 24, 8192, 1024)
    args = (to_dev_bf16(x), *_dev(codes, s, b))
    for path in PATHS.values():
        a = bf16_bits(ql.forward8(*args, path=path))
        c = bf16_bits(ql.forward8(*args, path=path))
        assert np.array_equal(a, c)


def test_forward8_rejects_imatrix_pack_and_wrong_code_shape():
    L = ql.lib()
    w = torch.zeros((8, 128), dtype=torch.float32, device="cuda")
    imp = torch.ones(128, dtype=torch.float32, device="cuda")
    c = torch.empty((8, 32), dtype=torch.int32, device="cuda")
    sc = torch.empty((8, 2), dtype=torch.float16, device="cuda")
    bi = torch.empty((8, 2), dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert L.qlinear8_pack(w.data_ptr(), imp.data_ptr(), 128, 8, 64, c.data_ptr(), sc.data_ptr(), bi.data_ptr(),
                           st) == 3
    x = torch.zeros((2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        ql.forward8(x, c[:, :16].contiguous(), sc, bi)      # 4-bit-shaped codes


# ------------------------------------------------------------------ the conditioning projection at 8 bits

@pytest.mark.parametrize("M", S.TEXT_PROJ_M)
def test_full_text_proj_w8(M):
    w = S.WORKLOADS["text_proj_w8"]
    x = w.x(M)
    codes, s, b = w.w()
    y = ql.forward8(to_dev_bf16(x), *_dev(codes, s, b))
    rows = sample_rows(M, n_random=48, seed=M, tile=FUSED_TILE_TOKENS)
    y_ref = O.forward8_rows(x, codes, s, b, rows)
    t = O.tolerance(O.decode_bf16(bf16_bits(y)[rows]), y_ref)
    assert t["ok"], (M, t)
