"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Bit-exact where the result is integer or defined by a single rounding
(dequant, RTN pack, one-hot forward); within the tolerance of reading R5
(relative Frobenius <= 4e-3, half-ulp-adjusted max error <= 1.5e-2 * rms)
for the forward pass.
"""
import numpy as np
import pytest
import torch

import group_wise_affine_qlinear_b200 as ql
from group_wise_affine_qlinear_b200 import synthetic as S
from oracle import qlinear_oracle as O

from ._helpers import FUSED_TILE_TOKENS, bf16_bits, random_layer, sample_rows, to_dev_bf16, to_dev_codes, to_dev_f16

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


def _check_tol(y_dev, y_ref, bf16=True, limit_relF=4e-3, limit_max=1.5e-2):
    y = O.decode_bf16(bf16_bits(y_dev)) if bf16 else y_dev.double().cpu().numpy()
    t = O.tolerance(y, y_ref, bf16_output=bf16)
    assert t["relF"] <= limit_relF and t["max_gate"] <= limit_max, t
    return t


# ------------------------------------------------------------------ dequant

@pytest.mark.parametrize("name", ["tiny", "qkv"])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_dequant_bitexact(name, dt):
    codes, s, b = S.WORKLOADS[name].w()
    out = ql.dequant(*_dev(codes, s, b), out_dtype=dt)
    torch.cuda.synchronize()
    if dt == torch.float32:
        ref = O.dequant_f32(codes, s, b)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    else:
        assert np.array_equal(bf16_bits(out), O.dequant_bf16(codes, s, b))


def test_dequant_edge_values_bitexact():
    """Every code x f16 edge values (zeros, subnormals, max normal, negatives) for scale and bias."""
    e = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x0400, 0x3C00, 0xBC00, 0x7BFF, 0xFBFF,
                  0x1400, 0x2E66, 0xC000, 0x3555, 0x0200, 0x8200], dtype=np.uint16)
    S_, B_ = np.meshgrid(e, e, indexing="ij")
    N = S_.size
    s = S_.reshape(N, 1).view(np.float16)
    b = B_.reshape(N, 1).view(np.float16)
    q = np.tile(np.arange(16), 4)[None, :].repeat(N, 0)
    codes = O.pack_codes(q)
    for dt in (torch.float32, torch.bfloat16):
        out = ql.dequant(*_dev(codes, s, b), out_dtype=dt)
        if dt == torch.float32:
            got = out.cpu().numpy()
            ref = O.dequant_f32(codes, s, b)
            both_nan = np.isnan(got) & np.isnan(ref)
            assert np.array_equal(got.view(np.uint32)[~both_nan], ref.view(np.uint32)[~both_nan])
        else:
            assert np.array_equal(bf16_bits(out), O.dequant_bf16(codes, s, b))


# ------------------------------------------------------------------ pack

def _pack_inputs(seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((96, 512)) * 0.02).astype(np.float32)
    w[3, :64] = 0.125                        # constant group
    w[4, 64:128] = np.float32(-65504.0)      # extreme but packable
    w[4, 70] = 65504.0
    w[5, :64] = rng.standard_normal(64).astype(np.float32) * 1e-7   # scale rounds to an f16 subnormal/zero
    w[6, :] = np.round(w[6, :] * 1000) / 1000
    return w


def test_pack_rtn_bitexact():
    w = _pack_inputs(1)
    c, s, b = ql.pack(torch.from_numpy(w).cuda())
    rc, rs, rb = O.pack_rtn(w)
    assert np.array_equal(c.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(b.cpu().numpy().view(np.uint16), rb.view(np.uint16))
    assert ql.device_status() == 0


def test_pack_rtn_bitexact_dit_weight():
    w = S.dense_weight(2, 0, 512, 4608, 0.02)
    c, s, b = ql.pack(torch.from_numpy(w).cuda())
    rc, rs, rb = O.pack_rtn(w)
    assert np.array_equal(c.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(b.cpu().numpy().view(np.uint16), rb.view(np.uint16))


def test_pack_nonfinite_reports_status():
    w = np.zeros((8, 128), dtype=np.float32)
    w[2, 5] = np.nan
    w[5, 100] = 1e6
    c, s, b = ql.pack(torch.from_numpy(w).cuda())
    assert ql.device_status() == 1          # QL_ERR_INVALID_ARG
    assert ql.device_status() == 0          # read clears
    cs = c.cpu().numpy()
    assert np.all(cs[2, :8] == 0) and np.all(cs[5, 8:] == 0)
    with pytest.raises(ValueError):
        O.pack_rtn(w)


def _fit_case():
    """64 dense rows of N(0, 0.02^2) weights (the fitted MLP rows' recipe) with special groups, and the
    E[x^2] of 512 synthetic activation rows, rounded to fp32, with some channels never reached."""
    K = 4608
    w = S.dense_weight(2, 0, 64, K, 0.02)
    w[0, :64] = 0.0125                                   # constant group
    w[1, 64:128] = 0.0
    w[2, :64] *= 0.01
    w[2, 7] = 0.3                                        # one outlier dominates the range
    w[3, :64] = (np.arange(64) % 16).astype(np.float32) * np.float32(0.002) - np.float32(0.01)   # on a grid
    imp = O.imatrix_from_x(S.activations(2, 0, 512, K)).astype(np.float32)
    imp[100:164] = 0.0                                   # channels no activation reached
    imp[4000] = 0.0
    return w, imp


def test_pack_imatrix_bitexact():
    w, imp = _fit_case()
    c, s, b = ql.pack(torch.from_numpy(w).cuda(), imatrix=torch.from_numpy(imp).cuda())
    rc, rs, rb = O.pack_imatrix(w, imp.astype(np.float64))
    assert ql.device_status() == 0
    assert np.array_equal(c.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), rs.view(np.uint16))
    assert np.array_equal(b.cpu().numpy().view(np.uint16), rb.view(np.uint16))


def test_pack_imatrix_never_worse_than_rtn():
    """The pages' guarantee, checked on the device result against the oracle's objective."""
    w, imp = _fit_case()
    c, s, b = ql.pack(torch.from_numpy(w).cuda(), imatrix=torch.from_numpy(imp).cuda())
    imp64 = imp.astype(np.float64)
    imp64 = imp64 + 1e-6 * imp64.mean()
    e_fit = O.group_weighted_error(w, c.cpu().numpy().view(np.uint32), s.cpu().numpy(), b.cpu().numpy(), imp64)
    e_rtn = O.group_weighted_error(w, *O.pack_rtn(w), imp64)
    assert np.all(e_fit <= e_rtn * (1 + 1e-12))
    assert e_fit.sum() < e_rtn.sum()


def test_pack_imatrix_rejects_bad_importance():
    w = S.dense_weight(2, 1, 8, 128, 0.02)
    imp = np.ones(128, dtype=np.float32)
    imp[5] = -1.0
    c, s, b = ql.pack(torch.from_numpy(w).cuda(), imatrix=torch.from_numpy(imp).cuda())
    assert ql.device_status() == 1          # QL_ERR_INVALID_ARG
    assert not c.cpu().numpy().any() and not s.cpu().numpy().view(np.uint16).any()


# ------------------------------------------------------------------ forward: small and ragged

def test_skinny_rejects_large_m():
    rng = np.random.default_rng(12)
    x, codes, s, b = random_layer(rng, 65, 256, 64)
    with pytest.raises(ValueError):
        ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_SKINNY)


@pytest.mark.parametrize("M", [1, 8, 16, 17, 32])
@pytest.mark.parametrize("K,N", [(64, 8), (128, 4608), (4096, 264), (8192, 1032), (65536, 128), (4160, 200)])
def test_skinny_stream_k_shapes(M, K, N):
    """Runs that start and end inside tiles, tiles shorter than a run, ragged N, one tile shared by
    128 CTAs (65536 x 128), and a group count that is not a whole number of chunks (4160 = 65 groups)."""
    rng = np.random.default_rng(M * 7 + K + N)
    x, codes, s, b = random_layer(rng, M, K, N)
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_TC_SKINNY)
    _check_tol(y, O.forward_ref(x, codes, s, b))
    assert ql.last_dispatch().startswith("path=tc_skinny")


@pytest.mark.parametrize("path", list(PATHS))
def test_activation_dynamic_range(path):
    """Rows of very different magnitude: the tensor-core paths scale each activation row by its own
    power of two before rounding it to f16, so every row must meet the tolerance on its own, a zero
    row must give exact zeros, and a row of one spike plus tiny values must stay within tolerance."""
    rng = np.random.default_rng(11)
    K, N = 1024, 264
    _, codes, s, b = random_layer(rng, 6, K, N)
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
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path])
    ref = O.forward_ref(x, codes, s, b)
    got = O.decode_bf16(bf16_bits(y))
    assert np.all(got[1] == 0.0)
    for t in (0, 2, 3, 4, 5):
        tol = O.tolerance(got[t:t + 1], ref[t:t + 1], bf16_output=True)
        assert tol["relF"] <= 4e-3 and tol["max_gate"] <= 1.5e-2, (t, tol)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_forward_tiny(path, out):
    w = S.WORKLOADS["tiny"]
    x = w.x()
    codes, s, b = w.w()
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path], out_dtype=dt)
    _check_tol(y, O.forward_ref(x, codes, s, b), bf16=(out == "bf16"))


@pytest.mark.parametrize("path", list(PATHS))
def test_forward_one_hot_bitexact(path):
    """x rows = unit vectors: y selects single weights, so the result is exact.

    CUDA-core path (exact codes, fp32 scale and bias): y = RN_bf16(fp32 dequant).
    Tensor-core paths (weights dequantized to an f16 operand): y = RN_bf16(RN_f16(w)).
    """
    rng = np.random.default_rng(3)
    K, N = 320, 264
    _, codes, s, b = random_layer(rng, 1, K, N)
    ks = np.array([0, 1, 4, 7, 8, 63, 64, 65, 130, 200, 255, 256, 319] + list(range(9, 320, 23)))
    if path == "tc_skinny":
        ks = ks[:32]
    x = np.zeros((ks.size, K), dtype=np.uint16)
    x[np.arange(ks.size), ks] = 0x3F80
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path])
    got = bf16_bits(y)
    if path == "gemv":
        ref = O.dequant_bf16(codes, s, b)[:, ks].T
    else:
        ref = O.round_bf16(O.dequant_f16(codes, s, b).astype(np.float64))[:, ks].T
    assert np.array_equal(got, ref)


RAGGED_M = [1, 2, 3, 7, 8, 31, 32, 33, 127, 129, 255, 257, 513]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("K,N", [(64, 8), (320, 264), (1024, 520)])
def test_forward_ragged(path, K, N):
    rng = np.random.default_rng(K + N)
    for M in RAGGED_M:
        if M > MAX_M[path]:
            continue
        x, codes, s, b = random_layer(rng, M, K, N)
        y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=PATHS[path])
        _check_tol(y, O.forward_ref(x, codes, s, b))


@pytest.mark.parametrize("split", [1, 2, 3, 5, 16])
def test_gemv_split_k(split):
    rng = np.random.default_rng(split)
    x, codes, s, b = random_layer(rng, 4, 1024, 64)
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_GEMV, split_k=split)
    _check_tol(y, O.forward_ref(x, codes, s, b))


def test_gemv_split_k_beyond_groups_rejected():
    rng = np.random.default_rng(4)
    x, codes, s, b = random_layer(rng, 4, 1024, 64)
    with pytest.raises(ValueError):
        ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=ql.PATH_GEMV, split_k=17)


def test_forward_deterministic():
    rng = np.random.default_rng(7)
    x, codes, s, b = random_layer(rng, 300, 1024, 512)
    args = (to_dev_bf16(x), *_dev(codes, s, b))
    for name, path in PATHS.items():
        if name == "tc_skinny":
            continue
        a = bf16_bits(ql.forward(*args, path=path))
        c = bf16_bits(ql.forward(*args, path=path))
        assert np.array_equal(a, c)


def test_skinny_deterministic():
    rng = np.random.default_rng(17)
    x, codes, s, b = random_layer(rng, 24, 8192, 1024)
    args = (to_dev_bf16(x), *_dev(codes, s, b))
    a = bf16_bits(ql.forward(*args, path=ql.PATH_TC_SKINNY))
    c = bf16_bits(ql.forward(*args, path=ql.PATH_TC_SKINNY))
    assert np.array_equal(a, c)


def test_dispatch_record():
    rng = np.random.default_rng(8)
    x, codes, s, b = random_layer(rng, 256, 256, 256)
    ql.forward(to_dev_bf16(x), *_dev(codes, s, b))
    assert ql.last_dispatch().startswith("path=tc_fused")
    assert f" x {FUSED_TILE_TOKENS}t " in ql.last_dispatch()      # the tile the tests sample boundaries of
    ql.forward(to_dev_bf16(x[:1]), *_dev(codes, s, b))
    assert ql.last_dispatch().startswith("path=tc_skinny")


def test_workspace_and_alignment_errors():
    rng = np.random.default_rng(9)
    x, codes, s, b = random_layer(rng, 256, 256, 256)
    xd, cd, sd, bd = to_dev_bf16(x), *_dev(codes, s, b)
    L = ql.lib()
    y = torch.empty((256, 256), dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    need = ql.workspace_size(256, 256, 256)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ok = L.qlinear_forward(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                           256, 256, 256, 64, ws.data_ptr(), need, st)
    assert ok == 0
    assert L.qlinear_forward(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                             256, 256, 256, 64, ws.data_ptr(), need - 1, st) == 4
    assert L.qlinear_forward(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                             256, 256, 256, 64, None, 0, st) == 4
    assert L.qlinear_forward(xd.data_ptr() + 2, cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                             255, 256, 256, 64, ws.data_ptr(), need, st) == 2
    # y aliasing x
    assert L.qlinear_forward(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), xd.data_ptr(),
                             256, 256, 256, 64, ws.data_ptr(), need, st) == 1
    # workspace overlapping y
    assert L.qlinear_forward(xd.data_ptr(), cd.data_ptr(), sd.data_ptr(), bd.data_ptr(), y.data_ptr(),
                             256, 256, 256, 64, y.data_ptr(), need, st) == 1


# ------------------------------------------------------------------ forward: the full workloads (sampled rows)

def _full_case(name, M=None, path=ql.PATH_AUTO, fitted=None):
    w = S.WORKLOADS[name]
    M = w.M if M is None else M
    x = w.x(M)
    codes, s, b = w.w() if fitted is None else fitted
    y = ql.forward(to_dev_bf16(x), *_dev(codes, s, b), path=path)
    rows = sample_rows(M, n_random=48, seed=M, tile=FUSED_TILE_TOKENS)
    y_ref = O.forward_rows(x, codes, s, b, rows)
    got = bf16_bits(y)[rows]
    t = O.tolerance(O.decode_bf16(got), y_ref)
    assert t["ok"], (name, M, t)
    return t


@pytest.mark.parametrize("M", S.TEXT_PROJ_M)
def test_full_text_proj(M):
    _full_case("text_proj", M)


def test_full_qkv():
    _full_case("qkv")


def test_full_mlp_down():
    _full_case("mlp_down")


@pytest.mark.parametrize("name", ["canvas2048_n4608", "canvas2048_n13824"])
def test_full_canvas2048(name):
    _full_case(name)


@pytest.mark.parametrize("name,M,split", [("qkv", None, 0), ("text_proj", 512, 0), ("text_proj", 32, 0),
                                          ("mlp_down", None, 0)])
def test_full_size_repeatable_with_poisoned_workspace(name, M, split):
    """Three calls on the same input, the workspace filled with 0xFF bytes (NaN in every f16 and fp32 slot,
    0xFFFFFFFF in every count) before each: the same bytes every time, and no NaN.  The calls' pipelines
    (TMA rings, TMEM stages, accumulator hand-offs, split-K partials, stream-K segments) run at full size
    with every CTA busy, where an ordering race between roles or CTAs shows up as differing tiles."""
    w = S.WORKLOADS[name]
    M = w.M if M is None else M
    codes, s, b = w.w()
    xd = to_dev_bf16(w.x(M))
    cd, sd, bd = _dev(codes, s, b)
    ws = torch.empty(max(ql.workspace_size(M, w.K, w.N, ql.PATH_AUTO, split), 16), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        ws.fill_(0xFF)
        y = ql.forward(xd, cd, sd, bd, workspace=ws, split_k=split)
        assert ql.device_status() == 0
        outs.append(bf16_bits(y))
    assert not np.any((outs[0] & 0x7F80) == 0x7F80), "NaN or infinity in the output"
    for o in outs[1:]:
        diff = np.flatnonzero(o != outs[0])
        assert diff.size == 0, (name, M, diff.size, diff[:8])
