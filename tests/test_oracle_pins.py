"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test states what fixes the expected value: a library conversion, exact
rational arithmetic, a closed form, brute force, or a number the pages print.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import qlinear_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _random_layer(rng, M, K, N):
    codes = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint32)
    s = np.exp(rng.uniform(np.log(1e-3), np.log(2e-2), size=(N, K // 64))).astype(np.float16)
    b = (-7.5 * s.astype(np.float64) + 0.1 * s.astype(np.float64) * rng.standard_normal(s.shape)).astype(np.float16)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16), codes, s, b


# ---------------------------------------------------------------- decoding

def test_decode_f16_all_patterns_match_numpy():
    """All 65536 binary16 patterns: the bit-field decoder equals numpy's half->double conversion."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = O.decode_f16(bits)
    lib = bits.view(np.float16).astype(np.float64)
    both_nan = np.isnan(ours) & np.isnan(lib)
    assert np.array_equal(ours[~both_nan], lib[~both_nan])
    assert np.array_equal(np.isnan(ours), np.isnan(lib))


def test_decode_bf16_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):          # signalling-NaN patterns among the 65536
        ours = O.decode_bf16(bits)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    both_nan = np.isnan(ours) & np.isnan(lib)
    assert np.array_equal(ours[~both_nan], lib[~both_nan])


def test_round_bf16_from_f32_matches_torch():
    """For binary32 inputs the oracle's bf16 rounding equals torch's float->bfloat16 cast."""
    rng = _rng(1)
    u = rng.integers(0, 1 << 32, size=200000, dtype=np.uint64).astype(np.uint32)
    # include ties, near-ties and extremes
    extra = np.array([0x3F808000, 0x3F818000, 0x3F80FFFF, 0x7F7FFFFF, 0x7F7F8000, 0x00000001,
                      0x80000000, 0x00800000, 0x3F800000], dtype=np.uint32)
    u = np.concatenate([u, extra])
    f = u.view(np.float32)
    finite = np.isfinite(f)
    ours = O.round_bf16(f[finite].astype(np.float64))
    lib = torch.from_numpy(f[finite]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


def test_round_bf16_from_f64_is_nearest_with_ties_even():
    """Brute force: compare with the nearer of the two bf16 neighbours (exact rationals)."""
    rng = _rng(2)
    v = rng.standard_normal(3000) * np.exp(rng.uniform(-20, 20, 3000))
    got = O.decode_bf16(O.round_bf16(v))
    for val, g in zip(v, got):
        # neighbours: truncate the binary32 pattern of a value just below/above
        f32 = np.float32(val)
        cands = set()
        for t in (np.nextafter(f32, np.float32(-np.inf)), f32, np.nextafter(f32, np.float32(np.inf))):
            hi = (np.array([t], dtype=np.float32).view(np.uint32)[0] >> 16)
            for d in (-1, 0, 1):
                cands.add(int(hi) + d)
        best = None
        for c in sorted(cands):
            cv = Fraction(float(O.decode_bf16(np.array([c & 0xFFFF]))[0]))
            dist = abs(cv - Fraction(float(val)))
            key = (dist, c & 1)           # ties: even significand
            if best is None or key < best[0]:
                best = (key, cv)
        assert Fraction(float(g)) == best[1]


def test_nibble_order_low_first():
    """Reading R1: code k%8 sits in bits 4*(k%8)..; word 0x76543210 holds codes 0..7 in order."""
    codes = np.array([[0x76543210, 0xFEDCBA98]], dtype=np.uint32)
    q = O.unpack_codes(codes, 16)
    assert q.tolist() == [list(range(16))]
    assert np.array_equal(O.pack_codes(q), codes)


def test_pack_unpack_roundtrip():
    rng = _rng(3)
    codes = rng.integers(0, 1 << 32, size=(7, 40), dtype=np.uint32)
    assert np.array_equal(O.pack_codes(O.unpack_codes(codes, 320)), codes)


def test_bits_per_weight_is_4_5_golden():
    """Packed size = 4 bits/code + f16 scale + f16 bias per 64 = 4.5 bits/weight (the pages' figure)."""
    g = json.load(open(os.path.join(GOLDEN, "format_constants.json")))
    group = g["group_size"]["value"]
    bpw = g["code_bits"]["value"] + g["overhead_bits_per_weight"]["value"]
    K, N = 4608, 13824
    w = np.zeros((N, K), dtype=np.float32)
    w[:, ::2] = 1.0
    codes, s, b = O.pack_rtn(w[:64])          # small pack: check the per-row layout sizes
    assert codes.shape == (64, K // 8) and s.shape == (64, K // group) and b.shape == (64, K // group)
    row_bytes = codes[0].nbytes + s[0].nbytes + b[0].nbytes
    assert row_bytes * 8 == bpw * K
    assert row_bytes * N == 35_831_808


# ---------------------------------------------------------------- dequant

def _edge_f16():
    vals = [0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x0400, 0x3C00, 0xBC00, 0x7BFF, 0xFBFF,
            0x1400, 0x2E66, 0xC000, 0x3555, 0x0200, 0x8200]
    return np.array(vals, dtype=np.uint16)


def test_dequant_exact_equals_rational_arithmetic():
    """s*q + b computed with exact rationals equals dequant_exact for every code and edge f16 value."""
    e = _edge_f16()
    S, B = np.meshgrid(e, e, indexing="ij")
    S = S.reshape(-1, 1)
    B = B.reshape(-1, 1)
    N = S.shape[0]
    # one group per row, codes 0..15 repeated 4 times
    q = np.tile(np.arange(16), 4)[None, :].repeat(N, 0)
    codes = O.pack_codes(q)
    got = O.dequant_exact(codes, S.view(np.float16), B.view(np.float16))
    for n in range(N):
        s = Fraction(float(np.array(S[n]).view(np.float16)[0]))
        b = Fraction(float(np.array(B[n]).view(np.float16)[0]))
        for k in range(16):
            assert Fraction(float(got[n, k])) == s * k + b


def test_dequant_f32_is_correctly_rounded():
    """fp32 dequant = binary32 nearest (ties even) to the exact rational s*q + b."""
    rng = _rng(4)
    x, codes, s, b = _random_layer(rng, 1, 256, 64)
    w32 = O.dequant_f32(codes, s, b)
    q = O.unpack_codes(codes, 256)
    for n in range(0, 64, 7):
        for k in range(0, 256, 5):
            exact = Fraction(float(s[n, k // 64])) * int(q[n, k]) + Fraction(float(b[n, k // 64]))
            got = Fraction(float(w32[n, k]))
            # neighbours of got in binary32
            lo = Fraction(float(np.nextafter(w32[n, k], np.float32(-np.inf))))
            hi = Fraction(float(np.nextafter(w32[n, k], np.float32(np.inf))))
            assert abs(got - exact) <= abs(lo - exact) and abs(got - exact) <= abs(hi - exact)


def test_dequant_f16_is_correctly_rounded():
    """f16 operand = binary16 nearest to the exact rational s*q + b (checked against both neighbours)."""
    rng = _rng(17)
    _, codes, s, b = _random_layer(rng, 1, 128, 24)
    w16 = O.dequant_f16(codes, s, b)
    q = O.unpack_codes(codes, 128)
    for n in range(24):
        for k in range(0, 128, 3):
            exact = Fraction(float(s[n, k // 64])) * int(q[n, k]) + Fraction(float(b[n, k // 64]))
            got = Fraction(float(w16[n, k]))
            lo = Fraction(float(np.nextafter(w16[n, k], np.float16(-np.inf))))
            hi = Fraction(float(np.nextafter(w16[n, k], np.float16(np.inf))))
            assert abs(got - exact) <= abs(lo - exact) and abs(got - exact) <= abs(hi - exact)


def test_dequant_bf16_is_bf16_of_f32_dequant():
    rng = _rng(5)
    _, codes, s, b = _random_layer(rng, 1, 128, 32)
    w32 = O.dequant_f32(codes, s, b)
    lib = torch.from_numpy(w32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.dequant_bf16(codes, s, b), lib)


# ---------------------------------------------------------------- forward

@pytest.mark.parametrize("M,K,N", [(1, 64, 8), (3, 128, 16), (16, 256, 40), (5, 192, 64)])
def test_forward_equals_triple_loop(M, K, N):
    rng = _rng(M * 1000 + K + N)
    x, codes, s, b = _random_layer(rng, M, K, N)
    y = O.forward_ref(x, codes, s, b)
    yt = O.forward_triple_loop(x, codes, s, b)
    xa = np.abs(O.decode_bf16(x))
    wa = np.abs(O.dequant_f32(codes, s, b).astype(np.float64))
    bound = 1e-14 * (xa @ wa.T) + 1e-300
    assert np.all(np.abs(y - yt) <= bound)


def test_forward_constant_codes_closed_form():
    """All codes c, scale 1, bias 0 -> y[m][n] = c * sum_k x[m][k]."""
    rng = _rng(6)
    M, K, N = 4, 192, 16
    x = _random_layer(rng, M, K, N)[0]
    for c in (0, 1, 7, 15):
        codes = O.pack_codes(np.full((N, K), c))
        s = np.ones((N, K // 64), dtype=np.float16)
        b = np.zeros((N, K // 64), dtype=np.float16)
        y = O.forward_ref(x, codes, s, b)
        xs = O.decode_bf16(x).sum(axis=1)
        assert np.allclose(y, (c * xs)[:, None], rtol=1e-13, atol=1e-13)


def test_forward_constant_codes_per_group_affine():
    """Constant codes c per group with scale s_g, bias b_g -> y = sum_g (s_g*c + b_g) * sum_{k in g} x_k."""
    rng = _rng(7)
    M, K, N = 3, 256, 8
    x = _random_layer(rng, M, K, N)[0]
    s = np.array(rng.uniform(0.01, 0.1, (N, 4)), dtype=np.float16)
    b = np.array(rng.uniform(-0.5, 0.5, (N, 4)), dtype=np.float16)
    c = 11
    codes = O.pack_codes(np.full((N, K), c))
    y = O.forward_ref(x, codes, s, b)
    xs = O.decode_bf16(x).reshape(M, 4, 64).sum(axis=2)        # [M][G]
    w_g = s.astype(np.float64) * c + b.astype(np.float64)      # [N][G]
    expect = xs @ w_g.T
    assert np.allclose(y, expect, rtol=1e-12, atol=1e-12)


def test_forward_one_hot_selects_weight_column():
    """x = e_k -> y[:, n] = w(n, k) exactly, and its bf16 rounding is the bf16 dequant."""
    rng = _rng(8)
    K, N = 128, 24
    _, codes, s, b = _random_layer(rng, 1, K, N)
    one = np.uint16(0x3F80)     # bf16 1.0
    x = np.zeros((K, K), dtype=np.uint16)
    x[np.arange(K), np.arange(K)] = one
    y = O.forward_ref(x, codes, s, b)
    w32 = O.dequant_f32(codes, s, b)
    assert np.array_equal(y, w32.T.astype(np.float64))
    assert np.array_equal(O.round_bf16(y), O.dequant_bf16(codes, s, b).T)


def test_forward_power_of_two_linearity_exact():
    rng = _rng(9)
    x, codes, s, b = _random_layer(rng, 4, 128, 16)
    x2 = (x.astype(np.uint32) + (1 << 7)).astype(np.uint16)     # exponent + 1 -> 2x (no overflow here)
    y1 = O.forward_ref(x, codes, s, b)
    y2 = O.forward_ref(x2, codes, s, b)
    assert np.array_equal(y2, 2.0 * y1)


def test_forward_transposed_operand_would_fail():
    """A non-square case distinguishes W from W^T: the brute-force loop indexes W[n][k] explicitly."""
    rng = _rng(10)
    x, codes, s, b = _random_layer(rng, 2, 64, 8)
    y = O.forward_ref(x, codes, s, b)
    assert y.shape == (2, 8)
    w = O.dequant_f32(codes, s, b).astype(np.float64)
    assert np.allclose(y[1, 3], np.dot(O.decode_bf16(x)[1], w[3]), rtol=1e-14)


# ---------------------------------------------------------------- tolerance

def test_half_ulp_bf16_values():
    assert O.half_ulp_bf16(1.0) == 2.0 ** -8
    assert O.half_ulp_bf16(1.99) == 2.0 ** -8
    assert O.half_ulp_bf16(2.0) == 2.0 ** -7
    assert O.half_ulp_bf16(-0.75) == 2.0 ** -9


def test_tolerance_metrics_basic():
    y_ref = np.array([1.0, -2.0, 3.0, 0.5])
    t = O.tolerance(y_ref, y_ref)
    assert t["relF"] == 0 and t["max_gate"] == 0 and t["ok"]
    # exact result rounded to bf16 is always within the half-ulp allowance
    rng = _rng(11)
    r = rng.standard_normal(10000) * 3
    yb = O.decode_bf16(O.round_bf16(r))
    t = O.tolerance(yb, r)
    assert t["max_gate"] == 0.0 and t["ok"]
    bad = r * (1 + 1e-2)
    assert not O.tolerance(bad, r)["ok"]


# ---------------------------------------------------------------- RTN pack

def _rtn_case(seed, N=16, K=256):
    rng = _rng(seed)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    return w


def test_rtn_codes_are_nearest_grid_point():
    """Brute force over the 16 grid points: each RTN code is (one of) the nearest."""
    w = _rtn_case(12)
    codes, s, b = O.pack_rtn(w)
    N, K = w.shape
    q = O.unpack_codes(codes, K)
    sf = s.astype(np.float64)
    bf = b.astype(np.float64)
    for n in range(N):
        for k in range(K):
            g = k // 64
            grid = sf[n, g] * np.arange(16) + bf[n, g]
            d = np.abs(grid - float(w[n, k]))
            assert d[q[n, k]] <= d.min() + 4e-7 * max(abs(float(w[n, k])), 1e-3)


def test_rtn_reconstructs_group_extremes():
    """Reading R3 bounds: deq(code of min) within half an f16 ulp of min; max within 15*ulp(s)/2 + ulp(min)/2."""
    w = _rtn_case(13, N=32, K=512)
    codes, s, b = O.pack_rtn(w)
    deq = O.dequant_f32(codes, s, b).astype(np.float64).reshape(32, 8, 64)
    g = w.astype(np.float64).reshape(32, 8, 64)

    def half_ulp_f16(v):
        _, e = np.frexp(np.abs(v))
        return np.ldexp(1.0, np.maximum(e, -13) - 12)

    i_min = g.argmin(-1)
    i_max = g.argmax(-1)
    mn = np.take_along_axis(g, i_min[..., None], -1)[..., 0]
    mx = np.take_along_axis(g, i_max[..., None], -1)[..., 0]
    d_min = np.take_along_axis(deq, i_min[..., None], -1)[..., 0]
    d_max = np.take_along_axis(deq, i_max[..., None], -1)[..., 0]
    eps = 2.0 ** -23 * np.maximum(np.abs(mn), np.abs(mx))
    sf = s.astype(np.float64)
    assert np.all(np.abs(d_min - mn) <= half_ulp_f16(mn) + eps)
    assert np.all(np.abs(d_max - mx) <= 15 * half_ulp_f16(sf) + half_ulp_f16(mn) + eps)


def test_rtn_constant_group():
    w = np.full((2, 128), 0.3, dtype=np.float32)
    w[1, 64:] = -1.25
    codes, s, b = O.pack_rtn(w)
    assert np.all(O.unpack_codes(codes, 128) == 0)
    assert np.all(s == 0)
    assert np.array_equal(O.dequant_f32(codes, s, b), np.repeat(b.astype(np.float32), 64, axis=1))


def test_rtn_monotone_code_map():
    w = _rtn_case(14, N=8, K=128)
    codes, s, b = O.pack_rtn(w)
    q = O.unpack_codes(codes, 128).reshape(8, 2, 64)
    g = w.reshape(8, 2, 64)
    for n in range(8):
        for j in range(2):
            order = np.argsort(g[n, j], kind="stable")
            assert np.all(np.diff(q[n, j][order]) >= 0)


def test_rtn_on_grid_group_is_exact():
    """A group that already lies on an f16 affine grid spanning codes 0..15 is reproduced exactly."""
    s = np.float16(0.0078125 * 1.25)
    b = np.float16(-0.0625)
    q = np.tile(np.arange(16), 4)
    w = (np.float64(s) * q + np.float64(b)).astype(np.float32)[None, :]
    codes, s2, b2 = O.pack_rtn(w)
    assert s2[0, 0] == s and b2[0, 0] == b
    assert np.array_equal(O.unpack_codes(codes, 64)[0], q)


def test_rtn_rejects_non_finite_and_out_of_range():
    w = np.zeros((1, 64), dtype=np.float32)
    w[0, 3] = np.nan
    with pytest.raises(ValueError):
        O.pack_rtn(w)
    w[0, 3] = 70000.0
    with pytest.raises(ValueError):
        O.pack_rtn(w)


# ---------------------------------------------------------------- imatrix fit

def test_fit_never_worse_than_rtn_per_group():
    """The pages: RTN is candidate 0 of the search, so the fit is never worse by the weighted objective."""
    rng = _rng(15)
    N, K = 48, 512
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = torch.from_numpy((rng.standard_normal((64, K)) * np.exp(rng.standard_normal(K))).astype(np.float32))
    xb = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    imp = O.imatrix_from_x(xb)
    cf, sf, bf = O.pack_imatrix(w, imp)
    cr, sr, br = O.pack_rtn(w)
    impr = imp + 1e-6 * imp.mean()
    ef = O.group_weighted_error(w, cf, sf, bf, impr)
    er = O.group_weighted_error(w, cr, sr, br, impr)
    assert np.all(ef <= er)
    assert ef.sum() < er.sum()          # the search does find better triples on Gaussian weights


def test_fit_without_statistics_is_rtn():
    w = _rtn_case(16)
    a = O.pack_imatrix(w, None)
    r = O.pack_rtn(w)
    for u, v in zip(a, r):
        assert np.array_equal(u, v)


def test_fit_on_grid_group_has_zero_error():
    s = np.float16(0.01)
    b = np.float16(-0.07)
    q = np.tile(np.arange(16), 4)
    w = (np.float64(s) * q + np.float64(b)).astype(np.float32)[None, :]
    imp = np.linspace(0.1, 3.0, 64)
    c, s2, b2 = O.pack_imatrix(w, imp)
    assert O.group_weighted_error(w, c, s2, b2, imp).max() == 0.0


def test_ls_refit_matches_library_least_squares():
    """The refit step solves the E[x^2]-weighted least squares of w ~ s*q + b for fixed codes: it agrees
    with numpy's lstsq on sqrt(imp)-scaled [q, 1] columns to float64 rounding, on random groups with
    random codes and log-normal importances (aimarketly "Ideogram-4-IQ4_M", "What IQ4 means here")."""
    rng = _rng(31)
    n, G = 6, 5
    g64 = rng.standard_normal((n, G, 64)) * 0.02
    q = rng.integers(0, 16, size=(n, G, 64))
    imp_g = np.exp(rng.standard_normal((1, G, 64)) * 2.0)
    sw = (imp_g * np.ones_like(g64)).sum(-1)
    swx = (imp_g * g64).sum(-1)
    s_ls, b_ls, solvable = O.weighted_ls_affine(g64, imp_g, q, sw, swx)
    assert solvable.all()
    for i in range(n):
        for g in range(G):
            r = np.sqrt(imp_g[0, g])
            A = np.stack([q[i, g] * r, r], axis=1)
            (s_ref, b_ref), *_ = np.linalg.lstsq(A, g64[i, g] * r, rcond=None)
            assert abs(s_ls[i, g] - s_ref) <= 1e-9 * abs(s_ref)
            assert abs(b_ls[i, g] - b_ref) <= 1e-9 * max(abs(b_ref), abs(s_ref))
    # all codes equal: the system is singular and flagged so
    _, _, solvable = O.weighted_ls_affine(g64[:1, :1], imp_g[:, :1], np.full((1, 1, 64), 7), sw[:1, :1], swx[:1, :1])
    assert not solvable.any()


def test_fit_refit_reaches_the_weighted_optimum():
    """A group whose heavily weighted channels lie on an f16 affine grid (s*, b*) while unweighted outliers
    set its min and max: RTN and every range-shrink candidate miss that grid, and only a refit of the
    candidate whose step equals s* recovers it.  The fit must land on the best triple that reproduces the
    weighted channels exactly, i.e. the f16 closed-form optimum, reaching its error."""
    s_star, b_star = 2.0 ** -7, -6.5 * 2.0 ** -7
    q_imp = np.array([0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 3, 7, 1, 5, 8, 2])
    w = np.zeros(64)
    w[:16] = s_star * q_imp + b_star
    w[16:] = np.linspace(b_star - 8 * s_star, b_star + 13.4286 * s_star, 48)   # range 21.4286 s*: step s* at shrink 0.3
    imp = np.zeros(64)
    imp[:16] = 100.0
    w32 = w.astype(np.float32)[None, :]
    c, s, b = O.pack_imatrix(w32, imp)
    impr = imp + 1e-6 * imp.mean()
    e_fit = O.group_weighted_error(w32, c, s, b, impr)[0, 0]
    # closed form: the triples (s*, b* - k s*) reproduce the weighted channels exactly for every shift k
    # that keeps their codes in range; the best of them is the weighted optimum up to the outliers' share
    best = np.inf
    for k in range(0, 16 - q_imp.max()):
        s16 = np.array([[s_star]], dtype=np.float16)
        b16 = np.array([[b_star - k * s_star]], dtype=np.float16)
        qk = np.clip(np.rint((w - (b_star - k * s_star)) / s_star), 0, 15).astype(np.int64)
        best = min(best, O.group_weighted_error(w32, O.pack_codes(qk[None, :]), s16, b16, impr)[0, 0])
    assert float(s[0, 0]) == s_star
    assert np.array_equal(O.dequant_f32(c, s, b)[0, :16], w32[0, :16])
    assert e_fit <= best * (1 + 1e-12)
    cr, sr, br = O.pack_rtn(w32)
    assert O.group_weighted_error(w32, cr, sr, br, impr)[0, 0] > 1e4 * e_fit


def test_imatrix_is_mean_square():
    x = np.array([[0x3F80, 0x4000], [0xBF80, 0x0000]], dtype=np.uint16)   # [[1, 2], [-1, 0]]
    assert np.array_equal(O.imatrix_from_x(x), np.array([1.0, 2.0]))


# ---------------------------------------------------------------- W8 g64 (reading R9)

def _w8_layer(rng, M, K, N):
    codes = rng.integers(0, 1 << 32, size=(N, K // 4), dtype=np.uint32)
    s = np.exp(rng.uniform(np.log(1e-4), np.log(2e-3), size=(N, K // 64))).astype(np.float16)
    b = (-127.5 * s.astype(np.float64) + 0.1 * s.astype(np.float64) * rng.standard_normal(s.shape)).astype(np.float16)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16), codes, s, b


def test_w8_byte_order_low_first():
    assert list(O.unpack_codes8(np.array([[0x04030201]], dtype=np.uint32), 4)[0]) == [1, 2, 3, 4]
    assert O.pack_codes8(np.array([[1, 2, 3, 4]]))[0, 0] == 0x04030201


def test_w8_pack_unpack_roundtrip():
    q = _rng(40).integers(0, 256, size=(5, 192))
    assert np.array_equal(O.unpack_codes8(O.pack_codes8(q), 192), q)


def test_w8_bits_per_weight_is_8_5_golden():
    """8-bit codes plus the pages' '+0.5' group overhead (one f16 scale and bias per 64)."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "format_constants.json")))
    K = 4608
    w = np.zeros((1, K), dtype=np.float32)
    codes, s, b = O.pack8_rtn(w)
    bits = 8 * (codes.nbytes + s.nbytes + b.nbytes)
    assert bits == (g["q8_code_bits"]["value"] + g["overhead_bits_per_weight"]["value"]) * K


def test_w8_dequant_exact_equals_rational_arithmetic():
    """All 256 codes x edge f16 values as scale and as bias."""
    edges = np.array([0.0, -0.0, 2.0 ** -24, 6.1e-5, 1.0, -1.0, 0.0078125, 3.140625, 65504.0, -65504.0,
                      1e-3, -7.5e-3, 2.0 ** -14, 0.5, -2.0, 1024.0], dtype=np.float16)
    q = np.arange(256)
    for sv in edges:
        for bv in edges:
            for part in range(4):
                qq = q[64 * part: 64 * part + 64]
                codes = O.pack_codes8(qq[None, :])
                got = O.dequant8_exact(codes, np.array([[sv]]), np.array([[bv]]))[0]
                for j in range(64):
                    exact = Fraction(float(sv)) * int(qq[j]) + Fraction(float(bv))
                    assert Fraction(float(got[j])) == exact


def test_w8_dequant_f32_is_correctly_rounded():
    rng = _rng(41)
    _, codes, s, b = _w8_layer(rng, 1, 256, 48)
    w32 = O.dequant8_f32(codes, s, b)
    q = O.unpack_codes8(codes, 256)
    for n in range(0, 48, 5):
        for k in range(0, 256, 7):
            exact = Fraction(float(s[n, k // 64])) * int(q[n, k]) + Fraction(float(b[n, k // 64]))
            got = Fraction(float(w32[n, k]))
            lo = Fraction(float(np.nextafter(w32[n, k], np.float32(-np.inf))))
            hi = Fraction(float(np.nextafter(w32[n, k], np.float32(np.inf))))
            assert abs(got - exact) <= abs(lo - exact) and abs(got - exact) <= abs(hi - exact)


def test_w8_dequant_f16_is_correctly_rounded():
    """f16 operand of 8-bit codes = binary16 nearest to the exact rational s*q + b."""
    _, codes, s, b = _w8_layer(_rng(47), 1, 128, 24)
    w16 = O.dequant8_f16(codes, s, b)
    q = O.unpack_codes8(codes, 128)
    for n in range(24):
        for k in range(0, 128, 3):
            exact = Fraction(float(s[n, k // 64])) * int(q[n, k]) + Fraction(float(b[n, k // 64]))
            got = Fraction(float(w16[n, k]))
            lo = Fraction(float(np.nextafter(w16[n, k], np.float16(-np.inf))))
            hi = Fraction(float(np.nextafter(w16[n, k], np.float16(np.inf))))
            assert abs(got - exact) <= abs(lo - exact) and abs(got - exact) <= abs(hi - exact)


def test_w8_forward_rows_equals_full_forward():
    x, codes, s, b = _w8_layer(_rng(48), 9, 192, 16)
    rows = np.array([0, 4, 8])
    assert np.array_equal(O.forward8_rows(x, codes, s, b, rows), O.forward8_ref(x, codes, s, b)[rows])


def test_w8_dequant_bf16_is_bf16_of_f32_dequant():
    _, codes, s, b = _w8_layer(_rng(42), 1, 128, 16)
    w32 = O.dequant8_f32(codes, s, b)
    lib = torch.from_numpy(w32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.dequant8_bf16(codes, s, b), lib)


@pytest.mark.parametrize("M,K,N", [(3, 64, 5), (2, 192, 7)])
def test_w8_forward_equals_triple_loop(M, K, N):
    """Pure-Python triple loop with exactly rounded sums (math.fsum) against the float64 matrix product."""
    import math
    x, codes, s, b = _w8_layer(_rng(43 + M + K + N), M, K, N)
    y = O.forward8_ref(x, codes, s, b)
    xf = O.decode_bf16(x)
    q = O.unpack_codes8(codes, K)
    for m in range(M):
        for n in range(N):
            terms = []
            for k in range(K):
                wv = float(np.float32(float(s[n, k // 64]) * int(q[n, k]) + float(b[n, k // 64])))
                terms.append(float(xf[m, k]) * wv)
            ref = math.fsum(terms)
            bound = 1e-14 * math.fsum(abs(t) for t in terms) + 1e-300
            assert abs(y[m, n] - ref) <= bound


def _w8_rtn_case(seed, N=16, K=256):
    rng = _rng(seed)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, :64] *= 100.0
    w[1, 64:128] = np.abs(w[1, 64:128]) + 1.0
    return w


def test_w8_rtn_codes_are_nearest_grid_point():
    """Brute force over the 256 grid points: each RTN code is (one of) the nearest."""
    w = _w8_rtn_case(44)
    codes, s, b = O.pack8_rtn(w)
    N, K = w.shape
    q = O.unpack_codes8(codes, K)
    sf = s.astype(np.float64)
    bf = b.astype(np.float64)
    for n in range(N):
        for k in range(K):
            g = k // 64
            grid = sf[n, g] * np.arange(256) + bf[n, g]
            d = np.abs(grid - float(w[n, k]))
            assert d[q[n, k]] <= d.min() + 4e-7 * max(abs(float(w[n, k])), 1e-3)


def test_w8_rtn_reconstructs_group_extremes():
    """R9 bounds: deq(code of min) within half an f16 ulp of min; max within 255*ulp(s)/2 + ulp(min)/2."""
    w = _w8_rtn_case(45, N=24, K=512)
    codes, s, b = O.pack8_rtn(w)
    deq = O.dequant8_f32(codes, s, b).astype(np.float64).reshape(24, 8, 64)
    g = w.astype(np.float64).reshape(24, 8, 64)

    def half_ulp_f16(v):
        _, e = np.frexp(np.abs(v))
        return np.ldexp(1.0, np.maximum(e, -13) - 12)

    i_min, i_max = g.argmin(-1), g.argmax(-1)
    mn = np.take_along_axis(g, i_min[..., None], -1)[..., 0]
    mx = np.take_along_axis(g, i_max[..., None], -1)[..., 0]
    d_min = np.take_along_axis(deq, i_min[..., None], -1)[..., 0]
    d_max = np.take_along_axis(deq, i_max[..., None], -1)[..., 0]
    eps = 2.0 ** -23 * np.maximum(np.abs(mn), np.abs(mx))
    assert np.all(np.abs(d_min - mn) <= half_ulp_f16(mn) + eps)
    assert np.all(np.abs(d_max - mx) <= 255 * half_ulp_f16(s.astype(np.float64)) + half_ulp_f16(mn) + eps)


def test_w8_rtn_constant_group_and_monotone_codes():
    w = np.full((2, 128), -0.7, dtype=np.float32)
    codes, s, b = O.pack8_rtn(w)
    assert np.all(O.unpack_codes8(codes, 128) == 0) and np.all(s == 0)
    w = _w8_rtn_case(46, N=6, K=128)
    q = O.unpack_codes8(O.pack8_rtn(w)[0], 128).reshape(6, 2, 64)
    g = w.reshape(6, 2, 64)
    for n in range(6):
        for j in range(2):
            order = np.argsort(g[n, j], kind="stable")
            assert np.all(np.diff(q[n, j][order]) >= 0)


def test_w8_rtn_on_grid_group_is_exact():
    """A group on an f16 affine grid that uses codes 0 and 255 is reproduced exactly."""
    s = np.float16(2.0 ** -10)
    b = np.float16(-0.125)
    q = np.concatenate([[0, 255], np.arange(1, 255, 4)[:62]])
    w = (np.float64(s) * q + np.float64(b)).astype(np.float32)[None, :]
    codes, s2, b2 = O.pack8_rtn(w)
    assert s2[0, 0] == s and b2[0, 0] == b
    assert np.array_equal(O.unpack_codes8(codes, 64)[0], q)


def test_w8_and_w4_agree_on_a_shared_grid():
    """Weights whose 64-groups use only the 16 levels b + 17 s' q (q <= 15) of an 8-bit grid with step
    s' = s/17: the W4 and W8 packs dequantize to the same values."""
    s4 = np.float16(0.0078125 * 1.0625 * 17)           # 17 * s8, exact in f16
    s8 = np.float16(np.float64(s4) / 17)
    assert np.float64(s8) * 17 == np.float64(s4)
    b = np.float16(-0.0625)
    q4 = np.tile(np.arange(16), 4)
    w = (np.float64(s4) * q4 + np.float64(b)).astype(np.float32)[None, :]
    d4 = O.dequant_f32(*O.pack_rtn(w))
    d8 = O.dequant8_f32(*O.pack8_rtn(w))
    assert np.array_equal(d4, d8)


# ---------------------------------------------------------------- SwiGLU pair (readings R10, R11)

def test_silu_matches_library_sigmoid():
    """silu(z) = z * expit(z), expit being scipy's logistic sigmoid (a library routine)."""
    from scipy.special import expit
    z = np.concatenate([np.linspace(-50, 50, 20001), [0.0, -0.0, 1e-300, -1e-300, 700.0, -700.0, 745.0, -745.0,
                                                      800.0, -800.0]])
    ours = O.silu(z)
    lib = z * expit(z)
    assert np.all(np.abs(ours - lib) <= 4 * np.spacing(np.abs(lib)) + 1e-320)
    assert O.silu(np.array([-800.0]))[0] == 0.0 and O.silu(np.array([800.0]))[0] == 800.0


def test_silu_slope_bound_is_tight():
    """The constant R11 uses: max silu' = sigma(z)(1 + z(1 - sigma(z))) <= 1.1, attained near 1.0998."""
    from scipy.special import expit
    z = np.linspace(-40, 40, 800001)
    sg = expit(z)
    d = sg * (1 + z * (1 - sg))
    assert d.max() <= O.SILU_SLOPE_MAX and d.max() > 1.0998 and d.min() > -0.1


def test_swiglu_equals_brute_force():
    """Pure-Python h[m][n] = silu(sum_k x w_g) * sum_k x w_u with exactly rounded sums and math.exp."""
    import math
    rng = _rng(60)
    x, cg, sg, bg = _random_layer(rng, 3, 128, 5)
    _, cu, su, bu = _random_layer(rng, 3, 128, 5)
    h = O.swiglu_ref(x, (cg, sg, bg), (cu, su, bu))
    xf = O.decode_bf16(x)
    wg = O.dequant_f32(cg, sg, bg).astype(np.float64)
    wu = O.dequant_f32(cu, su, bu).astype(np.float64)
    for m in range(3):
        for n in range(5):
            g = math.fsum(float(xf[m, k]) * float(wg[n, k]) for k in range(128))
            u = math.fsum(float(xf[m, k]) * float(wu[n, k]) for k in range(128))
            ref = g / (1.0 + math.exp(-g)) * u
            assert abs(h[m, n] - ref) <= 1e-12 * (abs(ref) + 1e-6)


def test_swiglu_one_hot_selects_weights():
    """x = e_k: g = w_g(n, k) and u = w_u(n, k) exactly, so h = w_g * expit(w_g) * w_u (scipy's sigmoid)."""
    from scipy.special import expit
    rng = _rng(61)
    _, cg, sg, bg = _random_layer(rng, 1, 192, 24)
    _, cu, su, bu = _random_layer(rng, 1, 192, 24)
    ks = np.array([0, 5, 63, 64, 130, 191])
    x = np.zeros((ks.size, 192), dtype=np.uint16)
    x[np.arange(ks.size), ks] = 0x3F80
    h = O.swiglu_ref(x, (cg, sg, bg), (cu, su, bu))
    wg = O.dequant_f32(cg, sg, bg).astype(np.float64)[:, ks].T
    wu = O.dequant_f32(cu, su, bu).astype(np.float64)[:, ks].T
    ref = wg * expit(wg) * wu
    assert np.all(np.abs(h - ref) <= 4 * np.spacing(np.abs(ref)) + 1e-300)


def test_swiglu_negated_up_weight_negates_output():
    """(s, b) -> (-s, -b) negates every up weight exactly, hence u and h exactly."""
    rng = _rng(62)
    x, cg, sg, bg = _random_layer(rng, 4, 256, 8)
    _, cu, su, bu = _random_layer(rng, 4, 256, 8)
    h = O.swiglu_ref(x, (cg, sg, bg), (cu, su, bu))
    hn = O.swiglu_ref(x, (cg, sg, bg), (cu, -su, -bu))
    assert np.array_equal(hn, -h)


def test_swiglu_tolerance_gates():
    """R11's gate: the reference rounded to bf16 passes; an error of twice the bound, or a relF above 8e-3, fails."""
    rng = _rng(63)
    x, cg, sg, bg = _random_layer(rng, 6, 256, 16)
    _, cu, su, bu = _random_layer(rng, 6, 256, 16)
    g, u = O.swiglu_linears(x, (cg, sg, bg), (cu, su, bu))
    h_ref = O.silu(g) * u
    h_bf16 = O.decode_bf16(O.round_bf16(h_ref))
    assert O.swiglu_tolerance(h_bf16, g, u)["ok"]
    d_g = 1.5e-2 * np.sqrt(np.mean(g * g))
    d_u = 1.5e-2 * np.sqrt(np.mean(u * u))
    bound = 1.1 * d_g * (abs(u[2, 3]) + d_u) + abs(O.silu(g[2, 3])) * d_u
    bad = h_ref.copy()
    bad[2, 3] += 2 * bound + 2 * abs(h_ref[2, 3])
    t = O.swiglu_tolerance(bad, g, u, bf16_output=False)
    assert not t["ok"] and t["max_ratio"] > 1.0
    assert not O.swiglu_tolerance(h_ref * 1.01, g, u, bf16_output=False)["ok"]     # relF = 1e-2


def test_pack_sizes_on_the_pages_fix_the_half_bit_overhead_of_both_widths():
    """The pages' disk sizes (bf16 ~50 GB, Q4 ~14 GB, Q8 ~27 GB, each rounded to the GB) agree with
    4 + 0.5 and 8 + 0.5 bits per weight (R1, R9): 50 GB of bf16 is 25e9 +- 0.25e9 weights, and both packed
    sizes fall within their rounding.  Nearby overheads for the 8-bit pack (8.25 or 9 bits per weight) do not."""
    g = json.load(open(os.path.join(GOLDEN, "format_constants.json")))
    snap, q4, q8 = g["bf16_snapshot_gb"]["value"], g["q4_pack_gb"]["value"], g["q8_pack_gb"]["value"]
    n_lo, n_hi = (snap - 0.5) * 1e9 / 2, (snap + 0.5) * 1e9 / 2          # weights, from bf16 bytes

    def fits(bits, size_gb):
        lo, hi = n_lo * bits / 8 / 1e9, n_hi * bits / 8 / 1e9
        return hi >= size_gb - 0.5 and lo <= size_gb + 0.5

    four = g["code_bits"]["value"] + g["overhead_bits_per_weight"]["value"]
    eight = g["q8_code_bits"]["value"] + g["overhead_bits_per_weight"]["value"]
    assert (four, eight) == (4.5, 8.5)
    assert fits(four, q4) and fits(eight, q8)
    assert not fits(8.25, q8) and not fits(9.0, q8)


def test_w8_rtn_rejects_non_finite_and_out_of_range():
    """Like the 4-bit pack: NaN, infinities and magnitudes beyond the f16 range have no scale and bias."""
    for bad in (np.nan, np.inf, -np.inf, 70000.0):
        w = np.zeros((2, 64), dtype=np.float32)
        w[1, 7] = bad
        with pytest.raises(ValueError):
            O.pack8_rtn(w)
    w = np.zeros((1, 64), dtype=np.float32)
    w[0, 0] = 65504.0                            # the f16 maximum itself is packable
    codes, s, b = O.pack8_rtn(w)
    assert np.all(np.isfinite(O.dequant8_f32(codes, s, b)))
