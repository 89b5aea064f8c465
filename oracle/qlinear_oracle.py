"""CPU oracle for the group-wise affine W4 g64 quantized linear layer.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline leg use this module.  The library's product path never imports, calls
or links it, and it shares no code with the CUDA sources: it decodes the packed
format, dequantizes, multiplies and quantizes with its own plain numpy code.

What the layer computes, and where the pages say it:
  * Format: 4-bit codes; every 64 consecutive weights along the input
    dimension share one f16 scale and one f16 bias, which is the "+0.5 bit"
    overhead on top of the 4-bit width (aimarketly "Ideogram-4-IQ4_M", intro;
    huggingface "SceneWorks/ideogram-4-mlx", Versions: group-wise affine,
    group size 64).
  * Dequantization is the uniform affine grid w = scale * q + bias, the grid
    the MLX quantized matmul reads (aimarketly "Ideogram-4-IQ4_M", "What IQ4
    means here").
  * The layer is y = x . W^T with bf16 activations, fp32 accumulation and bf16
    output; here the product is formed in float64 from the fp32 dequantized
    weights, the reference the CUDA path is measured against.
  * Quantization: MLX's min/max round-to-nearest (RTN) solution, and an
    importance-weighted least-squares fit searched with RTN as candidate 0, so
    the fit is never worse than RTN on sum_j E[x_j^2] * dW_j^2 (aimarketly
    "Ideogram-4-IQ4_M", "What IQ4 means here"); weights with no activation
    statistics fall back to RTN (same page, "How the statistics were
    collected").  The packer is deterministic ("byte-equivalent to load-time
    quantization", huggingface "SceneWorks/ideogram-4-mlx", Provenance).

Readings adopted where the pages are silent (each is also listed in the design
notes of the repository):
  R1 layout: W is [N][K] (a PyTorch Linear weight); codes are uint32 [N][K/8]
     with code (n, k) = (codes[n][k/8] >> 4*(k%8)) & 0xF (low nibble first);
     scales and biases are f16 [N][K/64].
  R2 "fp32 dequant" is the correctly rounded binary32 value of the exact
     s*q + b.
  R3 RTN: per group of 64 fp32 weights, s = RN32(RN32(max - min) / 15),
     scale = RN_f16(s), bias = RN_f16(min) (no zero snapping), and
     q = clamp(round_half_even(RN32(RN32(w - bias) / scale)), 0, 15), q = 0
     when scale == 0; codes are computed from the stored f16 parameters.
  R4 imatrix fit: candidate grid, refits and the regularisation of
     unobserved channels as documented on pack_imatrix().
  R5 tolerance: bf16 output is gated on relative Frobenius error <= 4e-3 and
     on max_i(|y_i - y_ref_i| - half_ulp_bf16(max(|y_i|, |y_ref_i|)))^+ <=
     1.5e-2 * rms(y_ref); the literal max error is reported beside it.
  R9 W8 g64, the 8-bit width the pages keep for the modulation and
     conditioning projections (aimarketly "Ideogram-4-IQ4_M", Conversion) and
     ship as a Q8 pack (huggingface "SceneWorks/ideogram-4-mlx", Versions):
     codes are uint32 [N][K/4] with code (n, k) = (codes[n][k/4] >> 8*(k%4)) &
     0xFF (low byte first), q in [0, 255]; scales and biases as in R1, so a
     weight costs 8 + 0.5 bits (the same "+0.5" overhead); RTN as R3 with 255
     levels in place of 15.
  R10 SwiGLU up/gate pair: the DiT block's MLP is a SwiGLU of three Linears
     with intermediate size 12288 (jimmysue "Ideogram 4" notes, sec. 2.1
     block diagram and sec. 2.8 spec table); the pages print no formula, so
     the plain one: h = silu(x . W_gate^T) * (x . W_up^T) elementwise, with
     silu(z) = z / (1 + exp(-z)); gate and up are two packed [I][K] weights of
     the same format, and h is rounded once to bf16.
  R11 tolerance of h: each linear output may err by R5's per-element allowance
     d = 1.5e-2 * rms of that output; since |silu'| <= 1.1 everywhere, the mean
     value theorem gives |dh| <= 1.1 * d_g * (|u| + d_u) + |silu(g)| * d_u per
     element (plus half a bf16 ulp of h), and relative Frobenius error <= 8e-3
     (two factors, each within R5's 4e-3).

Parity status: the imatrix fit (pack_imatrix) is a search heuristic with no
printed reference values.  Its invariants are pinned ("never worse than RTN"
per group, exact recovery of on-grid groups), its least-squares refit is
pinned to numpy's lstsq, and a group that only a refit can fit exactly pins
the search to the weighted closed-form optimum.  Everything else is pinned to
closed forms, library conversions or brute force by the CPU tests.
"""
from __future__ import annotations

import struct

import numpy as np

GROUP = 64
F16_MAX = 65504.0


# --------------------------------------------------------------------------
# Format decoding (R1)
# --------------------------------------------------------------------------

def decode_f16(bits) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64, from the sign/exponent/fraction fields."""
    b = np.asarray(bits).astype(np.uint16).astype(np.int64)
    sign = np.where((b >> 15) & 1, -1.0, 1.0)
    e = (b >> 10) & 0x1F
    f = (b & 0x3FF).astype(np.float64)
    normal = np.ldexp(1024.0 + f, (e - 25).astype(np.int32))      # (1 + f/2^10) * 2^(e-15)
    subnormal = np.ldexp(f, -24)                                  # f/2^10 * 2^-14
    special = np.where(f == 0, np.inf, np.nan)
    mag = np.where(e == 0, subnormal, np.where(e == 31, special, normal))
    return sign * mag


def f16_array_bits(a) -> np.ndarray:
    """Bit patterns of an f16 array (a view; no conversion)."""
    return np.ascontiguousarray(a).view(np.uint16)


def decode_bf16(bits) -> np.ndarray:
    """bf16 bit patterns -> float64: a bf16 value is the upper half of a binary32."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def unpack_codes(codes, K: int) -> np.ndarray:
    """uint32 [N][K/8] -> int64 codes q [N][K], code k%8 in bits 4*(k%8) .. 4*(k%8)+3."""
    c = np.asarray(codes, dtype=np.uint32).astype(np.int64)
    N = c.shape[0]
    assert c.shape[1] * 8 == K
    shifts = 4 * np.arange(8, dtype=np.int64)
    q = (c[:, :, None] >> shifts[None, None, :]) & 0xF
    return q.reshape(N, K)


def pack_codes(q) -> np.ndarray:
    """int codes [N][K] in [0, 15] -> uint32 [N][K/8], low nibble first."""
    q = np.asarray(q, dtype=np.uint64)
    N, K = q.shape
    assert K % 8 == 0 and q.max(initial=0) <= 15
    shifts = 4 * np.arange(8, dtype=np.uint64)
    words = (q.reshape(N, K // 8, 8) << shifts[None, None, :]).sum(axis=-1)
    return words.astype(np.uint32)


# --------------------------------------------------------------------------
# Dequantization (R2)
# --------------------------------------------------------------------------

def dequant_exact(codes, scales, biases) -> np.ndarray:
    """Exact w = s*q + b as float64 [N][K].

    Exact because s and b are f16 values, i.e. integer multiples of 2^-24 below
    2^16, and q <= 15: s*q + b = i * 2^-24 with |i| < 2^45, which float64 holds
    without rounding (both the product and the sum are exact).
    """
    N, G = np.shape(scales)
    K = G * GROUP
    q = unpack_codes(codes, K).astype(np.float64)
    s = np.repeat(decode_f16(f16_array_bits(scales)), GROUP, axis=1)
    b = np.repeat(decode_f16(f16_array_bits(biases)), GROUP, axis=1)
    return s * q + b


def dequant_f32(codes, scales, biases) -> np.ndarray:
    """fp32 dequant: RN_fp32 of the exact value (numpy's float64->float32 cast rounds to nearest even)."""
    return dequant_exact(codes, scales, biases).astype(np.float32)


def round_bf16(v) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits, nearest, ties to even) -> uint16 bits.

    Works from the exact value: v = f * 2^e with 0.5 <= |f| < 1, keep f * 2^8
    rounded half-to-even.  Overflow goes to +-inf, NaN stays NaN.  (bf16
    subnormals, |v| < 2^-126, are rounded on the subnormal grid 2^-133.)
    """
    v = np.asarray(v, dtype=np.float64)
    f, e = np.frexp(v)
    e = np.maximum(e, -125)                      # below 2^-126 the grid is fixed at 2^-133
    m = np.rint(np.ldexp(v, 8 - e))             # integer significand, ties to even
    r = np.ldexp(m, e - 8)
    r = np.where(np.isnan(v), np.nan, r)
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, v), r)
    r32 = r.astype(np.float32)                  # exact: r has <= 8 significant bits
    return (r32.view(np.uint32) >> 16).astype(np.uint16)


def dequant_f16(codes, scales, biases) -> np.ndarray:
    """RN_f16 of the exact s*q + b (one rounding; numpy's float64->float16 cast rounds to nearest even).

    The precision of the weight operand of the tensor-core path for large M.
    """
    return dequant_exact(codes, scales, biases).astype(np.float16)


def dequant_bf16(codes, scales, biases) -> np.ndarray:
    """bf16 dequant = RN_bf16(fp32 dequant) as uint16 bits (the fp32 value is rounded again)."""
    return round_bf16(dequant_f32(codes, scales, biases).astype(np.float64))


# --------------------------------------------------------------------------
# The layer y = x . W^T
# --------------------------------------------------------------------------

def forward_ref(x_bits, codes, scales, biases) -> np.ndarray:
    """y_ref[m][n] = sum_k x[m][k] * w(n, k) in float64, w the fp32 dequant.

    Every product x*w is exact in float64 (8 + 24 significant bits); the sum is
    a float64 matrix product.
    """
    x = decode_bf16(x_bits)
    w = dequant_f32(codes, scales, biases).astype(np.float64)
    return x @ w.T


def forward_rows(x_bits, codes, scales, biases, rows) -> np.ndarray:
    """forward_ref restricted to the given rows of x (rows are independent)."""
    x = decode_bf16(np.asarray(x_bits)[np.asarray(rows)])
    w = dequant_f32(codes, scales, biases).astype(np.float64)
    return x @ w.T


def forward_triple_loop(x_bits, codes, scales, biases):
    """Brute force: nibble, f16 and bf16 decoded inline per element, float64 sum in k order.

    Pure Python; tiny shapes only.
    """
    x_bits = np.asarray(x_bits)
    M, K = x_bits.shape
    N = np.shape(codes)[0]
    s_bits = f16_array_bits(scales)
    b_bits = f16_array_bits(biases)
    y = [[0.0] * N for _ in range(M)]
    for m in range(M):
        xs = [struct.unpack("<f", struct.pack("<I", int(x_bits[m, k]) << 16))[0] for k in range(K)]
        for n in range(N):
            acc = 0.0
            for k in range(K):
                word = int(codes[n, k // 8])
                q = (word >> (4 * (k % 8))) & 0xF
                s = struct.unpack("<e", struct.pack("<H", int(s_bits[n, k // GROUP])))[0]
                b = struct.unpack("<e", struct.pack("<H", int(b_bits[n, k // GROUP])))[0]
                w32 = struct.unpack("<f", struct.pack("<f", s * q + b))[0]   # RN to binary32
                acc += xs[k] * w32
            y[m][n] = acc
    return np.array(y, dtype=np.float64)


def half_ulp_bf16(v) -> np.ndarray:
    """Half a bf16 unit in the last place at |v| (normal range)."""
    _, e = np.frexp(np.abs(np.asarray(v, dtype=np.float64)))
    return np.ldexp(1.0, np.maximum(e, -125) - 9)


def tolerance(y, y_ref, bf16_output: bool = True) -> dict:
    """Error metrics of reading R5.

    relF     = ||y - y_ref||_F / ||y_ref||_F                (gate <= 4e-3)
    max_rel  = max|y - y_ref| / rms(y_ref)                  (literal, reported)
    max_gate = max(|y - y_ref| - half_ulp)^+ / rms(y_ref)   (gate <= 1.5e-2; half_ulp = 0 for fp32 output)
    """
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    d = np.abs(y - y_ref)
    rms = float(np.sqrt(np.mean(y_ref * y_ref)))
    ref_norm = float(np.linalg.norm(y_ref))
    relF = float(np.linalg.norm(y - y_ref) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(y - y_ref))
    allowance = half_ulp_bf16(np.maximum(np.abs(y), np.abs(y_ref))) if bf16_output else 0.0
    excess = np.maximum(d - allowance, 0.0)
    denom = rms if rms > 0 else 1.0
    return {
        "relF": relF,
        "max_rel": float(d.max(initial=0.0) / denom),
        "max_gate": float(excess.max(initial=0.0) / denom),
        "rms": rms,
        "ok": bool(relF <= 4e-3 and excess.max(initial=0.0) <= 1.5e-2 * denom),
    }


# --------------------------------------------------------------------------
# RTN quantization (R3)
# --------------------------------------------------------------------------

def _check_packable(w: np.ndarray) -> None:
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    if np.any(np.abs(w) > F16_MAX):
        raise ValueError("weight magnitude beyond the f16 range")


def nearest_codes(w32, scale16, bias16) -> np.ndarray:
    """q = clamp(round_half_even(RN32(RN32(w - b) / s)), 0, 15) per group; 0 where s == 0.

    w32 float32 [N][G][64]; scale16, bias16 float16 [N][G].
    """
    s = scale16.astype(np.float32)[..., None]
    b = bias16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (w32 - b) / np.where(s == 0, np.float32(1), s)      # float32 subtract and divide
    q = np.clip(np.rint(t), 0, 15)
    q = np.where(s == 0, 0, q)
    return q.astype(np.int64)


def pack_rtn(w):
    """Min/max round-to-nearest quantization of float32 W [N][K] -> (codes, scales f16, biases f16)."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % GROUP == 0
    _check_packable(w)
    g = w.reshape(N, K // GROUP, GROUP)
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    s32 = (mx - mn) / np.float32(15.0)                            # float32: RN32(RN32(mx - mn) / 15)
    scale16 = s32.astype(np.float16)
    bias16 = mn.astype(np.float16)
    q = nearest_codes(g, scale16, bias16)
    return pack_codes(q.reshape(N, K)), scale16, bias16


# --------------------------------------------------------------------------
# Importance-weighted fit (R4)
# --------------------------------------------------------------------------

def imatrix_from_x(x_bits) -> np.ndarray:
    """Per-input-channel mean squared activation E[x_j^2] over the rows of x, float64."""
    x = decode_bf16(x_bits)
    return np.mean(x * x, axis=0)


def group_weighted_error(w, codes, scales, biases, imp) -> np.ndarray:
    """E[n][g] = sum_{j in g} imp_j * (w_j - deq_j)^2 in float64, deq the fp32 dequant."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    deq = dequant_f32(codes, scales, biases).astype(np.float64)
    d2 = (w - deq) ** 2 * np.asarray(imp, dtype=np.float64)[None, :]
    return d2.reshape(N, K // GROUP, GROUP).sum(axis=-1)


FIT_SHRINK = tuple(0.025 * i for i in range(9))   # 0, 0.025, ..., 0.2
FIT_REFITS = 2


def pack_imatrix(w, imatrix, row_chunk: int = 256):
    """Importance-weighted least-squares group fit, searched with RTN as candidate 0.

    Objective per group: E = sum_j imp_j * (w_j - deq_j)^2 (float64), deq the fp32
    dequant of the stored f16 triple.  imp = imatrix + 1e-6 * mean(imatrix), so a
    channel no activation reached still counts a little.  imatrix None -> RTN.

    Candidates, in order:
      0   the RTN triple (pack_rtn);
      1.. for each range shrink (a, b) in FIT_SHRINK^2 without (0, 0), in row-major
          order: lo = mn + a*r, hi = mx - b*r (r = mx - mn, float64),
          scale = RN_f16((hi - lo)/15), bias = RN_f16(lo), codes nearest (R3 rule);
          then FIT_REFITS rounds of: weighted least squares for (s, b) with the codes
          fixed (2x2 normal equations, float64; stop when the system is singular or
          s <= 0), scale = RN_f16(s), bias = RN_f16(b), codes re-chosen nearest.
    Every visited triple is scored; the lowest E wins, ties to the lowest index.
    For fixed (s, b) the nearest code is optimal for any imp >= 0 because the
    objective is a sum of independent non-negative terms.
    Every float64 sum (the imatrix mean, E and the least-squares moments of a
    group) is taken one term at a time in index order, so a device fit that
    follows the same steps with correctly rounded operations gives the same bytes.
    """
    w = np.asarray(w, dtype=np.float32)
    if imatrix is None:
        return pack_rtn(w)
    N, K = w.shape
    _check_packable(w)
    imp = np.asarray(imatrix, dtype=np.float64)
    total = 0.0
    for v in imp.tolist():                     # index order, one term at a time
        total = total + v
    imp = imp + 1e-6 * (total / imp.size)
    codes = np.empty((N, K // 8), dtype=np.uint32)
    scales = np.empty((N, K // GROUP), dtype=np.float16)
    biases = np.empty((N, K // GROUP), dtype=np.float16)
    for r0 in range(0, N, row_chunk):
        r1 = min(N, r0 + row_chunk)
        c, s, b = _fit_rows(w[r0:r1], imp)
        codes[r0:r1], scales[r0:r1], biases[r0:r1] = c, s, b
    return codes, scales, biases


def _seq_sum(t):
    """Sum over the last axis one term at a time in index order (float64)."""
    acc = np.zeros(t.shape[:-1], dtype=np.float64)
    for j in range(t.shape[-1]):
        acc = acc + t[..., j]
    return acc


def _score(g64, imp_g, q, s16, b16):
    """Weighted error of the triple (q, s16, b16) per group; deq = RN32(s*q + b)."""
    deq = (s16.astype(np.float64)[..., None] * q + b16.astype(np.float64)[..., None]).astype(np.float32)
    return _seq_sum(imp_g * (g64 - deq.astype(np.float64)) ** 2)


def weighted_ls_affine(g64, imp_g, q, sw, swx):
    """Weighted least squares of w ~ s*q + b over each group, the codes q held fixed.

    The refit step of the imatrix fit (aimarketly "Ideogram-4-IQ4_M", "What IQ4
    means here": the group parameters are a least-squares fit weighted by
    E[x^2]).  Minimising sum_j imp_j (w_j - s q_j - b)^2 over (s, b) gives the
    2x2 normal equations
        [sum imp q^2   sum imp q] [s]   [sum imp q w]
        [sum imp q     sum imp  ] [b] = [sum imp w  ]
    solved here by Cramer's rule in float64.  sw = sum imp and swx = sum imp w
    do not depend on q and are passed in; every moment is summed one term at a
    time in index order.  Returns (s, b, solvable), solvable False where the
    determinant vanishes relative to its terms (all codes equal).
    """
    qf = q.astype(np.float64)
    swq = _seq_sum(imp_g * qf)
    swqq = _seq_sum(imp_g * qf * qf)
    swqx = _seq_sum(imp_g * qf * g64)
    det = swqq * sw - swq * swq
    solvable = np.abs(det) > 1e-12 * np.maximum(swqq * sw, 1e-300)
    with np.errstate(divide="ignore", invalid="ignore"):
        s_ls = (swqx * sw - swq * swx) / det
        b_ls = (swqq * swx - swq * swqx) / det
    return s_ls, b_ls, solvable


def _fit_rows(w, imp):
    n, K = w.shape
    G = K // GROUP
    g32 = w.reshape(n, G, GROUP)
    g64 = g32.astype(np.float64)
    imp_g = imp.reshape(1, G, GROUP)

    c0, s0, b0 = pack_rtn(w)
    best_q = unpack_codes(c0, K).reshape(n, G, GROUP)
    best_s, best_b = s0.copy(), b0.copy()
    best_e = _score(g64, imp_g, best_q, best_s, best_b)

    def consider(q, s16, b16):
        nonlocal best_q, best_s, best_b, best_e
        e = _score(g64, imp_g, q, s16, b16)
        better = e < best_e                      # strict: ties keep the earlier candidate
        best_e = np.where(better, e, best_e)
        best_s = np.where(better, s16, best_s)
        best_b = np.where(better, b16, best_b)
        best_q = np.where(better[..., None], q, best_q)

    mn = g64.min(axis=-1)
    mx = g64.max(axis=-1)
    r = mx - mn
    sw = _seq_sum(imp_g)                                    # sum imp
    swx = _seq_sum(imp_g * g64)                             # sum imp * w
    for a in FIT_SHRINK:
        for bb in FIT_SHRINK:
            if a == 0 and bb == 0:
                continue
            lo = mn + a * r
            hi = mx - bb * r
            s16 = ((hi - lo) / 15.0).astype(np.float16)
            b16 = lo.astype(np.float16)
            q = nearest_codes(g32, s16, b16)
            consider(q, s16, b16)
            active = np.ones(s16.shape, dtype=bool)
            for _ in range(FIT_REFITS):
                s_ls, b_ls, solvable = weighted_ls_affine(g64, imp_g, q, sw, swx)
                ok = active & solvable
                ok &= np.isfinite(s_ls) & np.isfinite(b_ls) & (s_ls > 0)
                ok &= (np.abs(s_ls) <= F16_MAX) & (np.abs(b_ls) <= F16_MAX)
                active = ok
                if not ok.any():
                    break
                s_new = np.where(ok, s_ls, s16.astype(np.float64)).astype(np.float16)
                b_new = np.where(ok, b_ls, b16.astype(np.float64)).astype(np.float16)
                q_new = nearest_codes(g32, s_new, b_new)
                s16 = np.where(ok, s_new, s16)
                b16 = np.where(ok, b_new, b16)
                q = np.where(ok[..., None], q_new, q)
                e = _score(g64, imp_g, q, s16, b16)
                better = ok & (e < best_e)
                best_e = np.where(better, e, best_e)
                best_s = np.where(better, s16, best_s)
                best_b = np.where(better, b16, best_b)
                best_q = np.where(better[..., None], q, best_q)
    return pack_codes(best_q.reshape(n, K)), best_s.astype(np.float16), best_b.astype(np.float16)


# --------------------------------------------------------------------------
# W8 g64 (R9): 8-bit codes with the same per-64 f16 scale and bias
# --------------------------------------------------------------------------

def unpack_codes8(codes, K: int) -> np.ndarray:
    """uint32 [N][K/4] -> int64 codes q [N][K], code k%4 in bits 8*(k%4) .. 8*(k%4)+7."""
    c = np.asarray(codes, dtype=np.uint32).astype(np.int64)
    N = c.shape[0]
    assert c.shape[1] * 4 == K
    shifts = 8 * np.arange(4, dtype=np.int64)
    q = (c[:, :, None] >> shifts[None, None, :]) & 0xFF
    return q.reshape(N, K)


def pack_codes8(q) -> np.ndarray:
    """int codes [N][K] in [0, 255] -> uint32 [N][K/4], low byte first."""
    q = np.asarray(q, dtype=np.uint64)
    N, K = q.shape
    assert K % 4 == 0 and q.max(initial=0) <= 255
    shifts = 8 * np.arange(4, dtype=np.uint64)
    words = (q.reshape(N, K // 4, 4) << shifts[None, None, :]).sum(axis=-1)
    return words.astype(np.uint32)


def dequant8_exact(codes, scales, biases) -> np.ndarray:
    """Exact w = s*q + b as float64 [N][K] for 8-bit codes.

    s and b are integer multiples of 2^-24 below 2^16 and q <= 255, so
    s*q + b = i * 2^-24 with |i| < 2^49: float64 holds it without rounding.
    """
    N, G = np.shape(scales)
    K = G * GROUP
    q = unpack_codes8(codes, K).astype(np.float64)
    s = np.repeat(decode_f16(f16_array_bits(scales)), GROUP, axis=1)
    b = np.repeat(decode_f16(f16_array_bits(biases)), GROUP, axis=1)
    return s * q + b


def dequant8_f32(codes, scales, biases) -> np.ndarray:
    """fp32 dequant of 8-bit codes: RN_fp32 of the exact value (R2)."""
    return dequant8_exact(codes, scales, biases).astype(np.float32)


def dequant8_f16(codes, scales, biases) -> np.ndarray:
    """RN_f16 of the exact s*q + b for 8-bit codes: the weight operand of the tensor-core paths (R7)."""
    return dequant8_exact(codes, scales, biases).astype(np.float16)


def dequant8_bf16(codes, scales, biases) -> np.ndarray:
    """bf16 dequant of 8-bit codes = RN_bf16(fp32 dequant) as uint16 bits."""
    return round_bf16(dequant8_f32(codes, scales, biases).astype(np.float64))


def forward8_ref(x_bits, codes, scales, biases) -> np.ndarray:
    """y_ref[m][n] = sum_k x[m][k] * w(n, k) in float64, w the fp32 dequant of 8-bit codes."""
    x = decode_bf16(x_bits)
    w = dequant8_f32(codes, scales, biases).astype(np.float64)
    return x @ w.T


def forward8_rows(x_bits, codes, scales, biases, rows) -> np.ndarray:
    """forward8_ref restricted to the given rows of x (rows are independent)."""
    x = decode_bf16(np.asarray(x_bits)[np.asarray(rows)])
    w = dequant8_f32(codes, scales, biases).astype(np.float64)
    return x @ w.T


def nearest_codes8(w32, scale16, bias16) -> np.ndarray:
    """q = clamp(round_half_even(RN32(RN32(w - b) / s)), 0, 255) per group; 0 where s == 0."""
    s = scale16.astype(np.float32)[..., None]
    b = bias16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (w32 - b) / np.where(s == 0, np.float32(1), s)      # float32 subtract and divide
    q = np.clip(np.rint(t), 0, 255)
    q = np.where(s == 0, 0, q)
    return q.astype(np.int64)


def pack8_rtn(w):
    """Min/max round-to-nearest quantization of float32 W [N][K] to 8-bit codes (R9)."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % GROUP == 0
    _check_packable(w)
    g = w.reshape(N, K // GROUP, GROUP)
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    s32 = (mx - mn) / np.float32(255.0)                           # float32: RN32(RN32(mx - mn) / 255)
    scale16 = s32.astype(np.float16)
    bias16 = mn.astype(np.float16)
    q = nearest_codes8(g, scale16, bias16)
    return pack_codes8(q.reshape(N, K)), scale16, bias16


# --------------------------------------------------------------------------
# SwiGLU up/gate pair (R10, R11)
# --------------------------------------------------------------------------

SILU_SLOPE_MAX = 1.1      # max_z silu'(z) = 1.0998... (at z = 2.3994...); min is -0.0998...


def silu(z) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z)) in float64 (-0 for very negative z)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_linears(x_bits, gate, up, rows=None, bits: int = 4):
    """(g, u) = (x . W_gate^T, x . W_up^T) in float64 over the given rows of x.

    gate and up are (codes, scales, biases) triples of [I][K] weights with `bits`-bit codes.
    """
    x_bits = np.asarray(x_bits)
    rows = np.arange(x_bits.shape[0]) if rows is None else np.asarray(rows)
    fwd = forward_rows if bits == 4 else forward8_rows
    return fwd(x_bits, *gate, rows), fwd(x_bits, *up, rows)


def swiglu_ref(x_bits, gate, up, rows=None, bits: int = 4) -> np.ndarray:
    """h = silu(g) * u (R10), float64 [rows][I]."""
    g, u = swiglu_linears(x_bits, gate, up, rows, bits)
    return silu(g) * u


def swiglu_tolerance(h, g_ref, u_ref, bf16_output: bool = True) -> dict:
    """Error metrics of reading R11 for h against the float64 reference built from g_ref, u_ref.

    relF      = ||h - h_ref||_F / ||h_ref||_F                              (gate <= 8e-3)
    max_ratio = max_i (|h_i - h_ref_i| - half_ulp_i)^+ / bound_i             (gate <= 1)
    bound_i   = 1.1 * d_g * (|u_i| + d_u) + |silu(g_i)| * d_u,  d = 1.5e-2 * rms(output)
    """
    h = np.asarray(h, dtype=np.float64)
    g_ref = np.asarray(g_ref, dtype=np.float64)
    u_ref = np.asarray(u_ref, dtype=np.float64)
    h_ref = silu(g_ref) * u_ref
    d_g = 1.5e-2 * float(np.sqrt(np.mean(g_ref * g_ref)))
    d_u = 1.5e-2 * float(np.sqrt(np.mean(u_ref * u_ref)))
    bound = SILU_SLOPE_MAX * d_g * (np.abs(u_ref) + d_u) + np.abs(silu(g_ref)) * d_u
    d = np.abs(h - h_ref)
    allowance = half_ulp_bf16(np.maximum(np.abs(h), np.abs(h_ref))) if bf16_output else 0.0
    excess = np.maximum(d - allowance, 0.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(excess > 0, excess / np.where(bound > 0, bound, 1.0), 0.0)
        ratio = np.where((excess > 0) & (bound <= 0), np.inf, ratio)
    ref_norm = float(np.linalg.norm(h_ref))
    relF = float(np.linalg.norm(h - h_ref) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(h - h_ref))
    max_ratio = float(ratio.max(initial=0.0))
    return {"relF": relF, "max_ratio": max_ratio, "ok": bool(relF <= 8e-3 and max_ratio <= 1.0)}
