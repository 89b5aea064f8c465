// Importance-weighted group fit of fp32 weights into the W4 g64 format.
//
// The quantizer the pages describe (aimarketly "Ideogram-4-IQ4_M", "What IQ4
// means here") fits each group of 64 by weighted least squares against E[x^2]
// statistics, with MLX's own min/max round-to-nearest solution as candidate 0,
// so the fit is never worse than RTN on its objective.  The search, made
// concrete:
//   objective   E = sum_j imp_j (w_j - RN32(s q_j + b))^2 in float64, with
//               imp_j = imatrix_j + 1e-6 * mean(imatrix) (so a channel no
//               activation reached still counts a little);
//   candidate 0 the RTN triple (min/max, as qlinear_pack without an imatrix);
//   then        for each range shrink (a, c) in {0, 0.025, ..., 0.2}^2 except
//               (0, 0), row-major: lo = mn + a r, hi = mx - c r, r = mx - mn,
//               scale = RN_f16((hi - lo) / 15), bias = RN_f16(lo), codes
//               nearest; then up to two rounds of weighted least squares for
//               (s, b) with the codes fixed (2x2 normal equations in float64;
//               stop when singular, s <= 0 or out of the f16 range), rounded
//               to f16, codes re-chosen nearest.
//   The lowest E over every triple visited wins; ties keep the earlier one.
// Codes are chosen in fp32 exactly as the RTN packer does.  Every float64 sum is
// taken one term at a time in index order and every operation is a correctly
// rounded IEEE operation (explicit __d*_rn intrinsics, so nothing is fused), so
// the bytes equal those of any implementation that takes the same steps.
#pragma once

#include "ql_common.cuh"

namespace ql {

constexpr int kFitThreads = 128;     // one thread per (row, group): a CTA fits one group column of 128 rows

// Nearest codes in fp32: q = clamp(rint_half_even(RN32(RN32(w - b) / s)), 0, 15), q = 0 when s == 0;
// code j of the group goes to nibble j % 8 of word j / 8.
__device__ __forceinline__ void fit_codes(const float (*ws)[kFitThreads], float sf, float bf, uint32_t (&q)[8]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t word = 0u;
        if (sf != 0.0f) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float t = rintf(__fdiv_rn(__fsub_rn(ws[8 * c + j][threadIdx.x], bf), sf));
                word |= static_cast<uint32_t>(fminf(fmaxf(t, 0.0f), 15.0f)) << (4 * j);
            }
        }
        q[c] = word;
    }
}

__device__ __forceinline__ double fit_code(const uint32_t (&q)[8], int j) {
    return static_cast<double>((q[j >> 3] >> (4 * (j & 7))) & 0xFu);
}

// E = sum_j imp_j (w_j - RN32(s q_j + b))^2, index order.
__device__ __forceinline__ double fit_score(const float (*ws)[kFitThreads], const double* imp, __half s16, __half b16,
                                            const uint32_t (&q)[8]) {
    const double sd = static_cast<double>(__half2float(s16));
    const double bd = static_cast<double>(__half2float(b16));
    double e = 0.0;
    for (int j = 0; j < kGroup; ++j) {
        const float deq = __double2float_rn(__dadd_rn(__dmul_rn(sd, fit_code(q, j)), bd));
        const double d = __dsub_rn(static_cast<double>(ws[j][threadIdx.x]), static_cast<double>(deq));
        e = __dadd_rn(e, __dmul_rn(imp[j], __dmul_rn(d, d)));
    }
    return e;
}

// grid (G, ceil(N / 128)), 128 threads: CTA (g, nb) fits group column g of rows nb*128 ..
__global__ void __launch_bounds__(kFitThreads) pack_fit_kernel(const float* __restrict__ w,
                                                               const float* __restrict__ imatrix,
                                                               uint32_t* __restrict__ codes,
                                                               __half* __restrict__ scales,
                                                               __half* __restrict__ biases, int K, int N) {
    __shared__ float ws[kGroup][kFitThreads];      // ws[j][t]: weight j of row t's group
    __shared__ double imp[kGroup];
    __shared__ double floor_s;
    __shared__ int bad_imp;
    const int G = K / kGroup;
    const int g = blockIdx.x;
    const int row0 = blockIdx.y * kFitThreads;
    if (threadIdx.x == 0) {
        // mean of the importance vector, index order; a negative or non-finite entry is an argument error
        double total = 0.0;
        int bad = 0;
        for (int k = 0; k < K; ++k) {
            const float v = imatrix[k];
            bad |= !(v >= 0.0f && v <= 3.4028235e38f);
            total = __dadd_rn(total, static_cast<double>(v));
        }
        floor_s = __dmul_rn(1e-6, __ddiv_rn(total, static_cast<double>(K)));
        bad_imp = bad;
    }
    for (int i = threadIdx.x; i < kGroup * kFitThreads; i += kFitThreads) {     // coalesced: 64 floats per row
        const int r = i / kGroup, j = i % kGroup;
        ws[j][r] = (row0 + r < N) ? w[static_cast<int64_t>(row0 + r) * K + static_cast<int64_t>(g) * kGroup + j] : 0.0f;
    }
    __syncthreads();
    if (threadIdx.x < kGroup)
        imp[threadIdx.x] = __dadd_rn(static_cast<double>(imatrix[static_cast<int64_t>(g) * kGroup + threadIdx.x]), floor_s);
    __syncthreads();
    const int n = row0 + static_cast<int>(threadIdx.x);
    if (n >= N) return;
    const int64_t grp = static_cast<int64_t>(n) * G + g;
    uint32_t* out_codes = codes + static_cast<int64_t>(n) * (K / 8) + static_cast<int64_t>(g) * 8;

    bool bad = bad_imp != 0;
    float mn32 = ws[0][threadIdx.x], mx32 = mn32;
    for (int j = 0; j < kGroup; ++j) {
        const float v = ws[j][threadIdx.x];
        bad |= !(fabsf(v) <= 65504.0f);                // also catches NaN
        mn32 = fminf(mn32, v);
        mx32 = fmaxf(mx32, v);
    }
    if (bad) {
        for (int c = 0; c < 8; ++c) out_codes[c] = 0u;
        scales[grp] = __float2half_rn(0.0f);
        biases[grp] = __float2half_rn(0.0f);
        record_status(QL_ERR_INVALID_ARG);
        return;
    }

    // candidate 0: RTN
    uint32_t best_q[8];
    __half best_s = __float2half_rn(__fdiv_rn(__fsub_rn(mx32, mn32), 15.0f));
    __half best_b = __float2half_rn(mn32);
    fit_codes(ws, __half2float(best_s), __half2float(best_b), best_q);
    double best_e = fit_score(ws, imp, best_s, best_b, best_q);

    const double mn = static_cast<double>(mn32), mx = static_cast<double>(mx32);
    const double r = __dsub_rn(mx, mn);
    double sw = 0.0, swx = 0.0;
    for (int j = 0; j < kGroup; ++j) {
        sw = __dadd_rn(sw, imp[j]);
        swx = __dadd_rn(swx, __dmul_rn(imp[j], static_cast<double>(ws[j][threadIdx.x])));
    }
    uint32_t q[8];
    for (int ai = 0; ai < 9; ++ai) {
        for (int ci = 0; ci < 9; ++ci) {
            if (ai == 0 && ci == 0) continue;
            const double lo = __dadd_rn(mn, __dmul_rn(__dmul_rn(0.025, static_cast<double>(ai)), r));
            const double hi = __dsub_rn(mx, __dmul_rn(__dmul_rn(0.025, static_cast<double>(ci)), r));
            __half s16 = __double2half(__ddiv_rn(__dsub_rn(hi, lo), 15.0));
            __half b16 = __double2half(lo);
            fit_codes(ws, __half2float(s16), __half2float(b16), q);
            double e = fit_score(ws, imp, s16, b16, q);
            if (e < best_e) {
                best_e = e;
                best_s = s16;
                best_b = b16;
#pragma unroll
                for (int c = 0; c < 8; ++c) best_q[c] = q[c];
            }
            for (int it = 0; it < 2; ++it) {
                double swq = 0.0, swqq = 0.0, swqx = 0.0;
                for (int j = 0; j < kGroup; ++j) {
                    const double iq = __dmul_rn(imp[j], fit_code(q, j));
                    swq = __dadd_rn(swq, iq);
                    swqq = __dadd_rn(swqq, __dmul_rn(iq, fit_code(q, j)));
                    swqx = __dadd_rn(swqx, __dmul_rn(iq, static_cast<double>(ws[j][threadIdx.x])));
                }
                const double det = __dsub_rn(__dmul_rn(swqq, sw), __dmul_rn(swq, swq));
                if (!(fabs(det) > __dmul_rn(1e-12, fmax(__dmul_rn(swqq, sw), 1e-300)))) break;
                const double s_ls = __ddiv_rn(__dsub_rn(__dmul_rn(swqx, sw), __dmul_rn(swq, swx)), det);
                const double b_ls = __ddiv_rn(__dsub_rn(__dmul_rn(swqq, swx), __dmul_rn(swq, swqx)), det);
                if (!(isfinite(s_ls) && isfinite(b_ls) && s_ls > 0.0 && fabs(s_ls) <= 65504.0 && fabs(b_ls) <= 65504.0))
                    break;
                s16 = __double2half(s_ls);
                b16 = __double2half(b_ls);
                fit_codes(ws, __half2float(s16), __half2float(b16), q);
                e = fit_score(ws, imp, s16, b16, q);
                if (e < best_e) {
                    best_e = e;
                    best_s = s16;
                    best_b = b16;
#pragma unroll
                    for (int c = 0; c < 8; ++c) best_q[c] = q[c];
                }
            }
        }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) out_codes[c] = best_q[c];
    scales[grp] = best_s;
    biases[grp] = best_b;
}

}  // namespace ql
