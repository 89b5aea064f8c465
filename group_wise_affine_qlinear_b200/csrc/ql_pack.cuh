// Min/max round-to-nearest quantization of fp32 weights into the W4 g64 format.
//
// MLX's own min/max solution is candidate 0 of the importance-weighted search
// described in aimarketly "Ideogram-4-IQ4_M", "What IQ4 means here"; the
// packer must be deterministic ("byte-equivalent to load-time quantization",
// huggingface "SceneWorks/ideogram-4-mlx", Provenance).  Per group of 64:
//   s     = RN32(RN32(max - min) / 15)
//   scale = RN_f16(s), bias = RN_f16(min)
//   q     = clamp(rint_half_even(RN32(RN32(w - bias) / scale)), 0, 15); q = 0 if scale == 0
// Every operation is a correctly rounded IEEE operation, so the bytes are the
// same on any conforming implementation.
#pragma once

#include "ql_common.cuh"

namespace ql {

// One warp per (row, group): lane l holds w[2l], w[2l+1].
__global__ void __launch_bounds__(256) pack_rtn_kernel(const float* __restrict__ w,
                                                       uint32_t* __restrict__ codes,
                                                       __half* __restrict__ scales,
                                                       __half* __restrict__ biases,
                                                       int64_t n_groups) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t grp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         grp < n_groups; grp += warps_total) {
        const float2 v = reinterpret_cast<const float2*>(w + grp * kGroup)[lane];
        const bool bad = !(fabsf(v.x) <= 65504.0f) || !(fabsf(v.y) <= 65504.0f);   // also catches NaN
        const unsigned any_bad = __ballot_sync(0xFFFFFFFFu, bad);
        if (any_bad) {
            if (lane < 8) codes[grp * 8 + lane] = 0u;
            if (lane == 0) {
                scales[grp] = __float2half_rn(0.0f);
                biases[grp] = __float2half_rn(0.0f);
                record_status(QL_ERR_INVALID_ARG);
            }
            continue;
        }
        float mn = fminf(v.x, v.y);
        float mx = fmaxf(v.x, v.y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        }
        const float s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        const __half s_h = __float2half_rn(s);
        const __half b_h = __float2half_rn(mn);
        const float sf = __half2float(s_h);
        const float bf = __half2float(b_h);
        uint32_t q0 = 0, q1 = 0;
        if (sf != 0.0f) {
            const float t0 = rintf(__fdiv_rn(__fsub_rn(v.x, bf), sf));
            const float t1 = rintf(__fdiv_rn(__fsub_rn(v.y, bf), sf));
            q0 = static_cast<uint32_t>(fminf(fmaxf(t0, 0.0f), 15.0f));
            q1 = static_cast<uint32_t>(fminf(fmaxf(t1, 0.0f), 15.0f));
        }
        // lanes 4j..4j+3 hold the 8 codes of word j; lane l contributes one byte.
        uint32_t part = (q0 | (q1 << 4)) << (8 * (lane & 3));
        part |= __shfl_xor_sync(0xFFFFFFFFu, part, 1);
        part |= __shfl_xor_sync(0xFFFFFFFFu, part, 2);
        if ((lane & 3) == 0) codes[grp * 8 + (lane >> 2)] = part;
        if (lane == 0) {
            scales[grp] = s_h;
            biases[grp] = b_h;
        }
    }
}

// The same min/max round-to-nearest for 8-bit codes (255 levels):
//   s = RN32(RN32(max - min) / 255), scale = RN_f16(s), bias = RN_f16(min),
//   q = clamp(rint_half_even(RN32(RN32(w - bias) / scale)), 0, 255); q = 0 if scale == 0.
// One warp per (row, group): lane l holds w[2l], w[2l+1]; code word j (k = 4j .. 4j+3) gets its
// low half from lane 2j and its high half from lane 2j+1.
__global__ void __launch_bounds__(256) pack8_rtn_kernel(const float* __restrict__ w,
                                                        uint32_t* __restrict__ codes,
                                                        __half* __restrict__ scales,
                                                        __half* __restrict__ biases,
                                                        int64_t n_groups) {
    constexpr int kWordsPerGroup = kGroup / 4;
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t grp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         grp < n_groups; grp += warps_total) {
        const float2 v = reinterpret_cast<const float2*>(w + grp * kGroup)[lane];
        const bool bad = !(fabsf(v.x) <= 65504.0f) || !(fabsf(v.y) <= 65504.0f);   // also catches NaN
        const unsigned any_bad = __ballot_sync(0xFFFFFFFFu, bad);
        if (any_bad) {
            if (lane < kWordsPerGroup) codes[grp * kWordsPerGroup + lane] = 0u;
            if (lane == 0) {
                scales[grp] = __float2half_rn(0.0f);
                biases[grp] = __float2half_rn(0.0f);
                record_status(QL_ERR_INVALID_ARG);
            }
            continue;
        }
        float mn = fminf(v.x, v.y);
        float mx = fmaxf(v.x, v.y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        }
        const float s = __fdiv_rn(__fsub_rn(mx, mn), 255.0f);
        const __half s_h = __float2half_rn(s);
        const __half b_h = __float2half_rn(mn);
        const float sf = __half2float(s_h);
        const float bf = __half2float(b_h);
        uint32_t q0 = 0, q1 = 0;
        if (sf != 0.0f) {
            const float t0 = rintf(__fdiv_rn(__fsub_rn(v.x, bf), sf));
            const float t1 = rintf(__fdiv_rn(__fsub_rn(v.y, bf), sf));
            q0 = static_cast<uint32_t>(fminf(fmaxf(t0, 0.0f), 255.0f));
            q1 = static_cast<uint32_t>(fminf(fmaxf(t1, 0.0f), 255.0f));
        }
        uint32_t part = (q0 | (q1 << 8)) << (16 * (lane & 1));
        part |= __shfl_xor_sync(0xFFFFFFFFu, part, 1);
        if ((lane & 1) == 0) codes[grp * kWordsPerGroup + (lane >> 1)] = part;
        if (lane == 0) {
            scales[grp] = s_h;
            biases[grp] = b_h;
        }
    }
}

}  // namespace ql
