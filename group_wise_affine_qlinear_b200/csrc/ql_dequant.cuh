// Standalone dequantization (HBM-bound streaming kernel).
//
// out[n][k] = RN_fp32(s * q + b) with one fused multiply-add, which rounds the
// exact value once (aimarketly "Ideogram-4-IQ4_M", "What IQ4 means here":
// uniform affine grid w = scale * q + bias).  bf16 output rounds that fp32
// value once more, to nearest even.
#pragma once

#include "ql_common.cuh"

namespace ql {

// One thread per 32-bit code word (8 codes): word i covers out[8i .. 8i+7]
// and uses parameter index i / 8, because K/8 words per row are a multiple of
// the 8 words of a 64-group.  Consecutive threads write consecutive 32 B (fp32)
// or 16 B (bf16) so every warp store is contiguous.
template <bool kBf16Out>
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ codes,
                                                      const __half* __restrict__ scales,
                                                      const __half* __restrict__ biases,
                                                      void* __restrict__ out, int64_t n_words) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_words; i += stride) {
        const uint32_t v = __ldg(codes + i);
        const float s = __half2float(scales[i >> 3]);
        const float b = __half2float(biases[i >> 3]);
        float w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float q = static_cast<float>((v >> (4 * j)) & 0xFu);
            w[j] = __fmaf_rn(q, s, b);
        }
        if constexpr (kBf16Out) {
            uint4 o;
            o.x = pack_bf16x2(w[0], w[1]);
            o.y = pack_bf16x2(w[2], w[3]);
            o.z = pack_bf16x2(w[4], w[5]);
            o.w = pack_bf16x2(w[6], w[7]);
            reinterpret_cast<uint4*>(out)[i] = o;
        } else {
            float4* o = reinterpret_cast<float4*>(out) + 2 * i;
            o[0] = make_float4(w[0], w[1], w[2], w[3]);
            o[1] = make_float4(w[4], w[5], w[6], w[7]);
        }
    }
}

// 8-bit codes (huggingface "SceneWorks/ideogram-4-mlx", Versions: the Q8 pack; same f16 scale and
// bias per 64 weights): one thread per 32-bit word of 4 codes, low byte first.  Word i covers
// out[4i .. 4i+3] and uses parameter index i / 16 (a 64-group is 16 words).  q <= 255 times an
// 11-bit scale is exact in fp32, so the fused multiply-add again rounds s*q + b once.
template <bool kBf16Out>
__global__ void __launch_bounds__(256) dequant8_kernel(const uint32_t* __restrict__ codes,
                                                       const __half* __restrict__ scales,
                                                       const __half* __restrict__ biases,
                                                       void* __restrict__ out, int64_t n_words) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_words; i += stride) {
        const uint32_t v = __ldg(codes + i);
        const float s = __half2float(scales[i >> 4]);
        const float b = __half2float(biases[i >> 4]);
        float w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = __fmaf_rn(static_cast<float>((v >> (8 * j)) & 0xFFu), s, b);
        if constexpr (kBf16Out) {
            reinterpret_cast<uint2*>(out)[i] = make_uint2(pack_bf16x2(w[0], w[1]), pack_bf16x2(w[2], w[3]));
        } else {
            reinterpret_cast<float4*>(out)[i] = make_float4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace ql
