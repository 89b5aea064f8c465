// CUDA-core weight-streaming path (split-K GEMV) and the split-K reduction.
//
// y[m][n] = sum_g ( s(n,g) * sum_{k in g} q(n,k) x[m][k]  +  b(n,g) * sum_{k in g} x[m][k] )
// which is sum_k (s*q + b) * x rearranged per group, accumulated in fp32.
// Each warp streams one weight row's K-slice with 128-bit loads (32 codes =
// half a group per lane per step); x is small and served from L1/L2.
#pragma once

#include "ql_common.cuh"

namespace ql {

constexpr int kGemvWarps = 8;          // rows per CTA (one per warp)
constexpr int kGemvMChunk = 4;         // activation rows per register accumulator block

// grid: (N / kGemvWarps, S).  Slice z covers groups [z*G/S, (z+1)*G/S) (balanced, non-empty for S <= G).
// out: partial[z][M][N] fp32 when split_k > 1, else y (bf16 or fp32) directly.
// The body is a device function so more than one kernel entry can share it.
template <bool kBf16Out>
__device__ __forceinline__ void gemv_body(
    const __nv_bfloat16* __restrict__ x, const uint32_t* __restrict__ codes,
    const __half* __restrict__ scales, const __half* __restrict__ biases,
    void* __restrict__ out, int M, int K, int N, bool partial_out) {
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
    if (n >= N) return;
    const int G = K / kGroup;
    const int S = gridDim.y;
    const int g0 = static_cast<int>((static_cast<int64_t>(blockIdx.y) * G) / S);
    const int g1 = static_cast<int>((static_cast<int64_t>(blockIdx.y + 1) * G) / S);
    // half-groups (uint4 of codes) in this slice
    const int h0 = 2 * g0, h1 = 2 * g1;
    const uint4* crow = reinterpret_cast<const uint4*>(codes + static_cast<int64_t>(n) * (K / 8));
    const __half* srow = scales + static_cast<int64_t>(n) * G;
    const __half* brow = biases + static_cast<int64_t>(n) * G;

    for (int m0 = 0; m0 < M; m0 += kGemvMChunk) {
        float acc[kGemvMChunk];
#pragma unroll
        for (int i = 0; i < kGemvMChunk; ++i) acc[i] = 0.0f;
        for (int h = h0 + lane; h < h1; h += 32) {
            const uint4 c = __ldg(crow + h);
            const float s = __half2float(srow[h >> 1]);
            const float b = __half2float(brow[h >> 1]);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int i = 0; i < kGemvMChunk; ++i) {
                const int m = m0 + i;
                if (m >= M) break;
                const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + 32 * h);
                float dot = 0.0f, xs = 0.0f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint4 xv = __ldg(xr + w);
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float xa = bf16_lo(xw[p]);
                        const float xb = bf16_hi(xw[p]);
                        const float qa = static_cast<float>((cw[w] >> (8 * p)) & 0xFu);
                        const float qb = static_cast<float>((cw[w] >> (8 * p + 4)) & 0xFu);
                        dot = fmaf(qa, xa, dot);
                        dot = fmaf(qb, xb, dot);
                        xs += xa + xb;
                    }
                }
                acc[i] = fmaf(s, dot, fmaf(b, xs, acc[i]));
            }
        }
#pragma unroll
        for (int i = 0; i < kGemvMChunk; ++i) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
        }
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < kGemvMChunk; ++i) {
                const int m = m0 + i;
                if (m >= M) break;
                const int64_t o = static_cast<int64_t>(m) * N + n;
                if (partial_out) {
                    const int64_t at = static_cast<int64_t>(blockIdx.y) * M * N + o;
                    if (in_bounds(at, static_cast<int64_t>(gridDim.y) * M * N)) reinterpret_cast<float*>(out)[at] = acc[i];
                } else if constexpr (kBf16Out) {
                    reinterpret_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(acc[i]);
                } else {
                    reinterpret_cast<float*>(out)[o] = acc[i];
                }
            }
        }
    }
}

template <bool kBf16Out>
__global__ void __launch_bounds__(kGemvWarps * 32) cc_stream_kernel(
    const __nv_bfloat16* __restrict__ x, const uint32_t* __restrict__ codes,
    const __half* __restrict__ scales, const __half* __restrict__ biases,
    void* __restrict__ out, int M, int K, int N, bool partial_out) {
    gemv_body<kBf16Out>(x, codes, scales, biases, out, M, K, N, partial_out);
}

// The same split-K GEMV for 8-bit codes (codes uint32 [N][K/4], low byte first): each lane step
// streams a quarter group (16 codes, one 128-bit load) and the 16 matching activations.
template <bool kBf16Out>
__global__ void __launch_bounds__(kGemvWarps * 32) cc_stream8_kernel(
    const __nv_bfloat16* __restrict__ x, const uint32_t* __restrict__ codes,
    const __half* __restrict__ scales, const __half* __restrict__ biases,
    void* __restrict__ out, int M, int K, int N, bool partial_out) {
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
    if (n >= N) return;
    const int G = K / kGroup;
    const int S = gridDim.y;
    const int g0 = static_cast<int>((static_cast<int64_t>(blockIdx.y) * G) / S);
    const int g1 = static_cast<int>((static_cast<int64_t>(blockIdx.y + 1) * G) / S);
    // quarter groups (uint4 of codes) in this slice
    const int h0 = 4 * g0, h1 = 4 * g1;
    const uint4* crow = reinterpret_cast<const uint4*>(codes + static_cast<int64_t>(n) * (K / 4));
    const __half* srow = scales + static_cast<int64_t>(n) * G;
    const __half* brow = biases + static_cast<int64_t>(n) * G;

    for (int m0 = 0; m0 < M; m0 += kGemvMChunk) {
        float acc[kGemvMChunk];
#pragma unroll
        for (int i = 0; i < kGemvMChunk; ++i) acc[i] = 0.0f;
        for (int h = h0 + lane; h < h1; h += 32) {
            const uint4 c = __ldg(crow + h);
            const float s = __half2float(srow[h >> 2]);
            const float b = __half2float(brow[h >> 2]);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int i = 0; i < kGemvMChunk; ++i) {
                const int m = m0 + i;
                if (m >= M) break;
                // activations k = 16h .. 16h+15: two 128-bit loads; code word wd (k = 4wd .. 4wd+3)
                // meets the bf16 pairs (k 4wd, 4wd+1) and (k 4wd+2, 4wd+3)
                const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + 16 * h);
                const uint4 xa = __ldg(xr), xb = __ldg(xr + 1);
                float dot = 0.0f, xs = 0.0f;
                auto word = [&](uint32_t c, uint32_t x01, uint32_t x23) {
                    const float x0 = bf16_lo(x01), x1 = bf16_hi(x01), x2 = bf16_lo(x23), x3 = bf16_hi(x23);
                    dot = fmaf(static_cast<float>(c & 0xFFu), x0, dot);
                    dot = fmaf(static_cast<float>((c >> 8) & 0xFFu), x1, dot);
                    dot = fmaf(static_cast<float>((c >> 16) & 0xFFu), x2, dot);
                    dot = fmaf(static_cast<float>(c >> 24), x3, dot);
                    xs += (x0 + x1) + (x2 + x3);
                };
                word(cw[0], xa.x, xa.y);
                word(cw[1], xa.z, xa.w);
                word(cw[2], xb.x, xb.y);
                word(cw[3], xb.z, xb.w);
                acc[i] = fmaf(s, dot, fmaf(b, xs, acc[i]));
            }
        }
#pragma unroll
        for (int i = 0; i < kGemvMChunk; ++i) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
        }
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < kGemvMChunk; ++i) {
                const int m = m0 + i;
                if (m >= M) break;
                const int64_t o = static_cast<int64_t>(m) * N + n;
                if (partial_out) {
                    const int64_t at = static_cast<int64_t>(blockIdx.y) * M * N + o;
                    if (in_bounds(at, static_cast<int64_t>(gridDim.y) * M * N)) reinterpret_cast<float*>(out)[at] = acc[i];
                } else if constexpr (kBf16Out) {
                    reinterpret_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(acc[i]);
                } else {
                    reinterpret_cast<float*>(out)[o] = acc[i];
                }
            }
        }
    }
}

// y[i] = sum_{z=0}^{S-1} partial[z][i] in that fixed order (deterministic), four
// elements per thread.  count = M*N is a multiple of 8.
template <bool kBf16Out>
__device__ __forceinline__ void ordered_sum_body(const float* __restrict__ partial, void* __restrict__ y,
                                                   int64_t count, int S) {
    const int64_t n4 = count / 4;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 a = __ldg(reinterpret_cast<const float4*>(partial) + i);
        for (int z = 1; z < S; ++z) {
            const float4 b = __ldg(reinterpret_cast<const float4*>(partial + z * count) + i);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        if constexpr (kBf16Out) {
            uint2 o;
            o.x = pack_bf16x2(a.x, a.y);
            o.y = pack_bf16x2(a.z, a.w);
            reinterpret_cast<uint2*>(y)[i] = o;
        } else {
            reinterpret_cast<float4*>(y)[i] = a;
        }
    }
}

template <bool kBf16Out>
__global__ void __launch_bounds__(256) ordered_sum_kernel(const float* __restrict__ partial,
                                                            void* __restrict__ y, int64_t count, int S) {
    ordered_sum_body<kBf16Out>(partial, y, count, S);
}

// Split factor of the weight-streaming path: double it while the grid has fewer
// than four waves of 8-row CTAs and every slice keeps at least 64 groups.
inline int gemv_auto_split(int64_t K, int64_t N, int sm_count) {
    const int64_t G = K / kGroup;
    const int64_t ctas = N / kGemvWarps;
    int s = 1;
    while (ctas * s < 4 * sm_count && G / (2 * s) >= 64) s *= 2;
    return s;
}

}  // namespace ql
