// Operand preparation for the fused tensor-core path (large M).
//
// 1) Activations: bf16 x[M][K] -> f16 xh[M][K] * 2^-e_m with one power of two
//    per row chosen from the row's max |x| so that the largest magnitude lands
//    in [2^15, 2^16) below the f16 maximum.  A bf16 value (8 significant bits)
//    scaled by a power of two is exactly representable in f16 whenever it stays
//    in the f16 normal range; only entries more than ~2^29 below the row
//    maximum are rounded (to f16 subnormals).  rowscale[m] = 2^e_m undoes the
//    scaling in the epilogue.  Within every 8 consecutive k the f16 copy is
//    stored in the order the dequantizer produces weight pairs in, so that
//    permuting both operands alike leaves every dot product unchanged:
//    (0,4,1,5,2,6,3,7) for 4-bit codes (codes j and j+4 share one 32-bit
//    word's f16x2 pair), (0,2,1,3,4,6,5,7) for 8-bit codes (bytes j and j+2).
// 2) Group parameters: scales/biases [N][G] -> sb[G][N] of (scale, bias) f16
//    pairs, so one K-step's parameters for a run of N rows are contiguous and
//    can be fetched by the tensor memory accelerator.
#pragma once

#include "ql_ptx.cuh"

namespace ql {

// One CTA of kThreads per row.  Pass 1 reads the row for max|x|, keeping up to kCache 8-blocks per
// thread in registers, pass 2 converts them (re-reading, from L2, only what did not fit).  All of a
// thread's pass-1 loads are issued before the first is used.  Two shapes: 128 threads x 5 blocks hold a
// row of up to 5120 elements and let twice as many rows be in flight per SM as 256-thread CTAs (about 4 us
// less on the QKV projection's 4608 x 4608 activations, 20 us on the 2048^2 canvas's 33792 x 4608, on a
// B200); longer rows take 256 threads x 4 blocks, which measured faster there (K = 18432 and 53248).

// The f16 8-block of a bf16 8-block scaled by inv, in the k order the dequantizer of kBits-bit codes
// emits its pairs in.
template <int kBits>
__device__ __forceinline__ uint4 convert8(const uint4 v, float inv) {
    // source order 0..7 = (v.x lo, v.x hi, v.y lo, v.y hi, v.z lo, v.z hi, v.w lo, v.w hi)
    const float f0 = bf16_lo(v.x) * inv, f1 = bf16_hi(v.x) * inv;
    const float f2 = bf16_lo(v.y) * inv, f3 = bf16_hi(v.y) * inv;
    const float f4 = bf16_lo(v.z) * inv, f5 = bf16_hi(v.z) * inv;
    const float f6 = bf16_lo(v.w) * inv, f7 = bf16_hi(v.w) * inv;
    uint4 o;
    if constexpr (kBits == 4) {
        o.x = bits_of(__floats2half2_rn(f0, f4));
        o.y = bits_of(__floats2half2_rn(f1, f5));
        o.z = bits_of(__floats2half2_rn(f2, f6));
        o.w = bits_of(__floats2half2_rn(f3, f7));
    } else {
        static_assert(kBits == 8, "4- or 8-bit codes");
        o.x = bits_of(__floats2half2_rn(f0, f2));
        o.y = bits_of(__floats2half2_rn(f1, f3));
        o.z = bits_of(__floats2half2_rn(f4, f6));
        o.w = bits_of(__floats2half2_rn(f5, f7));
    }
    return o;
}

__device__ __forceinline__ float absmax_bf16x8(const uint4 v, float amax) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // bit-level |.|: NaN patterns compare above every finite value
        amax = fmaxf(amax, fabsf(bf16_lo(w[j])));
        amax = fmaxf(amax, fabsf(bf16_hi(w[j])));
    }
    return amax;
}

// kBits: width of the weight codes the activations will meet (4 or 8), which fixes the k order.
template <int kBits, int kThreads, int kCache>
__global__ void __launch_bounds__(kThreads) convert_x_kernel(const __nv_bfloat16* __restrict__ x,
                                                             __half* __restrict__ xh,
                                                             float* __restrict__ rowscale, int K) {
    ptx::launch_dependents();
    __shared__ float red[kThreads / 32];
    __shared__ int row_exp;
    const int64_t m = blockIdx.x;
    const uint4* src = reinterpret_cast<const uint4*>(x + m * K);   // 8 bf16 per uint4
    uint4* dst = reinterpret_cast<uint4*>(xh + m * K);
    const int n8 = K / 8;

    uint4 v[kCache];
#pragma unroll
    for (int j = 0; j < kCache; ++j) {
        const int i = threadIdx.x + j * kThreads;
        v[j] = i < n8 ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < kCache; ++j) amax = absmax_bf16x8(v[j], amax);
    for (int i = threadIdx.x + kCache * kThreads; i < n8; i += kThreads)
        amax = absmax_bf16x8(__ldg(src + i), amax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = red[0];
        for (int i = 1; i < kThreads / 32; ++i) a = fmaxf(a, red[i]);
        int e = 0;                         // zero, inf or nan rows: no scaling
        if (a > 0.0f && a <= 3.4028235e38f) {
            const int ea = static_cast<int>((__float_as_uint(a) >> 23) & 0xFF) - 127;   // floor(log2 a), a normal
            e = max(ea, -100) - 15;
        }
        row_exp = e;
        rowscale[m] = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);    // 2^e, e in [-115, 112]
    }
    __syncthreads();
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - row_exp) << 23);   // 2^-e, exact
#pragma unroll
    for (int j = 0; j < kCache; ++j) {
        const int i = threadIdx.x + j * kThreads;
        if (i < n8) dst[i] = convert8<kBits>(v[j], inv);
    }
    for (int i = threadIdx.x + kCache * kThreads; i < n8; i += kThreads)
        dst[i] = convert8<kBits>(__ldg(src + i), inv);
    // Launched behind the parameter transpose under programmatic dependent launch, this kernel runs beside
    // it; its last CTA waits for it before finishing, so that this kernel's completion implies both.
    if (blockIdx.x == gridDim.x - 1) ptx::grid_dependency_wait();
}

// sb[g][n] = (scale[n][g], bias[n][g]) through shared memory, one CTA per 32 groups x kTransposeCols
// rows: each thread issues all of its loads (kTransposeCols / 8 rows, scale and bias each) before the
// first is used, so a CTA waits for memory once instead of once per 32 x 32 tile.  The first kernel of a
// fused-path call: it lets the activation conversion start at once (programmatic dependent launch),
// which runs beside it and waits for it only in its last CTA.  grid: (ceil(G / 32), ceil(N / kTransposeCols)).
constexpr int kTransposeCols = 128;

__global__ void __launch_bounds__(256) transpose_params_kernel(const __half* __restrict__ scales,
                                                               const __half* __restrict__ biases,
                                                               uint32_t* __restrict__ sb, int N, int G) {
    ptx::launch_dependents();
    __shared__ uint32_t tile[kTransposeCols][33];
    const int g0 = blockIdx.x * 32, n0 = blockIdx.y * kTransposeCols;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;     // 8 rows per pass
    uint32_t v[kTransposeCols / 8];
#pragma unroll
    for (int j = 0; j < kTransposeCols / 8; ++j) {
        const int n = n0 + ty + 8 * j, g = g0 + tx;
        v[j] = 0;
        if (n < N && g < G) {
            const int64_t i = static_cast<int64_t>(n) * G + g;
            v[j] = static_cast<uint32_t>(__half_as_ushort(scales[i])) |
                   (static_cast<uint32_t>(__half_as_ushort(biases[i])) << 16);
        }
    }
#pragma unroll
    for (int j = 0; j < kTransposeCols / 8; ++j) tile[ty + 8 * j][tx] = v[j];
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int g = g0 + r;
        if (g >= G) break;
#pragma unroll
        for (int c = tx; c < kTransposeCols; c += 32) {
            const int n = n0 + c;
            if (n < N) sb[static_cast<int64_t>(g) * N + n] = tile[c][r];
        }
    }
}

// SwiGLU pair: sb[g][256 w + r] = (scale, bias) of gate row 128 w + r for r < 128, of up row
// 128 w + (r - 128) for r >= 128 (zeros past row I-1), so that one K-step's parameters of tile w are
// one contiguous run of 256 pairs in the fused kernel's row order.  As above, with kTransposeCols = 128
// destination columns per CTA: exactly one 128-row half, so they come from 128 consecutive rows of one
// weight.  grid: (ceil(G / 32), num_w * 2).  Launched first, like transpose_params_kernel.
__global__ void __launch_bounds__(256) transpose_params_pair_kernel(const __half* __restrict__ gate_scales,
                                                                    const __half* __restrict__ gate_biases,
                                                                    const __half* __restrict__ up_scales,
                                                                    const __half* __restrict__ up_biases,
                                                                    uint32_t* __restrict__ sb, int I, int G,
                                                                    int ncols) {
    static_assert(kTransposeCols == 128, "one CTA per 128-row half of a 256-column tile group");
    ptx::launch_dependents();
    __shared__ uint32_t tile[kTransposeCols][33];
    const int g0 = blockIdx.x * 32, c0 = blockIdx.y * kTransposeCols;     // c0: first destination column
    const int w = c0 >> 8;
    const bool up = (c0 & 255) >= 128;
    const int n0 = w * 128;                                                // first source row
    const __half* sc = up ? up_scales : gate_scales;
    const __half* bi = up ? up_biases : gate_biases;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    uint32_t v[kTransposeCols / 8];
#pragma unroll
    for (int j = 0; j < kTransposeCols / 8; ++j) {
        const int n = n0 + ty + 8 * j, g = g0 + tx;
        v[j] = 0;
        if (n < I && g < G) {
            const int64_t i = static_cast<int64_t>(n) * G + g;
            v[j] = static_cast<uint32_t>(__half_as_ushort(sc[i])) | (static_cast<uint32_t>(__half_as_ushort(bi[i])) << 16);
        }
    }
#pragma unroll
    for (int j = 0; j < kTransposeCols / 8; ++j) tile[ty + 8 * j][tx] = v[j];
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int g = g0 + r;
        if (g >= G) break;
#pragma unroll
        for (int c = tx; c < kTransposeCols; c += 32) {
            const int col = c0 + c;
            if (col < ncols) sb[static_cast<int64_t>(g) * ncols + col] = tile[c][r];
        }
    }
}

}  // namespace ql
