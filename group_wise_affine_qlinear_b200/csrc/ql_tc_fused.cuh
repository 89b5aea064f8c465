// Fused-dequant tensor-core GEMM for large M (tcgen05, TMEM accumulators).
//
// y[m][n] = rowscale[m] * sum_k xh[m][k] * wh(n, k)
//   xh    f16 activations prescaled per row by a power of two (prepass)
//   wh    RN_f16(s * q + b): the affine grid of aimarketly "Ideogram-4-IQ4_M",
//         "What IQ4 means here", formed by one fused f16x2 multiply-add from the
//         exact code q, i.e. rounded once
// Operands are f16 (both A and B must share a type in kind::f16); the
// accumulator is fp32 in tensor memory.  One K-step is exactly one 64-wide
// quantization group, so every weight row needs one (scale, bias) pair per step.
//
// Tile: 128 tokens (TMEM lanes) x 256 weight rows (TMEM columns) x 64 k.
// Warp roles of one persistent CTA per SM:
//   warps 0-7   dequantizers: one weight row each per K-step; read the 32 code
//               bytes and the (scale, bias) pair TMA brought in, write the f16
//               B tile in the K-major 128-byte-swizzle layout the MMA reads
//   warp 8      TMA producer: activation tile (swizzled), code tile, parameter tile
//   warp 9      TMEM allocator and single-thread MMA issuer
//   warps 10-13 epilogue: TMEM -> registers -> rowscale -> bf16/fp32 -> global
// Two rings decouple the roles: the TMA ring (activations, codes, parameters)
// and the B ring (dequantized tiles).  Two TMEM accumulators (2 x 256 columns)
// let the epilogue of one tile overlap the main loop of the next.
#pragma once

#include "ql_ptx.cuh"

namespace ql {
namespace fused {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int NS_T = 4;
constexpr int NS_B = 3;
constexpr int kDequantWarps = BN / 32;                  // one row per thread
constexpr int kWarpTma = kDequantWarps;                 // 8
constexpr int kWarpMma = kDequantWarps + 1;             // 9
constexpr int kWarpEpi0 = kDequantWarps + 2;            // 10..13 (ids % 4 = 2,3,0,1: every TMEM quarter once)
constexpr int kThreads = (kDequantWarps + 2 + 4) * 32;  // 448
constexpr uint32_t kTmemCols = 2 * BN;                  // 512

constexpr uint32_t kABytes = BM * BK * 2;               // 16 KB
constexpr uint32_t kBBytes = BN * BK * 2;               // 32 KB
constexpr uint32_t kCBytes = BN * BK / 2;               // 8 KB of codes
constexpr uint32_t kPBytes = BN * 4;                    // 1 KB of (scale, bias)
constexpr uint32_t kTxBytes = kABytes + kCBytes + kPBytes;

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + NS_T * kABytes;
constexpr uint32_t kOffC = kOffB + NS_B * kBBytes;
constexpr uint32_t kOffP = kOffC + NS_T * kCBytes;
constexpr uint32_t kOffBar = kOffP + NS_T * kPBytes;
constexpr uint32_t kNumBars = 2 * NS_T + 2 * NS_B + 4 + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack

static_assert(kOffB % 1024 == 0 && kBBytes % 1024 == 0 && kABytes % 1024 == 0, "swizzle atoms need 1 KB alignment");

struct Params {
    float* rowscale;      // [M] 2^e_m
    void* y;              // [M][N] bf16 or fp32
    int M, N, G;
    int num_m, num_n;
};

__device__ __forceinline__ void tile_coords(int t, int num_n, int& m_blk, int& n_blk) {
    // n fastest: a wave of CTAs shares a few activation row-blocks (streamed from HBM
    // once) and sweeps the whole (L2-resident) packed weight.
    m_blk = t / num_n;
    n_blk = t - m_blk * num_n;
}

// Dequantize one code word (8 codes, k order 0..7) into 4 f16x2 words holding the
// pairs (0,4), (1,5), (2,6), (3,7).  A nibble at bits 0-3 / 16-19 ORed into 1024.0
// (0x6400, unit in the last place 1) gives 1024 + q exactly; a nibble at bits
// 4-7 / 20-23 ORed into 64.0 (0x5400, unit 1/16) gives 64 + q exactly.
// Subtracting the magic leaves q exactly; one fused f16x2 FMA then forms
// RN_f16(s*q + b).
__device__ __forceinline__ uint4 dequant_word(uint32_t v, __half2 s2, __half2 b2) {
    const uint32_t v8 = v >> 8;
    uint32_t p0, p1, p2, p3;
    asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(p0) : "r"(v));
    asm("lop3.b32 %0, %1, 0x00F000F0, 0x54005400, 0xEA;" : "=r"(p1) : "r"(v));
    asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(p2) : "r"(v8));
    asm("lop3.b32 %0, %1, 0x00F000F0, 0x54005400, 0xEA;" : "=r"(p3) : "r"(v8));
    const __half2 m1024 = half2_of(0x64006400u);
    const __half2 m64 = half2_of(0x54005400u);
    uint4 o;
    o.x = bits_of(__hfma2(__hsub2(half2_of(p0), m1024), s2, b2));
    o.y = bits_of(__hfma2(__hsub2(half2_of(p1), m64), s2, b2));
    o.z = bits_of(__hfma2(__hsub2(half2_of(p2), m1024), s2, b2));
    o.w = bits_of(__hfma2(__hsub2(half2_of(p3), m64), s2, b2));
    return o;
}

template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads, 1) fused_gemm_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_codes,
    const __grid_constant__ CUtensorMap map_params, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* tfull = bars;
    uint64_t* tempty = tfull + NS_T;
    uint64_t* bfull = tempty + NS_T;
    uint64_t* bempty = bfull + NS_B;
    uint64_t* afull = bempty + NS_B;
    uint64_t* aempty = afull + 2;
    uint64_t* drain = aempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.num_m * p.num_n;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS_T; ++i) { ptx::mbar_init(&tfull[i], 1); ptx::mbar_init(&tempty[i], 1); }
        for (int i = 0; i < NS_B; ++i) { ptx::mbar_init(&bfull[i], kDequantWarps); ptx::mbar_init(&bempty[i], 1); }
        for (int i = 0; i < 2; ++i) { ptx::mbar_init(&afull[i], 1); ptx::mbar_init(&aempty[i], 4); }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) {
        ptx::prefetch_tensormap(&map_x);
        ptx::prefetch_tensormap(&map_codes);
        ptx::prefetch_tensormap(&map_params);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < kDequantWarps) {
        // ---------------------------------------------------------------- dequantizers
        const int r = threadIdx.x;                 // weight row within the tile
        int ts = 0, bs = 0;
        uint32_t tph = 0, bph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < p.G; ++kb) {
                bool got = ptx::mbar_wait(&tfull[ts], tph, abort_flag);
                got = got && ptx::mbar_wait(&bempty[bs], bph ^ 1, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                const uint4* crow = reinterpret_cast<const uint4*>(smem + kOffC + ts * kCBytes + r * 32);
                const uint4 c0 = crow[0], c1 = crow[1];
                const uint32_t sb = reinterpret_cast<const uint32_t*>(smem + kOffP + ts * kPBytes)[r];
                const __half2 sb2 = half2_of(sb);
                const __half2 s2 = __low2half2(sb2);
                const __half2 b2 = __high2half2(sb2);
                uint8_t* brow = smem + kOffB + bs * kBBytes + r * 128;
                const uint32_t sw = static_cast<uint32_t>(r & 7);
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    *reinterpret_cast<uint4*>(brow + ((c ^ sw) << 4)) = dequant_word(words[c], s2, b2);
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bfull[bs]);
                if (++ts == NS_T) { ts = 0; tph ^= 1; }
                if (++bs == NS_B) { bs = 0; bph ^= 1; }
            }
        }
    } else if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int ts = 0;
            uint32_t tph = 0;
            uint32_t issued[NS_T] = {};
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int m_blk, n_blk;
                tile_coords(t, p.num_n, m_blk, n_blk);
                for (int kb = 0; kb < p.G; ++kb) {
                    if (!ptx::mbar_wait(&tempty[ts], tph ^ 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&tfull[ts], kTxBytes);
                    ptx::tma_load_2d(smem + kOffA + ts * kABytes, &map_x, &tfull[ts], kb * BK, m_blk * BM);
                    ptx::tma_load_2d(smem + kOffC + ts * kCBytes, &map_codes, &tfull[ts], kb * (BK / 8), n_blk * BN);
                    ptx::tma_load_2d(smem + kOffP + ts * kPBytes, &map_params, &tfull[ts], n_blk * BN, kb);
                    ++issued[ts];
                    if (++ts == NS_T) { ts = 0; tph ^= 1; }
                }
            }
            // Never leave the CTA with bulk copies still landing in its shared memory.
            for (int i = 0; i < NS_T; ++i) {
                if (issued[i] > 0) ptx::mbar_wait(&tfull[i], (issued[i] - 1) & 1, nullptr);
            }
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_f16(BM, BN, false);
            int ts = 0, bs = 0;
            uint32_t tph = 0, bph = 0;
            bool ok = true;
            int j = 0;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++j) {
                const int a = j & 1;
                if (!ptx::mbar_wait(&aempty[a], ((j >> 1) & 1) ^ 1, abort_flag)) break;
                ptx::tc_fence_after_sync();
                const uint32_t d = tmem_base + static_cast<uint32_t>(a * BN);
                for (int kb = 0; kb < p.G; ++kb) {
                    if (!ptx::mbar_wait(&tfull[ts], tph, abort_flag)) { ok = false; break; }
                    if (!ptx::mbar_wait(&bfull[bs], bph, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after_sync();
                    const uint32_t a_addr = ptx::smem_addr(smem + kOffA + ts * kABytes);
                    const uint32_t b_addr = ptx::smem_addr(smem + kOffB + bs * kBBytes);
#pragma unroll
                    for (int u = 0; u < BK / UK; ++u) {
                        ptx::mma_f16_ss(d, ptx::sdesc_sw128(a_addr + u * UK * 2), ptx::sdesc_sw128(b_addr + u * UK * 2),
                                        idesc, (kb | u) != 0);
                    }
                    ptx::mma_commit(&tempty[ts]);
                    ptx::mma_commit(&bempty[bs]);
                    if (++ts == NS_T) { ts = 0; tph ^= 1; }
                    if (++bs == NS_B) { bs = 0; bph ^= 1; }
                }
                if (ok) ptx::mma_commit(&afull[a]);
            }
            // Wait until every MMA this thread issued has finished before TMEM is released.
            ptx::mma_commit(drain);
            ptx::mbar_wait(drain, 0, nullptr);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
        int j = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++j) {
            const int a = j & 1;
            const bool got = ptx::mbar_wait(&afull[a], (j >> 1) & 1, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            ptx::tc_fence_after_sync();
            int m_blk, n_blk;
            tile_coords(t, p.num_n, m_blk, n_blk);
            const int m = m_blk * BM + quarter * 32 + lane;
            const float rs = (m < p.M) ? p.rowscale[m] : 0.0f;
            const uint32_t taddr = tmem_base + static_cast<uint32_t>(a * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
            for (int chunk = 0; chunk < BN / 32; ++chunk) {
                uint32_t r[32];
                ptx::tmem_ld_32x32b_x32(taddr + chunk * 32, r);
                ptx::tmem_wait_ld();
                const int n0 = n_blk * BN + chunk * 32;
                if (m < p.M) {
                    if constexpr (kBf16Out) {
                        __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(p.y) + static_cast<int64_t>(m) * p.N;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (n0 + 8 * i < p.N) {
                                uint4 o;
                                o.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * rs, __uint_as_float(r[8 * i + 1]) * rs);
                                o.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * rs, __uint_as_float(r[8 * i + 3]) * rs);
                                o.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * rs, __uint_as_float(r[8 * i + 5]) * rs);
                                o.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * rs, __uint_as_float(r[8 * i + 7]) * rs);
                                *reinterpret_cast<uint4*>(yrow + n0 + 8 * i) = o;
                            }
                        }
                    } else {
                        float* yrow = reinterpret_cast<float*>(p.y) + static_cast<int64_t>(m) * p.N;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            if (n0 + 4 * i < p.N) {
                                *reinterpret_cast<float4*>(yrow + n0 + 4 * i) =
                                    make_float4(__uint_as_float(r[4 * i + 0]) * rs, __uint_as_float(r[4 * i + 1]) * rs,
                                                __uint_as_float(r[4 * i + 2]) * rs, __uint_as_float(r[4 * i + 3]) * rs);
                            }
                        }
                    }
                }
            }
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&aempty[a]);
        }
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        __syncwarp();
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace fused
}  // namespace ql
