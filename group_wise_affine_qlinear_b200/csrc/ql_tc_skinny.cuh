// Weight-streaming tensor-core path for small M (M <= 32): HBM-bound, so the job
// is to read the 4.5-bit weights once at full bandwidth and spend as few
// instructions per weight as possible.
//
// Per 64-group g of a 128-row weight tile, with q the exact codes:
//   D_g[n][t] = sum_{k in g} (128 + q(n,k)) * x[t][k]          (tcgen05.mma, kind::f16, bf16 in, fp32 acc)
//   y[t][n]  += s(n,g) * D_g[n][t] + (b(n,g) - 128 s(n,g)) * xsum_g[t]
// which equals sum_k (s q + b) x (aimarketly "Ideogram-4-IQ4_M", "What IQ4 means
// here": w = scale * q + bias).  128 + q is exact in bf16 (unit 1 at 128), so the
// tensor core sees the exact codes and the exact bf16 activations; the scale and
// bias are applied in fp32 per (row, group, token).  The A operand is built from
// the code nibbles with one shift and one AND-OR per pair of weights and is
// written to tensor memory (tcgen05.st); shared memory carries only the streamed
// code chunks, the activation tiles and the per-chunk scale/bias/xsum tiles.
//
// A word of codes holds k = 0..7 in nibbles 0..7; the builder pairs nibbles j and
// j + 4 (16 bits apart, so one AND-OR per pair), which puts k in the order
// 0,4,1,5,2,6,3,7 along each 8-block of the MMA's reduction dimension.  A small
// prepass kernel writes the activations in that same order, and the per-group
// activation sums xsum_g[t], once for all CTAs.  It runs under programmatic
// dependent launch: the main kernel starts streaming codes at once and waits for
// the prepass only before its first activation load.
//
// Stream-K schedule: the work is cut into chunks of CG consecutive groups of one
// 128-row weight tile (a tile has ceil(G/CG) chunks; a tile's last chunk may be
// partial).  The chunks, tile-major, are split into one equal contiguous run per
// CTA; a run covers at most a few tiles, and each covered tile segment leaves
// fp32 partials [2][tokens][128] in the workspace (one per group parity).  A
// reduce kernel sums, per output, the partials of the CTAs that covered its tile
// in CTA order (deterministic) and rounds to bf16.  The code boxes of a chunk
// bring CG * 32 contiguous bytes of each row, so DRAM sees long row segments.
//
// The builders and the drains run as two copies, on the even and the odd groups
// of the run, and so do the MMA issuers.  Each TMEM slot s (an A stage and an
// accumulator) serves one parity, with one barrier each way: ready[s] (A built
// by the 4 builder warps, accumulator read by the 4 drain warps) and done[s]
// (the slot's MMAs completed).
// Warp roles (608 threads, one CTA per SM; at most 5 warps per SM sub-partition leave 96 registers a thread):
//   warp 0        TMA producer: code chunks (128 rows x CG*32 B, 128B swizzle), scale/bias/xsum tiles,
//                 activation tiles of a chunk (NT x 64 per group, 128B swizzle)
//   warps 1, 2    MMA issuers for even / odd groups (warp 1 also allocates TMEM)
//   warps 3-10    A builders, even groups (3-6) / odd groups (7-10): one weight row per thread
//   warps 11-18   drains, even groups (11-14) / odd groups (15-18): one weight row per thread, fp32
//                 accumulation of s*D + c*xsum over the run
#pragma once

#include "ql_ptx.cuh"

namespace ql {
namespace skinny {

constexpr int BW = 128;
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kWarpTma = 0, kWarpMma0 = 1, kWarpBuild0 = 3, kWarpDrain0 = 11;
constexpr int kThreads = 19 * 32;
constexpr int CG = 8;                    // groups per chunk
constexpr int kBoxGroups = 4;            // groups per code box: 128 bytes of each row (the 128B-swizzle span)
constexpr int NS = 8;                    // TMEM slots (A stage + accumulator), even
constexpr int PR = 4;                    // scale/bias/xsum chunk stages
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBoxBytes = BW * BK / 2 * kBoxGroups;     // 16 KB: one code box
constexpr uint32_t kCBytes = kBoxBytes * (CG / kBoxGroups);  // codes per chunk
constexpr uint32_t kParHalf = BW * CG * 2;                   // one chunk's scales (or biases): [128][CG] f16
static_assert(CG % kBoxGroups == 0 && CG % 8 == 0, "whole code boxes and 16-byte scale rows per chunk");

template <int NT>
struct Layout {
    static constexpr int NC = NT == 16 ? 4 : 3;                          // code chunk stages
    static constexpr int NXC = NT == 16 ? 4 : 3;                         // activation chunk stages
    static constexpr uint32_t kXTile = NT * BK * 2;                      // one group's activation tile
    static constexpr uint32_t kXBytes = CG * kXTile;                     // one chunk's activation tiles
    static constexpr uint32_t kXsBytes = CG * NT * 4;                    // one chunk's xsum rows [CG][NT] fp32
    static constexpr uint32_t kParBytes = 2 * kParHalf + kXsBytes;       // [scales | biases | xsum]
    static constexpr uint32_t kOffC = 0;                                  // [NC][codes], 1 KB aligned
    static constexpr uint32_t kOffX = kOffC + NC * kCBytes;              // [NXC][CG][x tile], 1 KB aligned
    static constexpr uint32_t kOffPar = kOffX + NXC * kXBytes;           // [PR][par]
    static constexpr uint32_t kOffBar = kOffPar + PR * kParBytes;
    static constexpr uint32_t kNumBars = 2 * NC + 2 * PR + 2 * NXC + 2 * NS + 2;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
    static constexpr uint32_t kAccCol = 0;                                // accumulator of slot s at [s*NT, (s+1)*NT)
    static constexpr uint32_t kACol = NS * NT;                            // A stage of slot s at [kACol + 32s, +32)
    static_assert(kCBytes % 1024 == 0 && kXTile % 1024 == 0, "swizzled stage pieces need 1 KB alignment");
    static_assert(kParBytes % 128 == 0, "TMA destinations 128-byte aligned");
    static_assert(kACol + NS * 32 <= kTmemCols, "tensor memory budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Params {
    float* partial;          // [P][segmax][2][M][128] fp32
    const __half* scales;    // [N][G]
    const __half* biases;    // [N][G]
    int param_tma;           // 1: scales/biases arrive as TMA tiles (needs G % CG == 0); 0: direct loads
    int M, N, G, num_w;
    int cpt;                 // chunks per tile = ceil(G / CG)
    int64_t units;           // num_w * cpt chunks
    int segmax;
};

// First unit of CTA c's run (runs are [first(c), first(c+1))).
__host__ __device__ __forceinline__ int64_t run_first(int64_t units, int P, int c) {
    return units * c / P;
}

// Codes word (code j in nibble j) -> 4 words of bf16 pairs (128 + code j, 128 + code j+4), j = 0..3.
__device__ __forceinline__ void codes_to_bf16(uint32_t v, uint32_t* o) {
    o[0] = (v & 0x000F000Fu) | 0x43004300u;
    o[1] = ((v >> 4) & 0x000F000Fu) | 0x43004300u;
    o[2] = ((v >> 8) & 0x000F000Fu) | 0x43004300u;
    o[3] = ((v >> 12) & 0x000F000Fu) | 0x43004300u;
}

// x [M][K] bf16 -> xp [M][K] with each 8-block of k in the order 0,4,1,5,2,6,3,7, and
// xsum[g][t] = sum over group g of x[t][k] in fp32 for t < NT (zero for t >= M).
// One thread per (row, 8-block); the 8 threads of a group are 8 aligned lanes.
__global__ void __launch_bounds__(256) skinny_prepass_kernel(const uint4* __restrict__ x, uint4* __restrict__ xp,
                                                             float* __restrict__ xsum, int M, int K, int NT) {
    ptx::launch_dependents();
    const int kb = K / 8;
    const int64_t total = static_cast<int64_t>(NT) * kb;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const bool in = idx < total;
    const int t = in ? static_cast<int>(idx / kb) : 0;
    const int c = in ? static_cast<int>(idx % kb) : 0;
    float sum = 0.0f;
    if (in && t < M) {
        const uint4 v = x[static_cast<int64_t>(t) * kb + c];     // (k0,k1) (k2,k3) (k4,k5) (k6,k7), low half first
        uint4 o;
        asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(o.x) : "r"(v.x), "r"(v.z));   // (k0, k4)
        asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(o.y) : "r"(v.x), "r"(v.z));   // (k1, k5)
        asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(o.z) : "r"(v.y), "r"(v.w));   // (k2, k6)
        asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(o.w) : "r"(v.y), "r"(v.w));   // (k3, k7)
        xp[static_cast<int64_t>(t) * kb + c] = o;
        sum = ((bf16_lo(v.x) + bf16_hi(v.x)) + (bf16_lo(v.y) + bf16_hi(v.y))) +
              ((bf16_lo(v.z) + bf16_hi(v.z)) + (bf16_lo(v.w) + bf16_hi(v.w)));
    }
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
    if (in && (c & 7) == 0) xsum[static_cast<int64_t>(c >> 3) * NT + t] = sum;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) skinny_kernel(const __grid_constant__ CUtensorMap map_codes,
                                                            const __grid_constant__ CUtensorMap map_x,
                                                            const __grid_constant__ CUtensorMap map_scales,
                                                            const __grid_constant__ CUtensorMap map_biases,
                                                            const __grid_constant__ CUtensorMap map_xsum,
                                                            const Params p) {
    using L = Layout<NT>;
    constexpr int NC = L::NC;
    constexpr int NXC = L::NXC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* c_full = bars;
    uint64_t* c_empty = c_full + NC;
    uint64_t* p_full = c_empty + NC;
    uint64_t* p_empty = p_full + PR;
    uint64_t* x_full = p_empty + PR;
    uint64_t* x_empty = x_full + NXC;
    uint64_t* ready = x_empty + NXC;
    uint64_t* done = ready + NS;
    uint64_t* drain = done + NS;                // two: one per MMA issuer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int P = gridDim.x;
    const int64_t u0 = run_first(p.units, P, blockIdx.x);
    const int64_t u1 = run_first(p.units, P, blockIdx.x + 1);
    const uint32_t nchunks = static_cast<uint32_t>(u1 - u0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NC; ++i) { ptx::mbar_init(&c_full[i], 1); ptx::mbar_init(&c_empty[i], 8); }
        for (int i = 0; i < PR; ++i) { ptx::mbar_init(&p_full[i], 1); ptx::mbar_init(&p_empty[i], 8); }
        for (int i = 0; i < NXC; ++i) { ptx::mbar_init(&x_full[i], 1); ptx::mbar_init(&x_empty[i], 2); }
        for (int i = 0; i < NS; ++i) { ptx::mbar_init(&ready[i], 8); ptx::mbar_init(&done[i], 1); }
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(drain + 1, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) {
        ptx::prefetch_tensormap(&map_codes);
        ptx::prefetch_tensormap(&map_x);
        ptx::prefetch_tensormap(&map_xsum);
        if (p.param_tma) {
            ptx::prefetch_tensormap(&map_scales);
            ptx::prefetch_tensormap(&map_biases);
        }
    }
    if (warp == kWarpMma0) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    ptx::launch_dependents();

    // chunk u -> tile w = u / cpt, groups g = (u % cpt) * CG + q, q < ng.  Groups are numbered
    // gi along the run; group gi belongs to the copies of parity gi & 1 and uses TMEM slot gi % NS.
    auto chunk_groups = [&](int64_t u, int& w, int& g0, int& ng) {
        w = static_cast<int>(u / p.cpt);
        g0 = static_cast<int>(u % p.cpt) * CG;
        ng = min(CG, p.G - g0);
    };

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t ci = 0, pi = 0, xi = 0;     // chunks whose codes / parameters / activations were issued
            auto issue_codes = [&](uint32_t i) -> bool {
                int w, g0, ng;
                chunk_groups(u0 + i, w, g0, ng);
                const int s = static_cast<int>(i % NC);
                if (!ptx::mbar_wait(&c_empty[s], ((i / NC) & 1u) ^ 1u, abort_flag)) return false;
                uint8_t* st = smem + L::kOffC + s * kCBytes;
                ptx::mbar_arrive_expect_tx(&c_full[s], kCBytes);
#pragma unroll
                for (int bx = 0; bx < CG / kBoxGroups; ++bx)   // consecutive boxes: long contiguous row segments
                    ptx::tma_load_2d(st + bx * kBoxBytes, &map_codes, &c_full[s], (g0 + bx * kBoxGroups) * (BK / 8), w * BW);
                return true;
            };
            // the codes do not depend on the prepass: start streaming them at once
            bool ok = true;
            while (ok && ci < nchunks && ci < static_cast<uint32_t>(NC)) {
                ok = issue_codes(ci);
                if (ok) ++ci;
            }
            ptx::grid_dependency_wait();
            for (uint32_t i = 0; i < nchunks && ok; ++i) {
                int w, g0, ng;
                chunk_groups(u0 + i, w, g0, ng);
                // scales, biases and activation sums of the chunk
                const int pr = static_cast<int>(i % PR);
                if (!ptx::mbar_wait(&p_empty[pr], ((i / PR) & 1u) ^ 1u, abort_flag)) break;
                uint8_t* pt = smem + L::kOffPar + pr * L::kParBytes;
                ptx::mbar_arrive_expect_tx(&p_full[pr], (p.param_tma ? 2 * kParHalf : 0u) + L::kXsBytes);
                if (p.param_tma) {
                    ptx::tma_load_2d(pt, &map_scales, &p_full[pr], g0, w * BW);
                    ptx::tma_load_2d(pt + kParHalf, &map_biases, &p_full[pr], g0, w * BW);
                }
                ptx::tma_load_2d(pt + 2 * kParHalf, &map_xsum, &p_full[pr], 0, g0);   // rows past G read zeros
                ++pi;
                // activation tiles of the chunk
                const int xc = static_cast<int>(i % NXC);
                if (!ptx::mbar_wait(&x_empty[xc], ((i / NXC) & 1u) ^ 1u, abort_flag)) break;
                ptx::mbar_arrive_expect_tx(&x_full[xc], static_cast<uint32_t>(ng) * L::kXTile);
                for (int q = 0; q < ng; ++q)
                    ptx::tma_load_2d(smem + L::kOffX + xc * L::kXBytes + q * L::kXTile, &map_x, &x_full[xc], (g0 + q) * BK, 0);
                ++xi;
                // codes run NC chunks ahead
                if (ci < nchunks) {
                    if (!issue_codes(ci)) break;
                    ++ci;
                }
            }
            // never leave the CTA with bulk copies still landing in its shared memory
            for (uint32_t j = (ci > static_cast<uint32_t>(NC) ? ci - NC : 0u); j < ci; ++j)
                ptx::mbar_wait(&c_full[j % NC], (j / NC) & 1u, nullptr);
            for (uint32_t j = (pi > static_cast<uint32_t>(PR) ? pi - PR : 0u); j < pi; ++j)
                ptx::mbar_wait(&p_full[j % PR], (j / PR) & 1u, nullptr);
            for (uint32_t j = (xi > static_cast<uint32_t>(NXC) ? xi - NXC : 0u); j < xi; ++j)
                ptx::mbar_wait(&x_full[j % NXC], (j / NXC) & 1u, nullptr);
        }
    } else if (warp == kWarpMma0 || warp == kWarpMma0 + 1) {
        // ---------------------------------------------------------------- MMA issuers (even / odd groups)
        // The whole warp runs the loop, so the addresses stay warp-uniform; lane 0 issues.
        const uint32_t par = static_cast<uint32_t>(warp - kWarpMma0);
        constexpr uint32_t idesc = ptx::idesc_f16(BW, NT, true);
        const uint32_t x_base = ptx::smem_addr(smem + L::kOffX);
        uint32_t gi = 0;
        bool ok = true;
        for (uint32_t i = 0; i < nchunks && ok; ++i) {
            int w, g0, ng;
            chunk_groups(u0 + i, w, g0, ng);
            const int xc = static_cast<int>(i % NXC);
            bool got = ptx::mbar_wait(&x_full[xc], (i / NXC) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            for (int q = static_cast<int>((par - gi) & 1u); q < ng; q += 2) {
                const uint32_t gq = gi + static_cast<uint32_t>(q);
                const int sl = static_cast<int>(gq % NS);
                got = ptx::mbar_wait(&ready[sl], (gq / NS) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                const uint32_t xa = x_base + static_cast<uint32_t>(xc) * L::kXBytes + static_cast<uint32_t>(q) * L::kXTile;
                const uint32_t d = tmem_base + L::kAccCol + static_cast<uint32_t>(sl * NT);
                const uint32_t a_tm = tmem_base + L::kACol + 32u * static_cast<uint32_t>(sl);
                if (lane == 0) {
#pragma unroll
                    for (int u = 0; u < BK / UK; ++u)
                        ptx::mma_f16_ts(d, a_tm + u * (UK / 2), ptx::sdesc_sw128(xa + u * UK * 2), idesc, u != 0);
                    ptx::mma_commit(&done[sl]);
                }
                __syncwarp();
            }
            if (ok && lane == 0) ptx::mma_commit(&x_empty[xc]);
            __syncwarp();
            gi += static_cast<uint32_t>(ng);
        }
        if (lane == 0) ptx::mma_commit(drain + par);
        __syncwarp();
        ptx::mbar_wait(drain + par, 0, nullptr);
    } else if (warp >= kWarpBuild0 && warp < kWarpDrain0) {
        // ---------------------------------------------------------------- A builders (even / odd groups)
        const uint32_t par = static_cast<uint32_t>((warp - kWarpBuild0) >> 2);
        const int quarter = warp & 3;                      // TMEM lanes 32*quarter.. belong to this warp
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t gi = 0;
        bool ok = true;
        for (uint32_t i = 0; i < nchunks && ok; ++i) {
            int w, g0, ng;
            chunk_groups(u0 + i, w, g0, ng);
            const int s = static_cast<int>(i % NC);
            bool got = ptx::mbar_wait(&c_full[s], (i / NC) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            // this copy's groups of the chunk are q = q0, q0 + 2, ...  Row r's 32 code bytes of group q
            // sit in box q / 4 at the 16-byte pieces 2 (q % 4) and 2 (q % 4) + 1, stored with the
            // 128-byte swizzle (piece c at c ^ (r % 8)), so every 8 lanes of a load touch 8 bank groups.
            const int q0 = static_cast<int>((par - gi) & 1u);
            const uint8_t* crow = smem + L::kOffC + s * kCBytes + r * 128;
            uint4 cw[CG];
#pragma unroll
            for (int k = 0; k < CG / 2; ++k) {
                const int q = q0 + 2 * k;
                if (q < ng) {
                    const uint8_t* bxp = crow + (q / kBoxGroups) * kBoxBytes;
                    const int c = 2 * (q % kBoxGroups);
                    cw[2 * k] = *reinterpret_cast<const uint4*>(bxp + ((c ^ (r & 7)) << 4));
                    cw[2 * k + 1] = *reinterpret_cast<const uint4*>(bxp + (((c + 1) ^ (r & 7)) << 4));
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&c_empty[s]);
#pragma unroll
            for (int k = 0; k < CG / 2; ++k) {
                const int q = q0 + 2 * k;
                if (q >= ng) break;
                const uint32_t gq = gi + static_cast<uint32_t>(q);
                const int sl = static_cast<int>(gq % NS);
                const uint4 c0 = cw[2 * k], c1 = cw[2 * k + 1];
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t av[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) codes_to_bf16(words[c], &av[4 * c]);
                // the slot's previous MMAs must have finished reading its A stage
                got = ptx::mbar_wait(&done[sl], ((gq / NS) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                ptx::tmem_st_32x32b_x32(tmem_base + lane_addr + L::kACol + 32u * sl, av);
                ptx::tmem_wait_st();
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&ready[sl]);
            }
            gi += static_cast<uint32_t>(ng);
        }
    } else if (warp >= kWarpDrain0) {
        // ---------------------------------------------------------------- drains (even / odd groups)
        const uint32_t par = static_cast<uint32_t>((warp - kWarpDrain0) >> 2);
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        // a slot's first use has no accumulator to read back: arrive for it in advance
        if (lane == 0)
            for (int sl = static_cast<int>(par); sl < NS; sl += 2) ptx::mbar_arrive(&ready[sl]);
        float yacc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) yacc[t] = 0.0f;
        const int w_first = static_cast<int>(u0 / p.cpt);
        uint32_t gi = 0;
        bool ok = true;
        for (uint32_t i = 0; i < nchunks && ok; ++i) {
            int w, g0, ng;
            chunk_groups(u0 + i, w, g0, ng);
            const int n = w * BW + r;
            const int q0 = static_cast<int>((par - gi) & 1u);
            const int pr = static_cast<int>(i % PR);
            bool got = ptx::mbar_wait(&p_full[pr], (i / PR) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            const uint8_t* pt = smem + L::kOffPar + pr * L::kParBytes;
            // this copy's scales and biases of row r (groups q0, q0 + 2, ...)
            __half sv[CG / 2], bv[CG / 2];
            if (p.param_tma) {
                __align__(16) __half sa[CG], ba[CG];
#pragma unroll
                for (int c = 0; c < CG / 8; ++c) {
                    *reinterpret_cast<uint4*>(sa + 8 * c) = reinterpret_cast<const uint4*>(pt + r * CG * 2)[c];
                    *reinterpret_cast<uint4*>(ba + 8 * c) = reinterpret_cast<const uint4*>(pt + kParHalf + r * CG * 2)[c];
                }
#pragma unroll
                for (int k = 0; k < CG / 2; ++k) {
                    sv[k] = q0 ? sa[2 * k + 1] : sa[2 * k];
                    bv[k] = q0 ? ba[2 * k + 1] : ba[2 * k];
                }
            } else {
#pragma unroll
                for (int k = 0; k < CG / 2; ++k) {
                    const int q = q0 + 2 * k;
                    const bool in = n < p.N && q < ng;
                    sv[k] = in ? __ldg(p.scales + static_cast<int64_t>(n) * p.G + g0 + q) : __float2half_rn(0.0f);
                    bv[k] = in ? __ldg(p.biases + static_cast<int64_t>(n) * p.G + g0 + q) : __float2half_rn(0.0f);
                }
            }
            const float* xsp = reinterpret_cast<const float*>(pt + 2 * kParHalf);     // [CG][NT]
#pragma unroll
            for (int k = 0; k < CG / 2; ++k) {
                const int q = q0 + 2 * k;
                if (q >= ng) break;
                const uint32_t gq = gi + static_cast<uint32_t>(q);
                const int sl = static_cast<int>(gq % NS);
                float sc = 0.0f, cc = 0.0f;
                if (n < p.N) {
                    sc = __half2float(sv[k]);
                    cc = fmaf(-128.0f, sc, __half2float(bv[k]));
                }
                // the activation-sum term first (few live registers), then the tensor-core sums
                const float4* xsq = reinterpret_cast<const float4*>(xsp + q * NT);
#pragma unroll
                for (int t4 = 0; t4 < NT / 4; ++t4) {
                    const float4 v = xsq[t4];
                    yacc[4 * t4 + 0] = fmaf(cc, v.x, yacc[4 * t4 + 0]);
                    yacc[4 * t4 + 1] = fmaf(cc, v.y, yacc[4 * t4 + 1]);
                    yacc[4 * t4 + 2] = fmaf(cc, v.z, yacc[4 * t4 + 2]);
                    yacc[4 * t4 + 3] = fmaf(cc, v.w, yacc[4 * t4 + 3]);
                }
                got = ptx::mbar_wait(&done[sl], (gq / NS) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                uint32_t dv[NT];
                if constexpr (NT == 32) {
                    ptx::tmem_ld_32x32b_x32(tmem_base + lane_addr + L::kAccCol + static_cast<uint32_t>(sl * NT),
                                            *reinterpret_cast<uint32_t(*)[32]>(dv));
                } else {
                    ptx::tmem_ld_32x32b_x16(tmem_base + lane_addr + L::kAccCol + static_cast<uint32_t>(sl * NT),
                                            *reinterpret_cast<uint32_t(*)[16]>(dv));
                }
                ptx::tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < NT; ++t) yacc[t] = fmaf(sc, __uint_as_float(dv[t]), yacc[t]);
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&ready[sl]);
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&p_empty[pr]);
            gi += static_cast<uint32_t>(ng);
            // end of this tile's segment: write this copy's partial and start over
            const bool seg_end = (i + 1 == nchunks) || ((u0 + i + 1) % p.cpt == 0);
            if (seg_end) {
                float* dst = p.partial +
                             (((static_cast<int64_t>(blockIdx.x) * p.segmax + (w - w_first)) * 2 + par) * p.M) * BW;
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (t < p.M) dst[static_cast<int64_t>(t) * BW + r] = yacc[t];
                    yacc[t] = 0.0f;
                }
            }
        }
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma0) {
        __syncwarp();
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// y[t][n] = sum over the CTAs whose runs cover tile n/128, in CTA order, of their two partials for that tile.
template <bool kBf16Out>
__global__ void __launch_bounds__(256) skinny_reduce_kernel(const float* __restrict__ partial, void* __restrict__ y,
                                                            int M, int N, int cpt, int64_t units, int P, int segmax) {
    ptx::grid_dependency_wait();
    const int64_t total = static_cast<int64_t>(M) * N;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int t = static_cast<int>(e / N), n = static_cast<int>(e % N);
        const int w = n / BW, r = n % BW;
        // CTAs whose run of chunks [first(c), first(c+1)) meets [w*cpt, (w+1)*cpt)
        const int64_t lo = static_cast<int64_t>(w) * cpt, hi = lo + cpt;
        int c = static_cast<int>((lo * P) / units);
        while (c > 0 && run_first(units, P, c) > lo) --c;
        while (c + 1 <= P && run_first(units, P, c + 1) <= lo) ++c;
        float acc = 0.0f;
        for (; c < P && run_first(units, P, c) < hi; ++c) {
            if (run_first(units, P, c + 1) <= run_first(units, P, c)) continue;      // empty run
            const int w_first = static_cast<int>(run_first(units, P, c) / cpt);
            const int64_t seg = (static_cast<int64_t>(c) * segmax + (w - w_first)) * 2;
            acc += partial[((seg + 0) * M + t) * BW + r];
            acc += partial[((seg + 1) * M + t) * BW + r];
        }
        if constexpr (kBf16Out) {
            reinterpret_cast<__nv_bfloat16*>(y)[e] = __float2bfloat16_rn(acc);
        } else {
            reinterpret_cast<float*>(y)[e] = acc;
        }
    }
}

}  // namespace skinny
}  // namespace ql
