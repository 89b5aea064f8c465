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
// the code nibbles with two byte permutes and an OR per pair of weights and is
// written to tensor memory (tcgen05.st); shared memory carries only the streamed
// code chunks, the small activation tiles and the scale/bias tiles.
//
// Stream-K schedule: the work is cut into chunks of CG consecutive groups of one
// 128-row weight tile (a tile has ceil(G/CG) chunks; a tile's last chunk may be
// partial).  The chunks, tile-major, are split into one equal contiguous run per
// CTA; a run covers at most a few tiles, and each covered tile segment leaves
// fp32 partials [2][tokens][128] in the workspace (one per group parity).  A
// second kernel sums, per output, the partials of the CTAs that covered its tile
// in CTA order (deterministic) and rounds to bf16.  The code boxes of a chunk
// bring CG * 32 contiguous bytes of each row, so DRAM sees long row segments.
//
// Every role works group by group through a serial chain of waits, tensor-memory
// accesses and arithmetic, so each role runs twice: one copy takes the even
// groups of the run, the other the odd ones, and the two chains overlap.  The
// code chunks and the activation tiles have rings of their own, so a code stage
// is free as soon as the builders have read it into registers.
// Warp roles (640 threads, one CTA per SM; 5 warps per SM sub-partition leave 96 registers a thread):
//   warp 0        TMA producer: code chunks (128 rows x CG*32 B, 128B swizzle), scale/bias tiles,
//                 activation tiles (NT x 64 per group, 128B swizzle)
//   warps 1, 2    MMA issuers for even / odd groups (warp 1 also allocates TMEM)
//   warp 3        per-group activation sums xsum_g[t]
//   warps 4-11    A builders, even groups (4-7) / odd groups (8-11): one weight row per thread,
//                 codes -> bf16 (128+q) pairs -> TMEM
//   warps 12-19   drain, even (12-15) / odd (16-19): one weight row per thread, fp32
//                 accumulation of s*D + c*xsum over the run
#pragma once

#include "ql_ptx.cuh"

namespace ql {
namespace skinny {

constexpr int BW = 128;
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kWarpTma = 0, kWarpMma0 = 1, kWarpXsum = 3, kWarpBuild0 = 4, kWarpDrain0 = 12;
constexpr int kThreads = 20 * 32;
constexpr int CG = 8;                    // groups per code chunk, a multiple of 8
constexpr int kBoxGroups = 4;            // groups per code box: 128 bytes of each row (the 128B-swizzle span)
constexpr int NC = 4;                    // code chunk stages
constexpr int PR = 4;                    // scale/bias chunk stages
constexpr int NA = 4;                    // TMEM A stages (32 columns each), even
constexpr int ND = 8;                    // TMEM accumulator buffers (NT columns each), even
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBoxBytes = BW * BK / 2 * kBoxGroups;     // 16 KB: one code box
constexpr uint32_t kCBytes = kBoxBytes * (CG / kBoxGroups);  // codes per chunk
constexpr uint32_t kParHalf = BW * CG * 2;                   // one chunk's scales (or biases): [128][CG] f16
constexpr uint32_t kParBytes = 2 * kParHalf;
static_assert(CG % kBoxGroups == 0 && CG % 8 == 0, "whole code boxes and 16-byte scale rows per chunk");
static_assert(NA % 2 == 0 && ND % 2 == 0, "ring slots of one group parity only");

template <int NT>
struct Layout {
    static constexpr uint32_t kXBytes = NT * BK * 2;                    // one group's activation tile
    static constexpr int NX = NT == 16 ? 24 : 20;                       // activation stages (one group each), even
    static constexpr uint32_t kOffC = 0;                                 // [NC][codes], 1 KB aligned
    static constexpr uint32_t kOffX = kOffC + NC * kCBytes;             // [NX][x tile], 1 KB aligned
    static constexpr uint32_t kOffPar = kOffX + NX * kXBytes;           // [PR][scales|biases][128][CG]
    static constexpr uint32_t kOffXs = kOffPar + PR * kParBytes;        // xsum ring [ND][NT] fp32
    static constexpr uint32_t kOffBar = kOffXs + ND * NT * 4;
    static constexpr uint32_t kNumBars = 2 * NC + 2 * PR + 2 * NX + 2 * NA + 3 * ND + 2;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
    static constexpr uint32_t kAccCol = 0;                               // D buffer j at [j*NT, (j+1)*NT)
    static constexpr uint32_t kACol = ND * NT;                           // A stage a at [kACol + 32a, +32)
    static_assert(kCBytes % 1024 == 0 && kXBytes % 1024 == 0, "stage pieces need 1 KB alignment");
    static_assert(NX % 2 == 0, "ring slots of one group parity only");
    static_assert(kACol + NA * 32 <= kTmemCols, "tensor memory budget");
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

// Codes word (8 codes, k order 0..7) -> 4 words of bf16 pairs (128+q_2t, 128+q_2t+1), k order kept.
// prmt selector nibble = byte index (0-3 from a, 4-7 from b); bit 3 set replicates the
// selected byte's sign bit, which is 0 for a code byte, giving 0x00.
__device__ __forceinline__ void codes_to_bf16(uint32_t v, uint32_t* o) {
    const uint32_t lo = v & 0x0F0F0F0Fu;            // q0 q2 q4 q6
    const uint32_t hi = (v >> 4) & 0x0F0F0F0Fu;     // q1 q3 q5 q7
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const uint32_t sel = static_cast<uint32_t>(t) | (static_cast<uint32_t>(8 | t) << 4) |
                             (static_cast<uint32_t>(4 + t) << 8) | (static_cast<uint32_t>(12 + t) << 12);
        uint32_t w;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(w) : "r"(lo), "r"(hi), "r"(sel));
        o[t] = w | 0x43004300u;
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) skinny_kernel(const __grid_constant__ CUtensorMap map_codes,
                                                            const __grid_constant__ CUtensorMap map_x,
                                                            const __grid_constant__ CUtensorMap map_scales,
                                                            const __grid_constant__ CUtensorMap map_biases,
                                                            const Params p) {
    using L = Layout<NT>;
    constexpr int NX = L::NX;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* c_full = bars;
    uint64_t* c_empty = c_full + NC;
    uint64_t* p_full = c_empty + NC;
    uint64_t* p_empty = p_full + PR;
    uint64_t* x_full = p_empty + PR;
    uint64_t* x_empty = x_full + NX;
    uint64_t* a_full = x_empty + NX;
    uint64_t* a_empty = a_full + NA;
    uint64_t* d_full = a_empty + NA;
    uint64_t* d_empty = d_full + ND;
    uint64_t* xs_full = d_empty + ND;
    uint64_t* drain = xs_full + ND;             // two: one per MMA issuer
    float* xs = reinterpret_cast<float*>(smem + L::kOffXs);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int P = gridDim.x;
    const int64_t u0 = run_first(p.units, P, blockIdx.x);
    const int64_t u1 = run_first(p.units, P, blockIdx.x + 1);
    const uint32_t nchunks = static_cast<uint32_t>(u1 - u0);

    if (threadIdx.x == 0) {
        // a code stage is free once all 8 builder warps hold it in registers
        for (int i = 0; i < NC; ++i) { ptx::mbar_init(&c_full[i], 1); ptx::mbar_init(&c_empty[i], 8); }
        for (int i = 0; i < PR; ++i) { ptx::mbar_init(&p_full[i], 1); ptx::mbar_init(&p_empty[i], 8); }
        // an activation stage is free once its MMAs (one commit) and the xsum warp are done with it
        for (int i = 0; i < NX; ++i) { ptx::mbar_init(&x_full[i], 1); ptx::mbar_init(&x_empty[i], 2); }
        for (int i = 0; i < NA; ++i) { ptx::mbar_init(&a_full[i], 4); ptx::mbar_init(&a_empty[i], 1); }
        for (int i = 0; i < ND; ++i) {
            ptx::mbar_init(&d_full[i], 1);
            ptx::mbar_init(&d_empty[i], 4);
            ptx::mbar_init(&xs_full[i], 1);
        }
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(drain + 1, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) {
        ptx::prefetch_tensormap(&map_codes);
        ptx::prefetch_tensormap(&map_x);
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

    // chunk u -> tile w = u / cpt, groups g = (u % cpt) * CG + q, q < ng.
    // Groups are numbered gi along the run; group gi belongs to the role copies of parity gi & 1
    // and uses activation stage gi % NX, TMEM A stage gi % NA and accumulator gi % ND (all even
    // ring sizes, so every slot serves one parity only).
    auto chunk_groups = [&](int64_t u, int& w, int& g0, int& ng) {
        w = static_cast<int>(u / p.cpt);
        g0 = static_cast<int>(u % p.cpt) * CG;
        ng = min(CG, p.G - g0);
    };

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t i = 0, pi = 0, ci = 0, gi = 0;   // chunks started / with scales+biases / with codes; x tiles
            bool ok = true;
            for (; i < nchunks && ok; ++i) {
                int w, g0, ng;
                chunk_groups(u0 + i, w, g0, ng);
                if (p.param_tma) {
                    const int pr = static_cast<int>(i % PR);
                    if (!ptx::mbar_wait(&p_empty[pr], ((i / PR) & 1u) ^ 1u, abort_flag)) break;
                    uint8_t* pt = smem + L::kOffPar + pr * kParBytes;
                    ptx::mbar_arrive_expect_tx(&p_full[pr], kParBytes);
                    ptx::tma_load_2d(pt, &map_scales, &p_full[pr], g0, w * BW);
                    ptx::tma_load_2d(pt + kParHalf, &map_biases, &p_full[pr], g0, w * BW);
                    ++pi;
                }
                const int s = static_cast<int>(i % NC);
                if (!ptx::mbar_wait(&c_empty[s], ((i / NC) & 1u) ^ 1u, abort_flag)) break;
                uint8_t* st = smem + L::kOffC + s * kCBytes;
                ptx::mbar_arrive_expect_tx(&c_full[s], kCBytes);
#pragma unroll
                for (int bx = 0; bx < CG / kBoxGroups; ++bx)   // consecutive boxes: long contiguous row segments
                    ptx::tma_load_2d(st + bx * kBoxBytes, &map_codes, &c_full[s], (g0 + bx * kBoxGroups) * (BK / 8), w * BW);
                ++ci;
                for (int q = 0; q < ng; ++q) {
                    const int xst = static_cast<int>(gi % NX);
                    if (!ptx::mbar_wait(&x_empty[xst], ((gi / NX) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&x_full[xst], L::kXBytes);
                    ptx::tma_load_2d(smem + L::kOffX + xst * L::kXBytes, &map_x, &x_full[xst], (g0 + q) * BK, 0);
                    ++gi;
                }
            }
            // never leave the CTA with bulk copies still landing in its shared memory
            for (uint32_t j = (ci > static_cast<uint32_t>(NC) ? ci - NC : 0u); j < ci; ++j)
                ptx::mbar_wait(&c_full[j % NC], (j / NC) & 1u, nullptr);
            for (uint32_t j = (pi > static_cast<uint32_t>(PR) ? pi - PR : 0u); j < pi; ++j)
                ptx::mbar_wait(&p_full[j % PR], (j / PR) & 1u, nullptr);
            for (uint32_t j = (gi > static_cast<uint32_t>(NX) ? gi - NX : 0u); j < gi; ++j)
                ptx::mbar_wait(&x_full[j % NX], (j / NX) & 1u, nullptr);
        }
    } else if (warp == kWarpMma0 || warp == kWarpMma0 + 1) {
        // ---------------------------------------------------------------- MMA issuers (even / odd groups)
        const uint32_t par = static_cast<uint32_t>(warp - kWarpMma0);
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_f16(BW, NT, true);
            uint32_t gi = 0;
            bool ok = true;
            for (uint32_t i = 0; i < nchunks && ok; ++i) {
                int w, g0, ng;
                chunk_groups(u0 + i, w, g0, ng);
                for (int q = 0; q < ng; ++q, ++gi) {
                    if ((gi & 1u) != par) continue;
                    const int xst = static_cast<int>(gi % NX), a = static_cast<int>(gi % NA);
                    const int j = static_cast<int>(gi % ND);
                    if (!ptx::mbar_wait(&x_full[xst], (gi / NX) & 1u, abort_flag)) { ok = false; break; }
                    if (!ptx::mbar_wait(&a_full[a], (gi / NA) & 1u, abort_flag)) { ok = false; break; }
                    if (!ptx::mbar_wait(&d_empty[j], ((gi / ND) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after_sync();
                    const uint32_t x_addr = ptx::smem_addr(smem + L::kOffX + xst * L::kXBytes);
                    const uint32_t d = tmem_base + L::kAccCol + static_cast<uint32_t>(j * NT);
                    const uint32_t a_tm = tmem_base + L::kACol + 32u * a;
#pragma unroll
                    for (int u = 0; u < BK / UK; ++u)
                        ptx::mma_f16_ts(d, a_tm + u * (UK / 2), ptx::sdesc_sw128(x_addr + u * UK * 2), idesc, u != 0);
                    ptx::mma_commit(&x_empty[xst]);
                    ptx::mma_commit(&a_empty[a]);
                    ptx::mma_commit(&d_full[j]);
                }
            }
            ptx::mma_commit(drain + par);
            ptx::mbar_wait(drain + par, 0, nullptr);
        }
    } else if (warp == kWarpXsum) {
        // ---------------------------------------------------------------- activation sums per group
        // NT = 32: lane t sums all of token row t; NT = 16: lanes t and t+16 each sum half of row t
        uint32_t gi = 0;
        bool ok = true;
        for (uint32_t i = 0; i < nchunks && ok; ++i) {
            int w, g0, ng;
            chunk_groups(u0 + i, w, g0, ng);
            for (int q = 0; q < ng; ++q, ++gi) {
                const int xst = static_cast<int>(gi % NX), j = static_cast<int>(gi % ND);
                bool got = ptx::mbar_wait(&x_full[xst], (gi / NX) & 1u, abort_flag);
                got = got && ptx::mbar_wait(&d_empty[j], ((gi / ND) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                const uint8_t* xt = smem + L::kOffX + xst * L::kXBytes;
                const int row = (NT == 32) ? lane : (lane & 15);
                const int c0 = (NT == 32) ? 0 : ((lane >> 4) * 4), nc = (NT == 32) ? 8 : 4;
                float acc = 0.0f;
                for (int c = c0; c < c0 + nc; ++c) {          // 16-byte piece c of the row (swizzled position)
                    const uint4 v = *reinterpret_cast<const uint4*>(xt + row * 128 + ((c ^ (row & 7)) << 4));
                    acc += (bf16_lo(v.x) + bf16_hi(v.x)) + (bf16_lo(v.y) + bf16_hi(v.y)) +
                           (bf16_lo(v.z) + bf16_hi(v.z)) + (bf16_lo(v.w) + bf16_hi(v.w));
                }
                if (NT == 16) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 16);
                if (lane < NT) xs[j * NT + lane] = acc;
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(&xs_full[j]);
                    ptx::mbar_arrive(&x_empty[xst]);
                }
            }
        }
    } else if (warp >= kWarpBuild0 && warp < kWarpDrain0) {
        // ---------------------------------------------------------------- A builders (even / odd groups)
        const uint32_t par = static_cast<uint32_t>((warp - kWarpBuild0) >> 2);
        const int quarter = warp & 3;
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
                const int a = static_cast<int>(gq % NA);
                const uint4 c0 = cw[2 * k], c1 = cw[2 * k + 1];
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t av[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) codes_to_bf16(words[c], &av[4 * c]);
                got = ptx::mbar_wait(&a_empty[a], ((gq / NA) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                ptx::tmem_st_32x32b_x32(tmem_base + lane_addr + L::kACol + 32u * a, av);
                ptx::tmem_wait_st();
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&a_full[a]);
            }
            gi += static_cast<uint32_t>(ng);
        }
    } else if (warp >= kWarpDrain0) {
        // ---------------------------------------------------------------- drain (even / odd groups)
        const uint32_t par = static_cast<uint32_t>((warp - kWarpDrain0) >> 2);
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
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
            // this copy's scales and biases of row r in this chunk (groups q0, q0 + 2, ...): from the
            // scale/bias ring, else from global memory
            __half sv[CG / 2], bv[CG / 2];
            if (p.param_tma) {
                const int pr = static_cast<int>(i % PR);
                const bool got = ptx::mbar_wait(&p_full[pr], (i / PR) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) break;
                const uint8_t* pt = smem + L::kOffPar + pr * kParBytes;
                __align__(16) __half sa[CG], ba[CG];
#pragma unroll
                for (int c = 0; c < CG / 8; ++c) {
                    *reinterpret_cast<uint4*>(sa + 8 * c) = reinterpret_cast<const uint4*>(pt + r * CG * 2)[c];
                    *reinterpret_cast<uint4*>(ba + 8 * c) = reinterpret_cast<const uint4*>(pt + kParHalf + r * CG * 2)[c];
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&p_empty[pr]);
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
#pragma unroll
            for (int k = 0; k < CG / 2; ++k) {
                const int q = q0 + 2 * k;
                if (q >= ng) break;
                const uint32_t gq = gi + static_cast<uint32_t>(q);
                const int j = static_cast<int>(gq % ND);
                float sc = 0.0f, cc = 0.0f;
                if (n < p.N) {
                    sc = __half2float(sv[k]);
                    cc = fmaf(-128.0f, sc, __half2float(bv[k]));
                }
                // the activation-sum term first (few live registers), then the tensor-core sums
                bool got = ptx::mbar_wait(&xs_full[j], (gq / ND) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                const float4* xsj = reinterpret_cast<const float4*>(xs + j * NT);
#pragma unroll
                for (int t4 = 0; t4 < NT / 4; ++t4) {
                    const float4 v = xsj[t4];
                    yacc[4 * t4 + 0] = fmaf(cc, v.x, yacc[4 * t4 + 0]);
                    yacc[4 * t4 + 1] = fmaf(cc, v.y, yacc[4 * t4 + 1]);
                    yacc[4 * t4 + 2] = fmaf(cc, v.z, yacc[4 * t4 + 2]);
                    yacc[4 * t4 + 3] = fmaf(cc, v.w, yacc[4 * t4 + 3]);
                }
                got = ptx::mbar_wait(&d_full[j], (gq / ND) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                uint32_t dv[NT];
                if constexpr (NT == 32) {
                    ptx::tmem_ld_32x32b_x32(tmem_base + lane_addr + L::kAccCol + static_cast<uint32_t>(j * NT),
                                            *reinterpret_cast<uint32_t(*)[32]>(dv));
                } else {
                    ptx::tmem_ld_32x32b_x16(tmem_base + lane_addr + L::kAccCol + static_cast<uint32_t>(j * NT),
                                            *reinterpret_cast<uint32_t(*)[16]>(dv));
                }
                ptx::tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < NT; ++t) yacc[t] = fmaf(sc, __uint_as_float(dv[t]), yacc[t]);
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&d_empty[j]);
            }
            gi += static_cast<uint32_t>(ng);
            // end of this tile's segment: write this copy's partial and start over
            const bool seg_end = (i + 1 == nchunks) || ((u0 + i + 1) % p.cpt == 0);
            if (ok && seg_end) {
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
