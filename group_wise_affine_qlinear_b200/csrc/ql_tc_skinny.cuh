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
// written to tensor memory (tcgen05.st), so shared memory carries only the
// streamed code tiles and the small activation tiles.
//
// Stream-K schedule: the work is cut into chunks of CG consecutive groups of
// one 128-row weight tile (a tile has ceil(G/CG) chunks; a tile's last chunk may
// be partial).  The chunks, tile-major, are split into one equal contiguous run
// per CTA; a run covers at most a few tiles, and each covered tile segment
// leaves an fp32 partial [tokens][128] in the workspace.  The code boxes of a
// chunk bring CG * 32 contiguous bytes of each row, so DRAM sees long row
// segments instead of scattered 32-byte sectors.  A second kernel sums, per output, the partials of the CTAs
// that covered its tile in CTA order (deterministic) and rounds to bf16.
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0       TMA producer: L2 prefetch of the code chunk PD chunks ahead, then the code chunk
//                (128 rows x CG*32 B) + CG activation tiles (NT x 64), all 128B-swizzled
//   warps 1, 3   MMA issuers for even / odd groups (warp 1 also allocates TMEM)
//   warp 2       per-group activation sums xsum_g[t] from the staged activation tile
//   warps 4-7    A builders: one weight row per thread, codes -> bf16 (128+q) pairs -> TMEM
//   warps 8-11   drain: one weight row per thread, fp32 accumulation of s*D + c*xsum over the run
#pragma once

#include "ql_ptx.cuh"

namespace ql {
namespace skinny {

constexpr int BW = 128;
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kThreads = 12 * 32;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpXsum = 2, kWarpMma2 = 3, kWarpBuild0 = 4, kWarpDrain0 = 8;
constexpr int CG = 8;                    // groups per chunk (one TMA stage), a multiple of 4
constexpr int kBoxGroups = 4;            // groups per code box: 128 bytes of each row (the 128B-swizzle span)
constexpr int PD = 12;                   // chunks of codes prefetched into L2 ahead of the shared-memory loads
constexpr int NA = 4;                    // TMEM A stages (32 columns each)
constexpr int ND = 8;                    // TMEM accumulator buffers (NT columns each)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBoxBytes = BW * BK / 2 * kBoxGroups;   // 16 KB: one code box
constexpr uint32_t kCBytes = kBoxBytes * (CG / kBoxGroups);  // codes per chunk
constexpr int PR = 4;                                         // params ring depth (chunks)
constexpr uint32_t kParHalf = BW * CG * 2;                    // one chunk's scales (or biases): [128][CG] f16
constexpr uint32_t kParBytes = 2 * kParHalf;

template <int NT>
struct Layout {
    static constexpr uint32_t kXBytes = NT * BK * 2;                // one group's activation tile
    static constexpr uint32_t kStageBytes = kCBytes + CG * kXBytes;
    static constexpr int NS = static_cast<int>(212992 / kStageBytes);   // TMA stages (208 KB budget)
    static constexpr uint32_t kOffStage = 0;                       // [NS][codes | x_0 .. x_3], 1 KB aligned
    static constexpr uint32_t kOffXs = NS * kStageBytes;          // xsum ring [ND][NT] fp32
    static constexpr uint32_t kOffPar = kOffXs + ND * NT * 4;      // params ring [PR][scales|biases][128][CG] f16
    static constexpr uint32_t kOffBar = kOffPar + PR * kParBytes;
    static constexpr uint32_t kNumBars = 2 * NS + 2 * NA + 3 * ND + 2 * PR + 2;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
    static constexpr uint32_t kAccCol = 0;                          // D buffer j at [j*NT, (j+1)*NT)
    static constexpr uint32_t kACol = ND * NT;                      // A stage a at [kACol + 32a, +32)
    static_assert(kCBytes % 1024 == 0 && kXBytes % 1024 == 0, "stage pieces need 1 KB alignment");
    static_assert(kACol + NA * 32 <= kTmemCols, "tensor memory budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(NS >= 2, "at least two stages");
};

struct Params {
    float* partial;          // [P][segmax][M][128] fp32
    int param_tma;           // 1: scales/biases arrive by TMA tiles (needs G % CG == 0); 0: per-group loads
    const __half* scales;    // [N][G]
    const __half* biases;    // [N][G]
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
    constexpr int NS = L::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* s_full = bars;
    uint64_t* s_empty = s_full + NS;
    uint64_t* a_full = s_empty + NS;
    uint64_t* a_empty = a_full + NA;
    uint64_t* d_full = a_empty + NA;
    uint64_t* d_empty = d_full + ND;
    uint64_t* xs_full = d_empty + ND;
    uint64_t* p_full = xs_full + ND;
    uint64_t* p_empty = p_full + PR;
    uint64_t* drain = p_empty + PR;
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
        // a stage is free once both MMA warps (commits), the xsum warp and the 4 A builders are done with it
        for (int i = 0; i < NS; ++i) { ptx::mbar_init(&s_full[i], 1); ptx::mbar_init(&s_empty[i], 7); }
        for (int i = 0; i < NA; ++i) { ptx::mbar_init(&a_full[i], 4); ptx::mbar_init(&a_empty[i], 1); }
        for (int i = 0; i < ND; ++i) {
            ptx::mbar_init(&d_full[i], 1);
            ptx::mbar_init(&d_empty[i], 4);
            ptx::mbar_init(&xs_full[i], 1);
        }
        for (int i = 0; i < PR; ++i) { ptx::mbar_init(&p_full[i], 1); ptx::mbar_init(&p_empty[i], 4); }
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
    if (warp == kWarpMma) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    // Groups are counted along the run (gi); a/d/xs rings advance per valid group, the TMA ring per chunk.
    // chunk u -> tile w = u / cpt, groups g = (u % cpt) * CG + q, q < CG, valid while g < G.
    auto chunk_groups = [&](int64_t u, int& w, int& g0, int& ng) {
        w = static_cast<int>(u / p.cpt);
        g0 = static_cast<int>(u % p.cpt) * CG;
        ng = min(CG, p.G - g0);
    };

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            // HBM needs far more bytes in flight than the shared-memory stages hold: the code
            // boxes of chunk i + PD are prefetched into L2 while chunk i is loaded from there.
            auto prefetch = [&](uint32_t k) {
                int w, g0, ng;
                chunk_groups(u0 + k, w, g0, ng);
#pragma unroll
                for (int bx = 0; bx < CG / kBoxGroups; ++bx)
                    ptx::tma_prefetch_2d(&map_codes, (g0 + bx * kBoxGroups) * (BK / 8), w * BW);
            };
            for (uint32_t k = 0; k < nchunks && k < static_cast<uint32_t>(PD); ++k) prefetch(k);
            uint32_t i = 0, pi = 0;     // chunks whose codes / whose params were issued
            for (; i < nchunks; ++i) {
                const int s = static_cast<int>(i % NS);
                const uint32_t ph = (i / NS) & 1u;
                if (i + PD < nchunks) prefetch(i + PD);
                if (!ptx::mbar_wait(&s_empty[s], ph ^ 1, abort_flag)) break;
                int w, g0, ng;
                chunk_groups(u0 + i, w, g0, ng);
                uint8_t* st = smem + L::kOffStage + s * L::kStageBytes;
                if (p.param_tma) {
                    // the drain reads each chunk's scales and biases from a small ring of its own
                    const int pr = static_cast<int>(i % PR);
                    if (!ptx::mbar_wait(&p_empty[pr], ((i / PR) & 1u) ^ 1u, abort_flag)) break;
                    uint8_t* pt = smem + L::kOffPar + pr * kParBytes;
                    ptx::mbar_arrive_expect_tx(&p_full[pr], kParBytes);
                    ptx::tma_load_2d(pt, &map_scales, &p_full[pr], g0, w * BW);
                    ptx::tma_load_2d(pt + kParHalf, &map_biases, &p_full[pr], g0, w * BW);
                    ++pi;
                }
                ptx::mbar_arrive_expect_tx(&s_full[s], L::kStageBytes);
#pragma unroll
                for (int bx = 0; bx < CG / kBoxGroups; ++bx)   // consecutive boxes: longer contiguous row segments
                    ptx::tma_load_2d(st + bx * kBoxBytes, &map_codes, &s_full[s], (g0 + bx * kBoxGroups) * (BK / 8), w * BW);
#pragma unroll
                for (int q = 0; q < CG; ++q)       // boxes past K read zeros (counted bytes all the same)
                    ptx::tma_load_2d(st + kCBytes + q * L::kXBytes, &map_x, &s_full[s], (g0 + q) * BK, 0);
            }
            for (uint32_t j = (i > static_cast<uint32_t>(NS) ? i - NS : 0u); j < i; ++j)
                ptx::mbar_wait(&s_full[j % NS], (j / NS) & 1u, nullptr);
            for (uint32_t j = (pi > static_cast<uint32_t>(PR) ? pi - PR : 0u); j < pi; ++j)
                ptx::mbar_wait(&p_full[j % PR], (j / PR) & 1u, nullptr);
        }
    } else if (warp == kWarpMma || warp == kWarpMma2) {
        // ---------------------------------------------------------------- MMA issuers (even / odd groups)
        const uint32_t par = warp == kWarpMma ? 0u : 1u;
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_f16(BW, NT, true);
            uint32_t gi = 0;
            bool ok = true;
            for (uint32_t i = 0; i < nchunks && ok; ++i) {
                const int s = static_cast<int>(i % NS);
                if (!ptx::mbar_wait(&s_full[s], (i / NS) & 1u, abort_flag)) break;
                int w, g0, ng;
                chunk_groups(u0 + i, w, g0, ng);
                for (int q = 0; q < ng; ++q, ++gi) {
                    if ((gi & 1u) != par) continue;
                    const int a = static_cast<int>(gi % NA), j = static_cast<int>(gi % ND);
                    if (!ptx::mbar_wait(&a_full[a], (gi / NA) & 1u, abort_flag)) { ok = false; break; }
                    if (!ptx::mbar_wait(&d_empty[j], ((gi / ND) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after_sync();
                    const uint32_t x_addr = ptx::smem_addr(smem + L::kOffStage + s * L::kStageBytes + kCBytes + q * L::kXBytes);
                    const uint32_t d = tmem_base + L::kAccCol + static_cast<uint32_t>(j * NT);
                    const uint32_t a_tm = tmem_base + L::kACol + 32u * a;
#pragma unroll
                    for (int u = 0; u < BK / UK; ++u)
                        ptx::mma_f16_ts(d, a_tm + u * (UK / 2), ptx::sdesc_sw128(x_addr + u * UK * 2), idesc, u != 0);
                    ptx::mma_commit(&a_empty[a]);
                    ptx::mma_commit(&d_full[j]);
                }
                if (!ok) break;
                ptx::mma_commit(&s_empty[s]);
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
            const int s = static_cast<int>(i % NS);
            bool got = ptx::mbar_wait(&s_full[s], (i / NS) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            int w, g0, ng;
            chunk_groups(u0 + i, w, g0, ng);
            for (int q = 0; q < ng; ++q, ++gi) {
                const int j = static_cast<int>(gi % ND);
                got = ptx::mbar_wait(&d_empty[j], ((gi / ND) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                const uint8_t* xt = smem + L::kOffStage + s * L::kStageBytes + kCBytes + q * L::kXBytes;
                const int row = (NT == 32) ? lane : (lane & 15);
                const int c0 = (NT == 32) ? 0 : ((lane >> 4) * 4), nc = (NT == 32) ? 8 : 4;
                float acc = 0.0f;
                for (int c = c0; c < c0 + nc; ++c) {          // 16-byte chunk c of the row (swizzled position)
                    const uint4 v = *reinterpret_cast<const uint4*>(xt + row * 128 + ((c ^ (row & 7)) << 4));
                    acc += (bf16_lo(v.x) + bf16_hi(v.x)) + (bf16_lo(v.y) + bf16_hi(v.y)) +
                           (bf16_lo(v.z) + bf16_hi(v.z)) + (bf16_lo(v.w) + bf16_hi(v.w));
                }
                if (NT == 16) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 16);
                if (lane < NT) xs[j * NT + lane] = acc;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&xs_full[j]);
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&s_empty[s]);
        }
    } else if (warp >= kWarpBuild0 && warp < kWarpBuild0 + 4) {
        // ---------------------------------------------------------------- A builders
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t gi = 0;
        bool ok = true;
        for (uint32_t i = 0; i < nchunks && ok; ++i) {
            const int s = static_cast<int>(i % NS);
            bool got = ptx::mbar_wait(&s_full[s], (i / NS) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            int w, g0, ng;
            chunk_groups(u0 + i, w, g0, ng);
            // row r's code bytes of this chunk, 128 per box, stored by the TMA with the 128-byte
            // swizzle: logical 16-byte piece c of a box row sits at c ^ (r % 8), so every 8 lanes of
            // a load touch 8 bank groups
            const uint8_t* crow = smem + L::kOffStage + s * L::kStageBytes + r * 128;
            uint4 cw[2 * CG];
#pragma unroll
            for (int bx = 0; bx < CG / kBoxGroups; ++bx)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    cw[8 * bx + c] = *reinterpret_cast<const uint4*>(crow + bx * kBoxBytes + ((c ^ (r & 7)) << 4));
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&s_empty[s]);
#pragma unroll
            for (int q = 0; q < CG; ++q, ++gi) {
                if (q >= ng) break;
                const int a = static_cast<int>(gi % NA);
                const uint4 c0 = cw[2 * q], c1 = cw[2 * q + 1];
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t av[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) codes_to_bf16(words[c], &av[4 * c]);
                got = ptx::mbar_wait(&a_empty[a], ((gi / NA) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                ptx::tmem_st_32x32b_x32(tmem_base + lane_addr + L::kACol + 32u * a, av);
                ptx::tmem_wait_st();
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&a_full[a]);
            }
        }
    } else if (warp >= kWarpDrain0) {
        // ---------------------------------------------------------------- drain
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
            // this chunk's scales and biases of row r: from the params ring, else from global memory
            __half sv[CG], bv[CG];
            if (p.param_tma) {
                const int pr = static_cast<int>(i % PR);
                const bool got = ptx::mbar_wait(&p_full[pr], (i / PR) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) break;
                const uint8_t* pt = smem + L::kOffPar + pr * kParBytes;
#pragma unroll
                for (int c = 0; c < CG / 8; ++c) {
                    *reinterpret_cast<uint4*>(sv + 8 * c) = reinterpret_cast<const uint4*>(pt + r * CG * 2)[c];
                    *reinterpret_cast<uint4*>(bv + 8 * c) = reinterpret_cast<const uint4*>(pt + kParHalf + r * CG * 2)[c];
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&p_empty[pr]);
            } else {
#pragma unroll
                for (int q = 0; q < CG; ++q) {
                    const bool in = n < p.N && q < ng;
                    sv[q] = in ? __ldg(p.scales + static_cast<int64_t>(n) * p.G + g0 + q) : __float2half_rn(0.0f);
                    bv[q] = in ? __ldg(p.biases + static_cast<int64_t>(n) * p.G + g0 + q) : __float2half_rn(0.0f);
                }
            }
#pragma unroll
            for (int q = 0; q < CG; ++q, ++gi) {
                if (q >= ng) break;
                const int j = static_cast<int>(gi % ND);
                float sc = 0.0f, cc = 0.0f;
                if (n < p.N) {
                    const float s_ = __half2float(sv[q]);
                    sc = s_;
                    cc = fmaf(-128.0f, s_, __half2float(bv[q]));
                }
                bool got = ptx::mbar_wait(&d_full[j], (gi / ND) & 1u, abort_flag);
                got = got && ptx::mbar_wait(&xs_full[j], (gi / ND) & 1u, abort_flag);
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
                const float* xsj = xs + j * NT;
#pragma unroll
                for (int t = 0; t < NT; ++t) yacc[t] = fmaf(sc, __uint_as_float(dv[t]), fmaf(cc, xsj[t], yacc[t]));
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&d_empty[j]);
            }
            // end of this tile's segment: write the partial and start over
            const bool seg_end = (i + 1 == nchunks) || ((u0 + i + 1) % p.cpt == 0);
            if (ok && seg_end) {
                float* dst = p.partial + ((static_cast<int64_t>(blockIdx.x) * p.segmax + (w - w_first)) * p.M) * BW;
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
    if (warp == kWarpMma) {
        __syncwarp();
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// y[t][n] = sum over the CTAs whose runs cover tile n/128, in CTA order, of their partial for that tile.
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
            acc += partial[((static_cast<int64_t>(c) * segmax + (w - w_first)) * M + t) * BW + r];
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
