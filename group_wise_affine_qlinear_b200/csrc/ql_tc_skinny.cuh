// Weight-streaming tensor-core path for small M (M <= 32): HBM-bound, so the job
// is to read the 4.5-bit weights once at full bandwidth and spend as few
// instructions per weight as possible.
//
// The weight of row n, column k is w = s(n,g) q(n,k) + b(n,g) for the 64-group g
// holding k (aimarketly "Ideogram-4-IQ4_M", "What IQ4 means here": w = scale * q +
// bias), so per group
//   y[t][n] += s(n,g) * sum_{k in g} q(n,k) x[t][k] + b(n,g) * sum_{k in g} x[t][k].
// The tensor core (tcgen05.mma, kind::f16, f16 operands, fp32 accumulation) forms
// the first sum from the exact codes; the drain applies s and b in fp32.
//
// Codes as f16 operands.  A word of codes holds k = 0..7 of an 8-block in nibbles
// 0..7.  Read as a pair of f16 values, (v & 0x000F000F) is (q0, q4) * 2^-24 and
// (v & 0x00F000F0) is (q1, q5) * 16 * 2^-24 exactly (f16 subnormals), and the same
// masks on v >> 8 give (q2, q6) * 2^-24 and (q3, q7) * 16 * 2^-24: one shift and
// four ANDs per 8 weights, with k in the order 0,4,1,5,2,6,3,7 along each 8-block
// of the reduction dimension.  A prepass kernel writes the activations in that
// order as f16, x'[t][k] = x[t][k] * 2^e_t (a per-row power of two that puts the
// row maximum in [2^14, 2^15)) and a further 2^-4 at odd k to cancel the factor
// 16 on those codes, so that
//   D_g[n][t] = sum_{k in g} A[n][k] x'[t][k] = 2^(e_t - 24) sum_{k in g} q(n,k) x[t][k].
// The prepass also writes xs_g[t] = 2^(e_t - 24) sum_{k in g} x[t][k], so the drain
// accumulates s * D + b * xs, all scaled by 2^(e_t - 24), and the reduce kernel
// scales back by 2^(24 - e_t) (ldexpf, exact).  Activation entries below 2^-24 of
// the row maximum lose bits as f16 subnormals; nothing else is rounded before the
// fp32 accumulation.  The prepass kernels run under programmatic dependent launch:
// the main kernel starts streaming codes at once and waits for the prepass only
// before its first activation load.
//
// Stream-K schedule: the work is cut into chunks of CG = 8 consecutive groups of
// one 128-row weight tile (a tile has ceil(G/CG) chunks; a tile's last chunk may
// be partial).  The chunks, tile-major, are split into one equal contiguous run
// per CTA; a run covers at most a few tiles, and each covered tile segment leaves
// fp32 partials [2][tokens][128] in the workspace (one per drain copy).  The reduce
// kernel sums, per output, the partials of the CTAs that covered its tile in CTA
// order (deterministic).  The code boxes of a chunk bring CG * 32 contiguous bytes
// of each row, so DRAM sees long row segments.
//
// Each barrier wait, arrive or commit costs a role on the order of a hundred
// cycles, so the roles step over pairs of consecutive groups of a chunk (pair j =
// groups 2j, 2j+1): one wait and one signal per pair.  Pairs are numbered pc along
// the run.  The A builders, the slowest role, run as four copies (pair pc goes to
// copy pc % 4, one pair of every chunk each); the drains and the MMA issuers run
// as two (pc % 2).  TMEM slot pc % NS holds the pair's two A stages and two
// accumulators, with one barrier each way: ready[s] (A built by the 4 builder warps
// of the slot's copy, accumulators read back by the 4 drain warps of its copy) and
// done[s] (the slot's MMAs completed).
// Warp roles (864 threads, one CTA per SM; 7 warps per SM sub-partition leave 72 registers a thread):
//   warp 0        TMA producer: code chunks (128 rows x CG*32 B, 128B swizzle), scale/bias/xs tiles,
//                 activation tiles of a chunk (NT x 64 f16 per group, 128B swizzle)
//   warps 1, 2    MMA issuers for even / odd pairs (warp 1 also allocates TMEM)
//   warps 3-18    A builders, copies 0-3 of 4 warps: one weight row per thread
//   warps 19-26   drains, even pairs (19-22) / odd pairs (23-26): one weight row per thread, fp32
//                 accumulation of s*D + b*xs over the run
#pragma once

#include "ql_ptx.cuh"

namespace ql {
namespace skinny {

constexpr int BW = 128;
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kBuildCopies = 4, kDrainCopies = 2, kMmaCopies = 2;
constexpr int kWarpTma = 0, kWarpMma0 = 1, kWarpBuild0 = 3, kWarpDrain0 = kWarpBuild0 + 4 * kBuildCopies;
constexpr int kThreads = (kWarpDrain0 + 4 * kDrainCopies) * 32;
constexpr int CG = 8;                    // groups per chunk: four pairs, one per builder copy
constexpr int kBoxGroups = 4;            // groups per code box: 128 bytes of each row (the 128B-swizzle span)
constexpr int NS = 4;                    // TMEM slots (two A stages + two accumulators each)
constexpr int PR = 4;                    // scale/bias/xs chunk stages
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBoxBytes = BW * BK / 2 * kBoxGroups;     // 16 KB: one code box
constexpr uint32_t kCBytes = kBoxBytes * (CG / kBoxGroups);  // codes per chunk
constexpr uint32_t kParHalf = BW * CG * 2;                   // one chunk's scales (or biases): [128][CG] f16
static_assert(CG == 2 * kBuildCopies && kBoxGroups == 4, "one pair of every chunk per builder copy");
static_assert(NS % kBuildCopies == 0 && NS % kDrainCopies == 0 && NS % kMmaCopies == 0,
              "every TMEM slot serves one copy of each role");

template <int NT>
struct Layout {
    static constexpr int NC = NT == 16 ? 4 : 3;                          // code chunk stages
    static constexpr int NXC = NT == 16 ? 4 : 3;                         // activation chunk stages
    static constexpr uint32_t kXTile = NT * BK * 2;                      // one group's activation tile (f16)
    static constexpr uint32_t kXBytes = CG * kXTile;                     // one chunk's activation tiles
    static constexpr uint32_t kXsBytes = CG * NT * 4;                    // one chunk's xs rows [CG][NT] fp32
    static constexpr uint32_t kParBytes = 2 * kParHalf + kXsBytes;       // [scales | biases | xs]
    static constexpr uint32_t kOffC = 0;                                  // [NC][codes], 1 KB aligned
    static constexpr uint32_t kOffX = kOffC + NC * kCBytes;              // [NXC][CG][x tile], 1 KB aligned
    static constexpr uint32_t kOffPar = kOffX + NXC * kXBytes;           // [PR][par]
    static constexpr uint32_t kOffBar = kOffPar + PR * kParBytes;
    static constexpr uint32_t kNumBars = 2 * NC + 2 * PR + 2 * NXC + 2 * NS + kMmaCopies;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
    static constexpr uint32_t kAccCol = 0;                                // accumulator h of slot s at (2s+h)*NT
    static constexpr uint32_t kACol = 2 * NS * NT;                        // A stage h of slot s at kACol + 32(2s+h)
    static_assert(kCBytes % 1024 == 0 && kXTile % 1024 == 0, "swizzled stage pieces need 1 KB alignment");
    static_assert(kParBytes % 128 == 0, "TMA destinations 128-byte aligned");
    static_assert(kACol + 2 * NS * 32 <= kTmemCols, "tensor memory budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Params {
    float* partial;          // [P][segmax][2][M][128] fp32, scaled by 2^(e_t - 24)
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

// Codes word (code j in nibble j) -> 4 words of f16 pairs (subnormals, exact):
// (q0, q4) 2^-24, (q1, q5) 16 2^-24, (q2, q6) 2^-24, (q3, q7) 16 2^-24.
__device__ __forceinline__ void codes_to_f16(uint32_t v, uint32_t* o) {
    const uint32_t u = v >> 8;
    o[0] = v & 0x000F000Fu;
    o[1] = v & 0x00F000F0u;
    o[2] = u & 0x000F000Fu;
    o[3] = u & 0x00F000F0u;
}

// Packed fp32 FMA on two lanes: d = a * b + c, each lane rounded as fmaf.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)),
          "l"(*reinterpret_cast<const uint64_t*>(&c)));
    return *reinterpret_cast<float2*>(&d);
}

// Activation prepass, two kernels over a grid of (slice, row): one thread per 8-block of k, 256 per
// CTA, so every 8-block of a row is read in parallel.

// pmax[t][slice] = max |x[t][k]| over the slice's 8-blocks.
__global__ void __launch_bounds__(256) skinny_rowmax_kernel(const uint4* __restrict__ x, float* __restrict__ pmax,
                                                            int K) {
    ptx::launch_dependents();
    __shared__ float red[8];
    const int t = blockIdx.y, kb = K / 8;
    const int c = blockIdx.x * 256 + threadIdx.x;
    float m = 0.0f;
    if (c < kb) {
        const uint4 v = x[static_cast<int64_t>(t) * kb + c];
        m = fmaxf(fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))),
                  fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
        pmax[static_cast<int64_t>(t) * gridDim.x + blockIdx.x] = fmaxf(m, red[0]);
    }
}

// For row t: e_t puts max_k |x[t][k]| in [2^14, 2^15) (0 for a zero or non-finite row);
// xp[t][k] = f16(x * 2^e_t), times 2^-4 at odd k, in the order 0,4,1,5,2,6,3,7 of each 8-block;
// xs[g][t] = 2^(e_t - 24) * (sum over group g of x[t][k], fp32); rowexp[t] = 24 - e_t.  The 8
// blocks of a group are 8 aligned lanes.  Columns t >= M of xs are never read back.
__global__ void __launch_bounds__(256) skinny_prepass_kernel(const uint4* __restrict__ x, const float* __restrict__ pmax,
                                                             uint4* __restrict__ xp, float* __restrict__ xs,
                                                             int* __restrict__ rowexp, int K, int NT) {
    ptx::launch_dependents();
    ptx::grid_dependency_wait();                               // pmax comes from the kernel before
    const int t = blockIdx.y, kb = K / 8;
    const int c = blockIdx.x * 256 + threadIdx.x;
    float m = 0.0f;
    for (int i = 0; i < static_cast<int>(gridDim.x); ++i) m = fmaxf(m, pmax[static_cast<int64_t>(t) * gridDim.x + i]);
    int ex = 0;
    if (m > 0.0f && m <= 3.4028235e38f) {
        int E;
        frexpf(m, &E);                                         // m = f 2^E, f in [0.5, 1)
        ex = 15 - E;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) rowexp[t] = 24 - ex;
    const bool in = c < kb;
    float sum = 0.0f;
    if (in) {
        const uint4 v = x[static_cast<int64_t>(t) * kb + c];
        const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                            bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
        sum = ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
        // slot pairs (k0, k4) (k1, k5) (k2, k6) (k3, k7); odd k carry the extra 2^-4
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int sh = ex - ((j & 1) ? 4 : 0);
            const __half2 h = __halves2half2(__float2half_rn(ldexpf(f[j], sh)), __float2half_rn(ldexpf(f[j + 4], sh)));
            o[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        xp[static_cast<int64_t>(t) * kb + c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
    if (in && (c & 7) == 0) xs[static_cast<int64_t>(c >> 3) * NT + t] = ldexpf(sum, ex - 24);
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) skinny_kernel(const __grid_constant__ CUtensorMap map_codes,
                                                            const __grid_constant__ CUtensorMap map_x,
                                                            const __grid_constant__ CUtensorMap map_scales,
                                                            const __grid_constant__ CUtensorMap map_biases,
                                                            const __grid_constant__ CUtensorMap map_xs,
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
    uint64_t* drain = done + NS;                // one per MMA issuer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int P = gridDim.x;
    const int64_t u0 = run_first(p.units, P, blockIdx.x);
    const int64_t u1 = run_first(p.units, P, blockIdx.x + 1);
    const uint32_t nchunks = static_cast<uint32_t>(u1 - u0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NC; ++i) { ptx::mbar_init(&c_full[i], 1); ptx::mbar_init(&c_empty[i], 4 * kBuildCopies); }
        for (int i = 0; i < PR; ++i) { ptx::mbar_init(&p_full[i], 1); ptx::mbar_init(&p_empty[i], 4 * kDrainCopies); }
        for (int i = 0; i < NXC; ++i) { ptx::mbar_init(&x_full[i], 1); ptx::mbar_init(&x_empty[i], kMmaCopies); }
        for (int i = 0; i < NS; ++i) { ptx::mbar_init(&ready[i], 8); ptx::mbar_init(&done[i], 1); }
        for (int i = 0; i < kMmaCopies; ++i) ptx::mbar_init(&drain[i], 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) {
        ptx::prefetch_tensormap(&map_codes);
        ptx::prefetch_tensormap(&map_x);
        ptx::prefetch_tensormap(&map_xs);
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

    // chunk u is chunk cq = u % cpt of tile w = u / cpt, groups g = cq * CG + q, q < ng; pair j of the
    // chunk is groups 2j and 2j + 1 (the second may be missing in a tile's last chunk).  Each role
    // walks its chunks with a (w, cq) position advanced by one per chunk, without dividing.
    struct ChunkPos {
        int w, cq;
    };
    const ChunkPos start{static_cast<int>(u0 / p.cpt), static_cast<int>(u0 % p.cpt)};
    auto advance = [&](ChunkPos& c) {
        if (++c.cq == p.cpt) {
            c.cq = 0;
            ++c.w;
        }
    };
    auto chunk_groups = [&](const ChunkPos& c, int& w, int& g0, int& ng) {
        w = c.w;
        g0 = c.cq * CG;
        ng = min(CG, p.G - g0);
    };
    // first pair j of a chunk whose run-wide number pb + j is copy (mod ncopies)
    auto first_pair = [](uint32_t pb, int copy, int ncopies) {
        const uint32_t nc = static_cast<uint32_t>(ncopies);
        return static_cast<int>((static_cast<uint32_t>(copy) + nc - pb % nc) % nc);
    };

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t ci = 0, pi = 0, xi = 0;     // chunks whose codes / parameters / activations were issued
            ChunkPos cpc = start, cpi = start;    // positions of chunk ci and of chunk i
            auto issue_codes = [&](uint32_t i) -> bool {
                int w, g0, ng;
                chunk_groups(cpc, w, g0, ng);
                const int s = static_cast<int>(i % NC);
                if (!ptx::mbar_wait(&c_empty[s], ((i / NC) & 1u) ^ 1u, abort_flag)) return false;
                uint8_t* st = smem + L::kOffC + s * kCBytes;
                ptx::mbar_arrive_expect_tx(&c_full[s], kCBytes);
#pragma unroll
                for (int bx = 0; bx < CG / kBoxGroups; ++bx)   // consecutive boxes: long contiguous row segments
                    ptx::tma_load_2d(st + bx * kBoxBytes, &map_codes, &c_full[s], (g0 + bx * kBoxGroups) * (BK / 8), w * BW);
                advance(cpc);
                return true;
            };
            // the codes do not depend on the prepass: start streaming them at once
            bool ok = true;
            while (ok && ci < nchunks && ci < static_cast<uint32_t>(NC)) {
                ok = issue_codes(ci);
                if (ok) ++ci;
            }
            ptx::grid_dependency_wait();
            for (uint32_t i = 0; i < nchunks && ok; ++i, advance(cpi)) {
                int w, g0, ng;
                chunk_groups(cpi, w, g0, ng);
                // scales, biases and activation sums of the chunk
                const int pr = static_cast<int>(i % PR);
                if (!ptx::mbar_wait(&p_empty[pr], ((i / PR) & 1u) ^ 1u, abort_flag)) break;
                uint8_t* pt = smem + L::kOffPar + pr * L::kParBytes;
                ptx::mbar_arrive_expect_tx(&p_full[pr], (p.param_tma ? 2 * kParHalf : 0u) + L::kXsBytes);
                if (p.param_tma) {
                    ptx::tma_load_2d(pt, &map_scales, &p_full[pr], g0, w * BW);
                    ptx::tma_load_2d(pt + kParHalf, &map_biases, &p_full[pr], g0, w * BW);
                }
                ptx::tma_load_2d(pt + 2 * kParHalf, &map_xs, &p_full[pr], 0, g0);   // rows past G read zeros
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
    } else if (warp < kWarpMma0 + kMmaCopies) {
        // ---------------------------------------------------------------- MMA issuers (even / odd pairs)
        // The whole warp runs the loop; one elected lane issues the MMAs and the commits.
        const int copy = warp - kWarpMma0;
        const bool leader = ptx::elect_one();
        constexpr uint32_t idesc = ptx::idesc_f16(BW, NT, false);
        const uint64_t xdesc0 = ptx::sdesc_sw128(ptx::smem_addr(smem + L::kOffX));
        uint32_t pb = 0;     // pairs of the run before this chunk
        bool ok = true;
        ChunkPos cp = start;
        for (uint32_t i = 0; i < nchunks && ok; ++i, advance(cp)) {
            int w, g0, ng;
            chunk_groups(cp, w, g0, ng);
            const int np = (ng + 1) >> 1;
            const int xc = static_cast<int>(i % NXC);
            bool got = ptx::mbar_wait(&x_full[xc], (i / NXC) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            // descriptor of the chunk's first activation tile (the address field counts 16-byte units)
            const uint64_t xdesc = xdesc0 + ((static_cast<uint32_t>(xc) * L::kXBytes) >> 4);
            for (int j = first_pair(pb, copy, kMmaCopies); j < np; j += kMmaCopies) {
                const uint32_t pc = pb + static_cast<uint32_t>(j);
                const int sl = static_cast<int>(pc % NS);
                got = ptx::mbar_wait(&ready[sl], (pc / NS) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                if (leader) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (2 * j + h < ng) {
                            const uint32_t d = tmem_base + L::kAccCol + static_cast<uint32_t>((2 * sl + h) * NT);
                            const uint32_t a_tm = tmem_base + L::kACol + 32u * static_cast<uint32_t>(2 * sl + h);
                            const uint64_t bd = xdesc + ((static_cast<uint32_t>(2 * j + h) * L::kXTile) >> 4);
#pragma unroll
                            for (int u = 0; u < BK / UK; ++u)
                                ptx::mma_f16_ts(d, a_tm + u * (UK / 2), bd + ((u * UK * 2) >> 4), idesc, u != 0);
                        }
                    }
                    ptx::mma_commit(&done[sl]);
                }
                __syncwarp();
            }
            if (ok && leader) ptx::mma_commit(&x_empty[xc]);
            __syncwarp();
            pb += static_cast<uint32_t>(np);
        }
        if (leader) ptx::mma_commit(&drain[copy]);
        __syncwarp();
        ptx::mbar_wait(&drain[copy], 0, nullptr);
    } else if (warp >= kWarpBuild0 && warp < kWarpDrain0) {
        // ---------------------------------------------------------------- A builders (four copies)
        const int copy = (warp - kWarpBuild0) >> 2;
        const int quarter = warp & 3;                      // TMEM lanes 32*quarter.. belong to this warp
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t pb = 0;
        bool ok = true;
        ChunkPos cp = start;
        for (uint32_t i = 0; i < nchunks && ok; ++i, advance(cp)) {
            int w, g0, ng;
            chunk_groups(cp, w, g0, ng);
            const int np = (ng + 1) >> 1;
            const int j = first_pair(pb, copy, kBuildCopies);     // this copy's pair of the chunk, if j < np
            const bool mine = j < np;
            const int s = static_cast<int>(i % NC);
            bool got = ptx::mbar_wait(&c_full[s], (i / NC) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            // row r's 32 code bytes of group q sit in code box q / 4 at the 16-byte pieces 2 (q % 4) and
            // 2 (q % 4) + 1 of its box row, stored with the 128-byte swizzle (piece c at c ^ (r % 8)), so
            // every 8 lanes of a load touch 8 bank groups
            uint4 cw[4];
            if (mine) {
                const uint8_t* crow = smem + L::kOffC + s * kCBytes + (j >> 1) * kBoxBytes + r * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = 2 * ((2 * j + h) & 3);
                    if (2 * j + h < ng) {
                        cw[2 * h] = *reinterpret_cast<const uint4*>(crow + ((c ^ (r & 7)) << 4));
                        cw[2 * h + 1] = *reinterpret_cast<const uint4*>(crow + (((c + 1) ^ (r & 7)) << 4));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&c_empty[s]);
            if (mine) {
                const uint32_t pc = pb + static_cast<uint32_t>(j);
                const int sl = static_cast<int>(pc % NS);
                // the slot's previous MMAs must have finished reading its A stages
                got = ptx::mbar_wait(&done[sl], ((pc / NS) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (2 * j + h < ng) {
                        const uint4 c0 = cw[2 * h], c1 = cw[2 * h + 1];
                        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                        uint32_t av[32];
#pragma unroll
                        for (int c = 0; c < 8; ++c) codes_to_f16(words[c], &av[4 * c]);
                        ptx::tmem_st_32x32b_x32(tmem_base + lane_addr + L::kACol + 32u * static_cast<uint32_t>(2 * sl + h), av);
                    }
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&ready[sl]);
            }
            pb += static_cast<uint32_t>(np);
        }
    } else {
        // ---------------------------------------------------------------- drains (even / odd pairs)
        const int copy = (warp - kWarpDrain0) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        // a slot's first use has no accumulators to read back: arrive for it in advance
        if (lane == 0)
            for (int sl = copy; sl < NS; sl += kDrainCopies) ptx::mbar_arrive(&ready[sl]);
        float2 yacc[NT / 2];
#pragma unroll
        for (int t = 0; t < NT / 2; ++t) yacc[t] = make_float2(0.0f, 0.0f);
        const int w_first = start.w;
        uint32_t pb = 0;
        bool ok = true;
        ChunkPos cp = start;
        for (uint32_t i = 0; i < nchunks && ok; ++i, advance(cp)) {
            int w, g0, ng;
            chunk_groups(cp, w, g0, ng);
            const int np = (ng + 1) >> 1;
            const int n = w * BW + r;
            const int j0 = first_pair(pb, copy, kDrainCopies);   // this copy's pairs: j0, j0 + 2
            const int pr = static_cast<int>(i % PR);
            bool got = ptx::mbar_wait(&p_full[pr], (i / PR) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            const uint8_t* pt = smem + L::kOffPar + pr * L::kParBytes;
            // scales and biases of row r for this copy's pairs j0 and j0 + 2: word jj holds the f16 values
            // of groups 2 (j0 + 2 jj) (low half) and 2 (j0 + 2 jj) + 1 (high half)
            uint32_t sw[2], bw[2];
            if (p.param_tma) {
                const uint4 sq = *reinterpret_cast<const uint4*>(pt + r * CG * 2);
                const uint4 bq = *reinterpret_cast<const uint4*>(pt + kParHalf + r * CG * 2);
                sw[0] = j0 ? sq.y : sq.x;
                sw[1] = j0 ? sq.w : sq.z;
                bw[0] = j0 ? bq.y : bq.x;
                bw[1] = j0 ? bq.w : bq.z;
            } else {
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    uint32_t sp = 0u, bp = 0u;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int q = 2 * (j0 + 2 * jj) + h;
                        if (n < p.N && q < ng) {
                            const int64_t at = static_cast<int64_t>(n) * p.G + g0 + q;
                            sp |= static_cast<uint32_t>(__half_as_ushort(__ldg(p.scales + at))) << (16 * h);
                            bp |= static_cast<uint32_t>(__half_as_ushort(__ldg(p.biases + at))) << (16 * h);
                        }
                    }
                    sw[jj] = sp;
                    bw[jj] = bp;
                }
            }
            const float* xsp = reinterpret_cast<const float*>(pt + 2 * kParHalf);     // [CG][NT]
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = j0 + 2 * jj;
                if (j >= np) break;
                const uint32_t pc = pb + static_cast<uint32_t>(j);
                const int sl = static_cast<int>(pc % NS);
                float sc[2];
                // the bias terms first (few live registers), then the tensor-core sums
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int q = 2 * j + h;
                    sc[h] = 0.0f;
                    if (q < ng) {
                        float bb = 0.0f;
                        if (n < p.N) {
                            sc[h] = __half2float(__ushort_as_half(static_cast<unsigned short>(sw[jj] >> (16 * h))));
                            bb = __half2float(__ushort_as_half(static_cast<unsigned short>(bw[jj] >> (16 * h))));
                        }
                        const float2 b2 = make_float2(bb, bb);
                        const float4* xsq = reinterpret_cast<const float4*>(xsp + q * NT);
#pragma unroll
                        for (int t4 = 0; t4 < NT / 4; ++t4) {
                            const float4 v = xsq[t4];
                            yacc[2 * t4] = fma2(b2, make_float2(v.x, v.y), yacc[2 * t4]);
                            yacc[2 * t4 + 1] = fma2(b2, make_float2(v.z, v.w), yacc[2 * t4 + 1]);
                        }
                    }
                }
                got = ptx::mbar_wait(&done[sl], (pc / NS) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (2 * j + h < ng) {
                        const float2 s2 = make_float2(sc[h], sc[h]);
#pragma unroll
                        for (int half = 0; half < NT / 16; ++half) {
                            uint32_t dv[16];
                            ptx::tmem_ld_32x32b_x16(tmem_base + lane_addr + L::kAccCol +
                                                        static_cast<uint32_t>((2 * sl + h) * NT + 16 * half), dv);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int t2 = 0; t2 < 8; ++t2)
                                yacc[8 * half + t2] = fma2(s2, make_float2(__uint_as_float(dv[2 * t2]), __uint_as_float(dv[2 * t2 + 1])),
                                                           yacc[8 * half + t2]);
                        }
                    }
                }
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&ready[sl]);
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&p_empty[pr]);
            pb += static_cast<uint32_t>(np);
            // end of this tile's segment: write this copy's partial and start over
            const bool seg_end = (i + 1 == nchunks) || (cp.cq + 1 == p.cpt);
            if (seg_end) {
                float* dst = p.partial +
                             (((static_cast<int64_t>(blockIdx.x) * p.segmax + (w - w_first)) * 2 + copy) * p.M) * BW;
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    if (t < p.M) dst[static_cast<int64_t>(t) * BW + r] = (t & 1) ? yacc[t >> 1].y : yacc[t >> 1].x;
#pragma unroll
                for (int t = 0; t < NT / 2; ++t) yacc[t] = make_float2(0.0f, 0.0f);
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

// y[t][n] = 2^rowexp[t] * (sum over the CTAs whose runs cover tile n/128, in CTA order, of their two
// partials for that tile).  One CTA per (tile, 2 tokens): thread 0 lists the covering CTAs' segment
// bases once, the other threads only load and add.
constexpr int kMaxCtas = 256;                // the planner launches at most this many CTAs, so every
                                             // tile's covering CTAs fit the reduce kernel's list
template <bool kBf16Out>
__global__ void __launch_bounds__(256) skinny_reduce_kernel(const float* __restrict__ partial,
                                                            const int* __restrict__ rowexp, void* __restrict__ y,
                                                            int M, int N, int cpt, int64_t units, int P, int segmax) {
    __shared__ int64_t seg_base[kMaxCtas];
    __shared__ int count;
    const int w = blockIdx.x;
    if (threadIdx.x == 0) {
        // CTAs whose run of chunks [first(c), first(c+1)) meets [w*cpt, (w+1)*cpt), in CTA order
        const int64_t lo = static_cast<int64_t>(w) * cpt, hi = lo + cpt;
        int c = static_cast<int>((lo * P) / units);
        while (c > 0 && run_first(units, P, c) > lo) --c;
        while (c + 1 <= P && run_first(units, P, c + 1) <= lo) ++c;
        int k = 0;
        int64_t f0 = run_first(units, P, c);
        for (; c < P && f0 < hi; ++c) {
            const int64_t f1 = run_first(units, P, c + 1);
            if (f1 > f0) {                                        // non-empty run
                const int w_first = static_cast<int>(f0 / cpt);
                seg_base[k++] = (static_cast<int64_t>(c) * segmax + (w - w_first)) * 2;
            }
            f0 = f1;
        }
        count = k;
    }
    ptx::grid_dependency_wait();                                  // partials come from the kernel before
    __syncthreads();
    const int t = blockIdx.y * 2 + (threadIdx.x >> 7), r = threadIdx.x & 127;
    const int n = w * BW + r;
    if (t >= M || n >= N) return;
    float acc = 0.0f;
    const int k_end = count;
    for (int k = 0; k < k_end; ++k) {
        const int64_t seg = seg_base[k];
        acc += partial[((seg + 0) * M + t) * BW + r];
        acc += partial[((seg + 1) * M + t) * BW + r];
    }
    acc = ldexpf(acc, rowexp[t]);
    const int64_t e = static_cast<int64_t>(t) * N + n;
    if constexpr (kBf16Out) {
        reinterpret_cast<__nv_bfloat16*>(y)[e] = __float2bfloat16_rn(acc);
    } else {
        reinterpret_cast<float*>(y)[e] = acc;
    }
}

}  // namespace skinny
}  // namespace ql
