// Weight-streaming tensor-core path for small M (M <= 32): HBM-bound, so the job
// is to read the 4.5-bit weights once at full bandwidth and spend as few
// instructions and as few cross-warp handshakes per weight as possible.
//
// The weight of row n, column k is w = s(n,g) q(n,k) + b(n,g) for the 64-group g
// holding k (aimarketly "Ideogram-4-IQ4_M", "What IQ4 means here": w = scale * q +
// bias).  Builder warps dequantize each group of a 128-row weight tile to the f16
// operand RN_f16(s q + b) (4-bit codes, dequant_word: one shift, four LOP3, four
// HSUB2 and four HFMA2 per 8 weights; 8-bit codes, dequant_word8: two byte permutes,
// two HSUB2 and two HFMA2 per 4 weights) straight into tensor memory, and tcgen05.mma (kind::f16,
// M = 128 weight rows, N = 16 or 32 tokens, fp32 accumulation) accumulates the
// whole run of groups the CTA owns in one tile, so nothing but the tensor core
// touches the partial sums until the CTA leaves the tile.  This is the large-M
// kernel's arithmetic (one f16 rounding of each weight, activations scaled per
// row by a power of two into f16, fp32 accumulation) in a layout for few tokens.
//
// The activations come from one prepass kernel (a cluster of CTAs per row that
// meet in distributed shared memory for the row maximum), which the main kernel
// follows under programmatic dependent launch: x' = f16(x * 2^e_t) with e_t putting
// the row maximum in [2^14, 2^15), in the order the dequantizer emits its pairs in
// (0,4,1,5,2,6,3,7 of every 8-block for 4-bit codes, 0,2,1,3,4,6,5,7 for 8-bit
// codes).  The main kernel starts streaming codes and parameters at once and waits
// for the prepass only before its first activation load.
//
// Stream-K schedule: the work is cut into chunks of CG consecutive groups of one
// 128-row tile (CG = 8 for 4-bit codes, 4 for the 8-bit codes of the Q8 pack,
// huggingface "SceneWorks/ideogram-4-mlx", Versions; either way 32 KB of codes; a
// tile has ceil(G/CG) chunks; a tile's last chunk may be partial).  The chunks, tile-major, are split into one equal contiguous run per
// CTA; each tile segment a run covers leaves one fp32 partial [tokens][128]
// (scaled by 2^e_t) in the workspace, and the reduce kernel sums, per output, the
// partials of the CTAs that covered its tile in CTA order (deterministic) and
// scales back by 2^-e_t.
//
// Roles step over pairs of consecutive groups of a chunk (pair j = groups 2j,
// 2j+1), numbered pc along the run: four builder copies (pc % 4) and two MMA
// issuers (pc % 2), each issuer accumulating into an accumulator of its own.  A
// ring of NA pair stages in tensor memory sits between them (a_full: the 4
// builder warps of the stage's copy; a_empty: the issuer's commit).  At the end
// of a tile segment both issuers commit to acc_full, and the drain warps add the
// two accumulators and write the partial; the accumulators are double-buffered
// across segments (acc_empty).
// Warp roles (768 threads, one CTA per SM; 6 warps per SM sub-partition leave 80 registers a thread):
//   warp 0        TMA producer of code chunks (128 rows x 256 B, 128B swizzle) with their scale and
//                 bias tiles
//   warp 1        TMA producer of activation tiles (NT x 64 f16 per group), its own ring: activation
//                 loads from L2 take about a microsecond, so they run several chunks ahead
//   warps 2, 3    MMA issuers for even / odd pairs (warp 2 also allocates TMEM)
//   warps 4-19    A builders, copies 0-3 of 4 warps: one weight row per thread
//   warps 20-23   drain: one weight row per thread, at the end of each tile segment
#pragma once

#include "ql_ptx.cuh"
#include "ql_dequant_f16.cuh"

namespace ql {
namespace skinny {

constexpr int BW = 128;
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kBuildCopies = 4, kMmaCopies = 2;
constexpr int kWarpTmaC = 0, kWarpTmaX = 1, kWarpMma0 = 2, kWarpBuild0 = 4, kWarpDrain0 = kWarpBuild0 + 4 * kBuildCopies;
constexpr int kThreads = (kWarpDrain0 + 4) * 32;
constexpr int NA = 4;                    // A pair stages in tensor memory
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBoxBytes = BW * 128;                     // 16 KB: one code box, 128 bytes of each row
constexpr int kParGroups = 8;                                // groups per scale (bias) box: 16-byte rows
constexpr uint32_t kParHalf = BW * kParGroups * 2;           // one box of scales (or biases): [128][8] f16
constexpr int kMaxCtas = 256;                // the planner launches at most this many CTAs, so every
                                             // tile's covering CTAs fit the reduce kernel's list
static_assert(NA % kBuildCopies == 0 && NA % kMmaCopies == 0, "every A stage serves one copy of each role");

// NT tokens, B-bit codes.  A chunk is CG groups: 8 for 4-bit codes (four pairs, one per builder copy),
// 4 for 8-bit codes (two pairs), so either way a chunk's codes are 32 KB in two 128-byte-wide boxes.
template <int NT, int B = 4>
struct Layout {
    static constexpr int kBits = B;
    static constexpr int CG = B == 4 ? 8 : 4;                            // groups per chunk
    static constexpr int kGroupWords = BK * B / 32;                      // code words of one row per group
    static constexpr int kBoxGroups = 128 / (4 * kGroupWords);           // groups per code box
    static constexpr uint32_t kCBytes = kBoxBytes * (CG / kBoxGroups);   // codes per chunk
    static constexpr uint32_t kStageBytes = kCBytes + 2 * kParHalf;      // [codes | scales | biases]
    // code/parameter and activation chunk stages: the activation tiles grow with NT, so the rings shrink
    static constexpr int NC = B == 4 ? (NT == 16 ? 4 : NT == 32 ? 3 : 2) : (NT == 16 ? 5 : NT == 32 ? 4 : 3);
    static constexpr int NXC = B == 4 ? (NT == 16 ? 4 : NT == 32 ? 3 : 2) : (NT == 16 ? 5 : NT == 32 ? 4 : 3);
    static constexpr uint32_t kXTile = NT * BK * 2;                      // one group's activation tile (f16)
    static constexpr uint32_t kXBytes = CG * kXTile;                     // one chunk's activation tiles
    static constexpr uint32_t kOffC = 0;                                  // [NC][codes | scales | biases]
    static constexpr uint32_t kOffX = kOffC + NC * kStageBytes;          // [NXC][CG][x tile], 1 KB aligned
    static constexpr uint32_t kOffBar = kOffX + NXC * kXBytes;
    static constexpr uint32_t kNumBars = 2 * NC + 2 * NXC + 2 * NA + 4 + kMmaCopies;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
    static constexpr uint32_t kAccCol = 0;                                // accumulator (set e, issuer c) at (2e+c)*NT
    static constexpr uint32_t kACol = 4 * NT;                             // A stage st, half h at kACol + 32(2st+h)
    static_assert(B == 4 || B == 8, "4- or 8-bit codes");
    static_assert(NT == 16 || NT == 32 || NT == 64, "MMA N of 16, 32 or 64 tokens");
    static_assert(CG <= 2 * kBuildCopies && CG % kBoxGroups == 0 && kParGroups % CG == 0,
                  "at most one pair of a chunk per builder copy; whole code boxes; whole chunks per parameter box");
    static_assert(kStageBytes % 1024 == 0, "swizzled code boxes need 1 KB alignment");
    static_assert(kXTile % 1024 == 0, "swizzled activation tiles need 1 KB alignment");
    static_assert(kACol + 2 * NA * 32 <= kTmemCols, "tensor memory budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Params {
    float* partial;          // [P][segmax][M][128] fp32, scaled by 2^e_t
    const __half* scales;    // [N][G]
    const __half* biases;    // [N][G]
    int param_tma;           // 1: scales/biases arrive as TMA tiles (needs G % 8 == 0); 0: direct loads
    int M, N, G, num_w;
    int cpt;                 // chunks per tile = ceil(G / CG)
    int64_t units;           // num_w * cpt chunks
    int segmax;
    int64_t partial_elems;   // floats in partial (index checks of the bounds-checked build)
};

// First unit of CTA c's run (runs are [first(c), first(c+1))).
__host__ __device__ __forceinline__ int64_t run_first(int64_t units, int P, int c) {
    return units * c / P;
}

// The activation prepass in one launch, one cluster of kPrepCluster CTAs per row t: each CTA takes
// 1/kPrepCluster of the row's 8-blocks, the CTAs' maxima meet in distributed shared memory, then
// e_t puts max_k |x[t][k]| in [2^14, 2^15) (0 for a zero or non-finite row);
// xp[t][k] = f16(x * 2^e_t) in the order the dequantizer of kBits-bit codes emits its pairs in
// (0,4,1,5,2,6,3,7 of each 8-block for 4-bit codes, 0,2,1,3,4,6,5,7 for 8-bit codes); rowexp[t] = -e_t.
// Grid (kPrepCluster, M); no thread leaves before the second cluster barrier, so every CTA's shared
// memory outlives its peers' reads of it.
constexpr int kPrepCluster = 8;
constexpr int kPrepThreads = 512;
constexpr int kPrepCache = 4;                 // 8-blocks a thread keeps in registers between the passes

__device__ __forceinline__ float absmax8(const uint4 v) {
    return fmaxf(fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))),
                 fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
}

template <int kBits>
__device__ __forceinline__ uint4 prescale8(const uint4 v, int ex) {
    const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // 4-bit: slot pairs (k0, k4) (k1, k5) (k2, k6) (k3, k7); 8-bit: (k0, k2) (k1, k3) (k4, k6) (k5, k7)
        const int lo = kBits == 4 ? j : 2 * (j & 2) + (j & 1);
        const int hi = kBits == 4 ? j + 4 : lo + 2;
        const __half2 h = __halves2half2(__float2half_rn(ldexpf(f[lo], ex)), __float2half_rn(ldexpf(f[hi], ex)));
        o[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int kBits>
__global__ void __cluster_dims__(kPrepCluster, 1, 1) __launch_bounds__(kPrepThreads)
    skinny_prepass_kernel(const uint4* __restrict__ x, uint4* __restrict__ xp, int* __restrict__ rowexp, int K) {
    ptx::launch_dependents();
    __shared__ float red[kPrepThreads / 32];
    const int t = blockIdx.y, kb = K / 8;
    const uint32_t rank = ptx::cluster_ctarank();
    const int per = (kb + kPrepCluster - 1) / kPrepCluster;
    const int c0 = static_cast<int>(rank) * per, c1 = min(kb, c0 + per);
    const uint4* xr = x + static_cast<int64_t>(t) * kb;
    uint4 v[kPrepCache];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < kPrepCache; ++j) {
        const int c = c0 + j * kPrepThreads + static_cast<int>(threadIdx.x);
        v[j] = c < c1 ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
        m = fmaxf(m, absmax8(v[j]));
    }
    for (int c = c0 + kPrepCache * kPrepThreads + static_cast<int>(threadIdx.x); c < c1; c += kPrepThreads)
        m = fmaxf(m, absmax8(xr[c]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < kPrepThreads / 32; ++i) m = fmaxf(m, red[i]);
        red[0] = m;                                   // this CTA's slice maximum
    }
    ptx::cluster_sync();                              // every CTA's red[0] is written
    m = 0.0f;
#pragma unroll
    for (int r = 0; r < kPrepCluster; ++r) m = fmaxf(m, ptx::ld_shared_cluster_f32(&red[0], static_cast<uint32_t>(r)));
    ptx::cluster_sync();                              // every peer has read this CTA's red[0]
    int ex = 0;
    if (m > 0.0f && m <= 3.4028235e38f) {
        int E;
        frexpf(m, &E);                                // m = f 2^E, f in [0.5, 1)
        ex = 15 - E;
    }
    if (rank == 0 && threadIdx.x == 0) rowexp[t] = -ex;
    uint4* xo = xp + static_cast<int64_t>(t) * kb;
#pragma unroll
    for (int j = 0; j < kPrepCache; ++j) {
        const int c = c0 + j * kPrepThreads + static_cast<int>(threadIdx.x);
        if (c < c1) xo[c] = prescale8<kBits>(v[j], ex);
    }
    for (int c = c0 + kPrepCache * kPrepThreads + static_cast<int>(threadIdx.x); c < c1; c += kPrepThreads)
        xo[c] = prescale8<kBits>(xr[c], ex);
}

template <int NT, int B>
__global__ void __launch_bounds__(kThreads, 1) skinny_kernel(const __grid_constant__ CUtensorMap map_codes,
                                                            const __grid_constant__ CUtensorMap map_x,
                                                            const __grid_constant__ CUtensorMap map_scales,
                                                            const __grid_constant__ CUtensorMap map_biases,
                                                            const Params p) {
    using L = Layout<NT, B>;
    constexpr int NC = L::NC;
    constexpr int NXC = L::NXC;
    constexpr int CG = L::CG;
    constexpr int kBoxGroups = L::kBoxGroups;
    constexpr uint32_t kCBytes = L::kCBytes;
    constexpr uint32_t kStageBytes = L::kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* c_full = bars;
    uint64_t* c_empty = c_full + NC;
    uint64_t* x_full = c_empty + NC;
    uint64_t* x_empty = x_full + NXC;
    uint64_t* a_full = x_empty + NXC;
    uint64_t* a_empty = a_full + NA;
    uint64_t* acc_full = a_empty + NA;          // two: one per accumulator set
    uint64_t* acc_empty = acc_full + 2;         // two
    uint64_t* drain = acc_empty + 2;            // one per MMA issuer
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
        for (int i = 0; i < NXC; ++i) { ptx::mbar_init(&x_full[i], 1); ptx::mbar_init(&x_empty[i], kMmaCopies); }
        for (int i = 0; i < NA; ++i) { ptx::mbar_init(&a_full[i], 4); ptx::mbar_init(&a_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { ptx::mbar_init(&acc_full[i], kMmaCopies); ptx::mbar_init(&acc_empty[i], 4); }
        for (int i = 0; i < kMmaCopies; ++i) ptx::mbar_init(&drain[i], 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTmaX && lane == 0) ptx::prefetch_tensormap(&map_x);
    if (warp == kWarpTmaC && lane == 0) {
        ptx::prefetch_tensormap(&map_codes);
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
    // walks its chunks with a (w, cq) position advanced by one per chunk, without dividing.  A tile
    // segment of the run ends with the run or with the tile's last chunk.
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

    if (warp == kWarpTmaC) {
        // ---------------------------------------------------------------- code + parameter producer
        test_delay(kDelayCodes);   // the checked build can hold this role back (qlinear_test_delay)
        // (codes and parameters do not depend on the prepass: no dependency wait; the checked build's
        // stall hook holds this producer back: no code or parameter load at all)
        if (lane == 0 && !stalled(kStallSkinny)) {
            uint32_t ci = 0;
            ChunkPos cp = start;
            for (; ci < nchunks; ++ci, advance(cp)) {
                int w, g0, ng;
                chunk_groups(cp, w, g0, ng);
                const int s = static_cast<int>(ci % NC);
                if (!ptx::mbar_wait(&c_empty[s], ((ci / NC) & 1u) ^ 1u, abort_flag)) break;
                uint8_t* st = smem + L::kOffC + s * kStageBytes;
                ptx::mbar_arrive_expect_tx(&c_full[s], kCBytes + (p.param_tma ? 2 * kParHalf : 0u));
#pragma unroll
                for (int bx = 0; bx < CG / kBoxGroups; ++bx)   // consecutive boxes: long contiguous row segments
                    ptx::tma_load_2d(st + bx * kBoxBytes, &map_codes, &c_full[s], (g0 + bx * kBoxGroups) * L::kGroupWords,
                                     w * BW);
                if (p.param_tma) {
                    // the 8-group box holding the chunk (a chunk of 4 groups uses half of it)
                    const int gp = g0 - g0 % kParGroups;
                    ptx::tma_load_2d(st + kCBytes, &map_scales, &c_full[s], gp, w * BW);
                    ptx::tma_load_2d(st + kCBytes + kParHalf, &map_biases, &c_full[s], gp, w * BW);
                }
            }
            // never leave the CTA with bulk copies still landing in its shared memory
            for (uint32_t j = (ci > static_cast<uint32_t>(NC) ? ci - NC : 0u); j < ci; ++j)
                ptx::mbar_wait(&c_full[j % NC], (j / NC) & 1u, nullptr);
        }
    } else if (warp == kWarpTmaX) {
        // ---------------------------------------------------------------- activation producer
        test_delay(kDelayActivations);   // the checked build can hold this role back (qlinear_test_delay)
        if (lane == 0) {
            ptx::grid_dependency_wait();              // the activations come from the prepass
            uint32_t xi = 0;
            ChunkPos cp = start;
            for (; xi < nchunks; ++xi, advance(cp)) {
                int w, g0, ng;
                chunk_groups(cp, w, g0, ng);
                const int xc = static_cast<int>(xi % NXC);
                if (!ptx::mbar_wait(&x_empty[xc], ((xi / NXC) & 1u) ^ 1u, abort_flag)) break;
                ptx::mbar_arrive_expect_tx(&x_full[xc], static_cast<uint32_t>(ng) * L::kXTile);
                for (int q = 0; q < ng; ++q)
                    ptx::tma_load_2d(smem + L::kOffX + xc * L::kXBytes + q * L::kXTile, &map_x, &x_full[xc], (g0 + q) * BK, 0);
            }
            for (uint32_t j = (xi > static_cast<uint32_t>(NXC) ? xi - NXC : 0u); j < xi; ++j)
                ptx::mbar_wait(&x_full[j % NXC], (j / NXC) & 1u, nullptr);
        }
    } else if (warp < kWarpMma0 + kMmaCopies) {
        // ---------------------------------------------------------------- MMA issuers (even / odd pairs)
        test_delay(kDelayMma);   // the checked build can hold this role back (qlinear_test_delay)
        // The whole warp runs the loop; one elected lane issues the MMAs and the commits.
        const int copy = warp - kWarpMma0;
        const bool leader = ptx::elect_one();
        constexpr uint32_t idesc = ptx::idesc_f16(BW, NT, false);
        const uint64_t xdesc0 = ptx::sdesc_sw128(ptx::smem_addr(smem + L::kOffX));
        uint32_t pb = 0, seg = 0;     // pairs of the run before this chunk; tile segments finished
        bool fresh = true;            // no MMA of this issuer in the current segment yet
        bool ok = true;
        ChunkPos cp = start;
        for (uint32_t i = 0; i < nchunks && ok; ++i, advance(cp)) {
            int w, g0, ng;
            chunk_groups(cp, w, g0, ng);
            const int np = (ng + 1) >> 1;
            const int xc = static_cast<int>(i % NXC);
            const uint32_t set = seg & 1u;
            if (i == 0 || cp.cq == 0) {
                // a new segment: its accumulator set must have been drained (segment seg - 2)
                const bool got = ptx::mbar_wait(&acc_empty[set], ((seg >> 1) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) break;
            }
            bool got = ptx::mbar_wait(&x_full[xc], (i / NXC) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            // descriptor of the chunk's first activation tile (the address field counts 16-byte units)
            const uint64_t xdesc = xdesc0 + ((static_cast<uint32_t>(xc) * L::kXBytes) >> 4);
            const uint32_t d = tmem_base + L::kAccCol + (2u * set + static_cast<uint32_t>(copy)) * NT;
            for (int j = first_pair(pb, copy, kMmaCopies); j < np; j += kMmaCopies) {
                const uint32_t pc = pb + static_cast<uint32_t>(j);
                const int st = static_cast<int>(pc % NA);
                got = ptx::mbar_wait(&a_full[st], (pc / NA) & 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
                if (leader) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (2 * j + h < ng) {
                            const uint32_t a_tm = tmem_base + L::kACol + 32u * static_cast<uint32_t>(2 * st + h);
                            const uint64_t bd = xdesc + ((static_cast<uint32_t>(2 * j + h) * L::kXTile) >> 4);
#pragma unroll
                            for (int u = 0; u < BK / UK; ++u)
                                ptx::mma_f16_ts(d, a_tm + u * (UK / 2), bd + ((u * UK * 2) >> 4), idesc,
                                                (fresh && h == 0 && u == 0) ? 0u : 1u);
                        }
                    }
                    ptx::mma_commit(&a_empty[st]);
                }
                fresh = false;
                __syncwarp();
            }
            if (!ok) break;
            if (leader) ptx::mma_commit(&x_empty[xc]);
            pb += static_cast<uint32_t>(np);
            if (i + 1 == nchunks || cp.cq + 1 == p.cpt) {     // end of the tile segment
                if (leader) ptx::mma_commit(&acc_full[set]);
                ++seg;
                fresh = true;
            }
            __syncwarp();
        }
        if (leader) ptx::mma_commit(&drain[copy]);
        __syncwarp();
        ptx::mbar_wait(&drain[copy], 0, nullptr);
    } else if (warp < kWarpDrain0) {
        // ---------------------------------------------------------------- A builders (four copies)
        test_delay(kDelayDequant);   // the checked build can hold this role back (qlinear_test_delay)
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
            // row r's code bytes of group q (32 for 4-bit codes, 64 for 8-bit codes) sit in code box
            // q / kBoxGroups at the 16-byte pieces kPieces (q % kBoxGroups) .. of its box row, stored with
            // the 128-byte swizzle (piece c at c ^ (r % 8)), so every 8 lanes of a load touch 8 bank
            // groups; its scales and biases of groups 2j, 2j + 1 are one 32-bit word each
            constexpr int kPieces = L::kGroupWords / 4;       // 16-byte pieces per group row: 2 or 4
            uint4 cw[2 * kPieces];
            uint32_t sp = 0u, bp = 0u;
            if (mine) {
                const uint8_t* st = smem + L::kOffC + s * kStageBytes;
                const uint8_t* crow = st + ((2 * j) / kBoxGroups) * kBoxBytes + r * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = kPieces * ((2 * j + h) % kBoxGroups);
                    if (2 * j + h < ng) {
#pragma unroll
                        for (int e = 0; e < kPieces; ++e)
                            cw[kPieces * h + e] = *reinterpret_cast<const uint4*>(crow + (((c + e) ^ (r & 7)) << 4));
                    }
                }
                const int n = w * BW + r;
                if (p.param_tma) {
                    const int pc0 = g0 % kParGroups + 2 * j;        // the pair's first column in the parameter box
                    sp = *reinterpret_cast<const uint32_t*>(st + kCBytes + r * kParGroups * 2 + 2 * pc0);
                    bp = *reinterpret_cast<const uint32_t*>(st + kCBytes + kParHalf + r * kParGroups * 2 + 2 * pc0);
                } else {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int q = 2 * j + h;
                        const int64_t at = static_cast<int64_t>(n) * p.G + g0 + q;
                        if (n < p.N && q < ng && in_bounds(at, static_cast<int64_t>(p.N) * p.G)) {
                            sp |= static_cast<uint32_t>(__half_as_ushort(__ldg(p.scales + at))) << (16 * h);
                            bp |= static_cast<uint32_t>(__half_as_ushort(__ldg(p.biases + at))) << (16 * h);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&c_empty[s]);
            if (mine) {
                const uint32_t pc = pb + static_cast<uint32_t>(j);
                const int st = static_cast<int>(pc % NA);
                // the stage's previous MMAs must have finished reading it
                got = ptx::mbar_wait(&a_empty[st], ((pc / NA) & 1u) ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                ptx::tc_fence_after_sync();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (2 * j + h < ng) {
                        const __half2 s2 = h ? __high2half2(half2_of(sp)) : __low2half2(half2_of(sp));
                        const __half2 b2 = h ? __high2half2(half2_of(bp)) : __low2half2(half2_of(bp));
                        uint32_t a[32];
                        if constexpr (B == 4) {
                            const uint4 c0 = cw[2 * h], c1 = cw[2 * h + 1];
                            const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                            for (int c = 0; c < 8; ++c) dequant_word(words[c], s2, b2, &a[4 * c]);
                        } else {
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint4 cv = cw[4 * h + c];
                                dequant_word8(cv.x, s2, b2, &a[8 * c + 0]);
                                dequant_word8(cv.y, s2, b2, &a[8 * c + 2]);
                                dequant_word8(cv.z, s2, b2, &a[8 * c + 4]);
                                dequant_word8(cv.w, s2, b2, &a[8 * c + 6]);
                            }
                        }
                        ptx::tmem_st_32x32b_x32(tmem_base + lane_addr + L::kACol + 32u * static_cast<uint32_t>(2 * st + h), a);
                    }
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&a_full[st]);
            }
            pb += static_cast<uint32_t>(np);
        }
    } else {
        // ---------------------------------------------------------------- drain (tile segment ends)
        test_delay(kDelayEpilogue);   // the checked build can hold this role back (qlinear_test_delay)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const int w_first = start.w;
        uint32_t pb = 0, seg = 0, seg_pb = 0;    // pairs so far; segments drained; first pair of the segment
        ChunkPos cp = start;
        for (uint32_t i = 0; i < nchunks; ++i, advance(cp)) {
            pb += static_cast<uint32_t>((min(CG, p.G - cp.cq * CG) + 1) >> 1);
            if (!(i + 1 == nchunks || cp.cq + 1 == p.cpt)) continue;
            const uint32_t set = seg & 1u;
            const bool got = ptx::mbar_wait(&acc_full[set], (seg >> 1) & 1u, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            ptx::tc_fence_after_sync();
            // issuer c accumulated in this segment iff one of its pairs (pc = c mod 2) lies in [seg_pb, pb)
            const uint32_t npairs = pb - seg_pb;
            const bool used0 = npairs >= 2 || (npairs == 1 && (seg_pb & 1u) == 0u);
            const bool used1 = npairs >= 2 || (npairs == 1 && (seg_pb & 1u) == 1u);
            float* dst = p.partial + ((static_cast<int64_t>(blockIdx.x) * p.segmax + (cp.w - w_first)) * p.M) * BW;
#pragma unroll
            for (int h16 = 0; h16 < NT / 16; ++h16) {
                uint32_t d0[16], d1[16];
                const uint32_t col = tmem_base + lane_addr + L::kAccCol + 2u * set * NT + 16u * h16;
                if (used0) ptx::tmem_ld_32x32b_x16(col, d0);
                if (used1) ptx::tmem_ld_32x32b_x16(col + NT, d1);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int tt = 16 * h16 + t;
                    if (tt < p.M && in_bounds((dst - p.partial) + static_cast<int64_t>(tt) * BW + r, p.partial_elems))
                        dst[static_cast<int64_t>(tt) * BW + r] = (used0 ? __uint_as_float(d0[t]) : 0.0f) +
                                                                 (used1 ? __uint_as_float(d1[t]) : 0.0f);
                }
            }
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acc_empty[set]);
            ++seg;
            seg_pb = pb;
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

// y[t][n] = 2^rowexp[t] * (sum over the CTAs whose runs cover tile n/128, in CTA order, of their
// partials for that tile).  One CTA per (tile, 2 tokens): thread 0 lists the covering CTAs' segment
// bases once, the other threads only load and add.
template <bool kBf16Out>
__global__ void __launch_bounds__(256) skinny_reduce_kernel(const float* __restrict__ partial,
                                                            const int* __restrict__ rowexp, void* __restrict__ y,
                                                            int M, int N, int cpt, int64_t units, int P, int segmax,
                                                            int64_t partial_elems) {
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
                seg_base[k++] = static_cast<int64_t>(c) * segmax + (w - w_first);
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
        const int64_t at = (seg_base[k] * M + t) * BW + r;
        if (in_bounds(at, partial_elems)) acc += partial[at];
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
