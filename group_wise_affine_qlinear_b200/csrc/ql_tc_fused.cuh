// Fused-dequant tensor-core GEMM for large M (tcgen05, TMEM operands and accumulators).
//
// y[m][n] = rowscale[m] * sum_k xh[m][k] * wh(n, k)
//   xh    f16 activations prescaled per row by a power of two (prepass)
//   wh    RN_f16(s * q + b): the affine grid of aimarketly "Ideogram-4-IQ4_M",
//         "What IQ4 means here", formed by one fused f16x2 multiply-add from the
//         exact code q, i.e. rounded once; q is a 4-bit code, or an 8-bit code of
//         the Q8 pack (huggingface "SceneWorks/ideogram-4-mlx", Versions) with the
//         same per-64 scale and bias
// Operands are f16 (A and B must share a type in kind::f16); the accumulator is
// fp32 in tensor memory.  One K-step is exactly one 64-wide quantization group,
// so every weight row needs one (scale, bias) pair per step.
//
// The MMA computes the transposed tile D[n][m] = sum_k wh(n, k) xh(m, k), for
// two groups of 128 weight rows that share one activation tile:
//   A = dequantized weights, 128 rows x 64 k per group, written by the
//       dequantizers straight into tensor memory (tcgen05.st), never into
//       shared memory;
//   B = activations, 192 tokens x 64 k, TMA-loaded into shared memory with the
//       128-byte swizzle, read by both groups' MMAs;
//   D = per group 128 lanes (weight rows) x 192 columns (tokens), fp32.
// Keeping the dequantized tiles out of shared memory leaves shared memory to the
// activation stream, and serving 256 weight rows from each activation tile
// halves the L2 -> SM traffic per FLOP compared with one group.  TMEM holds the
// two accumulators (2 x 192 columns) and two A stages of 2 x 32 columns: all
// 512 columns, so each accumulator is single-buffered; the MMA of the next tile
// waits only for its own group to be drained, which overlaps half the epilogue.
//
// Warp roles of one persistent CTA per SM (640 threads):
//   warps 0-7   dequantizers: warp w owns TMEM lanes 32*(w%4).. of group w/4,
//               one weight row per thread, every K-step
//   warp 8      TMA producer of activation tiles
//   warps 9, 11 single-thread MMA issuers for groups 0 / 1 (warp 9 also allocates TMEM);
//               (one thread issuing for both groups measured slower)
//   warp 10     TMA producer of code and parameter tiles
//   warps 12-19 epilogue: all eight drain group 0, then group 1 (warp w takes TMEM
//               lanes 32*(w%4).. and half of the tokens): TMEM -> registers ->
//               rowscale -> bf16/fp32 -> a 32x32 staging block in shared memory ->
//               TMA tensor store (which also clips the ragged edges of y)
// Rings: X (activation tiles, one K-step each, freed by MMA completion), C (codes +
// parameters of kS consecutive K-steps, freed once the dequantizers have read the
// last of them), A (TMEM weight stages, one K-step each); accumulators are freed per
// group by the epilogue.  Each MMA warp waits on one barrier and commits once per
// K-step: x_full[s] completes when the step's activation tile has landed and the
// dequantizers have written its TMEM stage, and the commit to x_empty[s] frees both
// the x stage and that step's A stage.  Issuing one tcgen05.mma costs its thread
// about 50 cycles, against 96 tensor cycles for a 128 x 192 x 16 MMA, so the
// issuers are held back by the tensor pipe, not by issue.  What the kernel loses
// against the pipe's peak is the time a step is not ready (its weights, its
// activations, a drained accumulator) and the clock that the board's power cap
// leaves while the tensor core and the dequantizers run together.
//
// SwiGLU mode (kSwiGLU): the DiT block's MLP is a SwiGLU of three Linears (jimmysue
// "Ideogram 4" notes, sec. 2.1 and 2.8); this mode fuses the gate and up
// projections and the gating.  A tile's two row groups are the same 128 rows of
// the gate weight (group 0) and of the up weight (group 1), loaded as two
// 128-row code boxes from two tensor maps, with their (scale, bias) pairs
// interleaved the same way by the parameter prepass.  The two accumulators then
// hold g and u for the same 128 intermediate columns and 192 tokens, and each of
// the 8 epilogue warps reads both for its lane quarter and half of the tokens and
// writes h = silu(g) * u = g / (1 + e^-g) * u in fp32 (the exponential and the
// division through the SFU's exp2 and reciprocal), rounded once.
#pragma once

#include "ql_ptx.cuh"
#include "ql_dequant_f16.cuh"

namespace ql {
namespace fused {

constexpr int BWG = 128;                // weight rows per group (MMA M, TMEM lanes)
constexpr int NG = 2;                   // groups per tile
constexpr int BW = NG * BWG;            // weight rows per tile
constexpr int BT = 192;                 // tokens per tile (MMA N, TMEM columns)
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kDequantWarps = 8;
constexpr int kWarpTmaX = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpTmaC = 10;
constexpr int kWarpMma2 = 11;
constexpr int kWarpEpi0 = 12;           // 12..19: quarters 0..3 of group 0, then of group 1
constexpr int kEpiWarps = 4 * NG;
constexpr int kThreads = (kWarpEpi0 + kEpiWarps) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;         // accumulator of group g at columns [g*BT, (g+1)*BT)
constexpr uint32_t kAStageCol = NG * BT;// A stage s, group g at columns [384 + 64 s + 32 g, +32)
constexpr int NA = 2;                   // TMEM weight stages
static_assert(kAStageCol + NA * NG * 32 <= kTmemCols, "tensor memory budget");

constexpr uint32_t kXBytes = BT * BK * 2;   // 24 KB
constexpr uint32_t kCodeRowBytes = 128;     // code bytes of one weight row per code stage

// NX activation stages; NC code stages, each holding kS = 128 / (8 * B) consecutive K-steps of B-bit
// codes (128 bytes of every one of the tile's 256 rows, stored with the 128-byte swizzle: 4 steps of
// 4-bit codes, 2 of 8-bit codes) with their (scale, bias) pairs; epilogue staging blocks of 32 x 32
// outputs of OB bytes each (2: bf16, 4: fp32), NB of them per epilogue warp.  Wide code rows keep the
// number of rows the TMA unit fetches per K-step low (64 rows of 128 bytes instead of 256 of 32); the
// narrower bf16 staging leaves room for a fifth activation stage.
template <int NX, int NC, int B, int OB, int NB>
struct Cfg {
    static constexpr int kNX = NX, kNC = NC, kBits = B, kOutBytes = OB, kNB = NB;
    static constexpr int kS = kCodeRowBytes / (BK * B / 8);
    static constexpr uint32_t kCBytes = BW * kCodeRowBytes;
    static constexpr uint32_t kPBytes = BW * 4 * kS;
    static constexpr uint32_t kStageBytes = 32 * 32 * OB;
    static constexpr uint32_t kEpiBytes = kEpiWarps * NB * kStageBytes;
    static constexpr uint32_t kOffX = 0;
    static constexpr uint32_t kOffC = kOffX + NX * kXBytes;
    static constexpr uint32_t kOffP = kOffC + NC * kCBytes;
    static constexpr uint32_t kOffEpi = kOffP + NC * kPBytes;
    static constexpr uint32_t kOffBar = kOffEpi + kEpiBytes;
    static constexpr uint32_t kNumBars = 2 * NX + 2 * NC + 1 + NG + NG;
    // the A stage of K-step i is released by the x_empty phase of step i - NA, which must not complete
    // its next phase (step i - NA + NX) before the dequantizers have written step i
    static_assert(NX >= NA, "the activation ring is at least as deep as the TMEM weight ring");
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;   // + alignment slack
    static_assert(kXBytes % 1024 == 0 && kCBytes % 1024 == 0, "swizzle atoms need 1 KB alignment");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// The configuration of each (code width, output type): bf16 outputs stage in half the space of fp32
// ones (split-K partials, fp32 outputs), which keep one staging block per warp to stay in budget.
template <int B, bool kBf16Out>
struct PickCfg;
template <> struct PickCfg<4, true> { using type = Cfg<5, 2, 4, 2, 2>; };
template <> struct PickCfg<4, false> { using type = Cfg<4, 2, 4, 4, 1>; };
template <> struct PickCfg<8, true> { using type = Cfg<5, 2, 8, 2, 2>; };
template <> struct PickCfg<8, false> { using type = Cfg<4, 2, 8, 4, 1>; };

struct Params {
    float* rowscale;      // [M] 2^e_m
    void* y;              // [M][N] bf16 or fp32
    int M, N, G;
    int num_t, num_w;     // token tiles, weight tiles
    int splits;           // K slices per tile (split-K instantiations; 1 otherwise)
};

__device__ __forceinline__ void tile_coords(int t, int num_w, int& t_blk, int& w_blk) {
    // weight tiles fastest: a wave of CTAs shares one or two activation row blocks
    // (streamed from HBM once) and sweeps the whole (L2-resident) packed weight.
    t_blk = t / num_w;
    w_blk = t - t_blk * num_w;
}

// Position in a ring of N stages for the i-th use overall.
template <int N>
__device__ __forceinline__ void ring_pos(uint32_t i, int& stage, uint32_t& phase) {
    stage = static_cast<int>(i % N);
    phase = (i / N) & 1u;
}

// map_codes2: the up weight's codes in SwiGLU mode (128-row boxes, like map_codes there); unused otherwise.
// kSplitK: every tile's K-steps are cut into p.splits slices, each its own work unit; a unit writes the
// fp32 partial of its slice through map_y, a 3-D map over partials [splits][M][N], and a separate
// reduction sums the slices in order (for shapes with fewer tiles than SMs).
template <bool kBf16Out, class C, bool kSwiGLU = false, bool kSplitK = false>
__global__ void __launch_bounds__(kThreads, 1) fused_gemm_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_codes,
    const __grid_constant__ CUtensorMap map_codes2, const __grid_constant__ CUtensorMap map_params,
    const __grid_constant__ CUtensorMap map_y, const Params p) {
    constexpr int NX = C::kNX, NC = C::kNC;
    static_assert(!kSwiGLU || C::kBits == 4, "the SwiGLU pair is built for 4-bit codes");
    static_assert(!kSplitK || (!kSwiGLU && !kBf16Out), "split-K units write fp32 partials of a plain layer");
    static_assert(kBf16Out == (C::kOutBytes == 2), "the staging blocks are sized for the output type");
    constexpr int kCodeWords = BK * C::kBits / 32;      // 32-bit code words of one row per K-step
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* x_full = bars;
    uint64_t* x_empty = x_full + NX;
    uint64_t* c_full = x_empty + NX;
    uint64_t* c_empty = c_full + NC;
    uint64_t* acc_full = c_empty + NC;          // one per tile
    uint64_t* acc_empty = acc_full + 1;         // one per group
    uint64_t* drain = acc_empty + NG;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.num_t * p.num_w;
    // Work units: a tile, or with kSplitK a (K slice, tile) pair, slice-major so that a wave of CTAs still
    // shares activation row blocks.  Unit u covers the K-steps [kb0, kb1) of tile t.
    const int num_units = kSplitK ? num_tiles * p.splits : num_tiles;
    auto unit = [&](int u, int& t, int& kb0, int& kb1) {
        if constexpr (kSplitK) {
            const int z = u / num_tiles;
            t = u - z * num_tiles;
            kb0 = static_cast<int>((static_cast<int64_t>(z) * p.G) / p.splits);
            kb1 = static_cast<int>((static_cast<int64_t>(z + 1) * p.G) / p.splits);
        } else {
            t = u;
            kb0 = 0;
            kb1 = p.G;
        }
    };
    // Every role walks the same units in the same order: the X and A ring positions follow the K-step
    // count, the C ring position the code-stage count (a unit's steps in stages of kS, the last partial).

    if (threadIdx.x == 0) {
        // a K-step's x stage is released by both MMA warps' commits, which also release its A stage
        // x_full[s]: the step's activation tile has landed (the producer's expect_tx and the TMA) and its
        // TMEM weight stage is written (one arrival per dequantizer warp), so the MMA warps wait once
        for (int i = 0; i < NX; ++i) { ptx::mbar_init(&x_full[i], 1 + kDequantWarps); ptx::mbar_init(&x_empty[i], NG); }
        for (int i = 0; i < NC; ++i) { ptx::mbar_init(&c_full[i], 1); ptx::mbar_init(&c_empty[i], kDequantWarps); }
        ptx::mbar_init(&acc_full[0], NG);
        static_assert(kWarpEpi0 % 4 == 0, "epilogue warp w must own TMEM lane quarter w % 4");
        // an accumulator is drained by all 8 epilogue warps (a lane quarter and half of the tokens each)
        for (int g = 0; g < NG; ++g) ptx::mbar_init(&acc_empty[g], kEpiWarps);
        for (int g = 0; g < NG; ++g) ptx::mbar_init(drain + g, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTmaX && lane == 0) ptx::prefetch_tensormap(&map_x);
    if (warp == kWarpEpi0 && lane == 0) ptx::prefetch_tensormap(&map_y);
    if (warp == kWarpTmaC && lane == 0) {
        ptx::prefetch_tensormap(&map_codes);
        if constexpr (kSwiGLU) ptx::prefetch_tensormap(&map_codes2);
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
        test_delay(kDelayDequant);   // the checked build can hold this role back (qlinear_test_delay)
        const int grp = warp >> 2;                 // weight-row group
        const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
        const int r = grp * BWG + quarter * 32 + lane;   // weight row within the tile
        const int sw = r & 7;                      // the 128-byte swizzle of row r's 16-byte pieces
        const uint8_t* crow0 = smem + C::kOffC + r * kCodeRowBytes;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t i = 0, ci = 0;                    // K-step and code-stage counters
        bool ok = true;
        for (int un = blockIdx.x; un < num_units && ok; un += gridDim.x) {
            int t, kb0, kb1;
            unit(un, t, kb0, kb1);
            for (int kc = kb0; kc < kb1 && ok; kc += C::kS, ++ci) {
                int cs;
                uint32_t cph;
                ring_pos<NC>(ci, cs, cph);
                // Codes arrive far ahead of the tensor core: unpack them into registers first
                // and wait for the TMEM stage only when the result is ready to be written.
                if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(&c_full[cs], cph, abort_flag))) { ok = false; break; }
                const uint8_t* crow = crow0 + cs * C::kCBytes;
                const uint32_t* sbs = reinterpret_cast<const uint32_t*>(smem + C::kOffP + cs * C::kPBytes);
                const int nsteps = min(C::kS, kb1 - kc);
                for (int st = 0; st < nsteps; ++st, ++i) {
                    const int as = static_cast<int>(i % NA);
                    uint32_t a[32];
                    const uint32_t sb = sbs[st * BW + r];
                    const __half2 sb2 = half2_of(sb);
                    const __half2 s2 = __low2half2(sb2);
                    const __half2 b2 = __high2half2(sb2);
                    if constexpr (C::kBits == 4) {
                        // step st is pieces 2st, 2st+1 of the row (16 codes each)
                        const uint4 c0 = *reinterpret_cast<const uint4*>(crow + (((2 * st) ^ sw) << 4));
                        const uint4 c1 = *reinterpret_cast<const uint4*>(crow + (((2 * st + 1) ^ sw) << 4));
                        if (st + 1 == nsteps) {            // the stage's codes and parameters are in registers
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(&c_empty[cs]);
                        }
                        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                        for (int c = 0; c < 8; ++c) dequant_word(words[c], s2, b2, &a[4 * c]);
                    } else {
                        // step st is pieces 4st .. 4st+3 of the row (16 byte codes each)
                        uint4 cv[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            cv[c] = *reinterpret_cast<const uint4*>(crow + (((4 * st + c) ^ sw) << 4));
                        if (st + 1 == nsteps) {
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(&c_empty[cs]);
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            dequant_word8(cv[c].x, s2, b2, &a[8 * c + 0]);
                            dequant_word8(cv[c].y, s2, b2, &a[8 * c + 2]);
                            dequant_word8(cv[c].z, s2, b2, &a[8 * c + 4]);
                            dequant_word8(cv[c].w, s2, b2, &a[8 * c + 6]);
                        }
                    }
                    // TMEM stage `as` was last read by the MMAs of K-step i - NA: their commit completes
                    // that step's x_empty phase (one commit per MMA warp releases both stages)
                    if (i >= static_cast<uint32_t>(NA)) {
                        int xs;
                        uint32_t xph;
                        ring_pos<NX>(i - NA, xs, xph);
                        if (!__all_sync(0xFFFFFFFFu, ptx::mbar_wait(&x_empty[xs], xph, abort_flag))) {
                            ok = false;
                            break;
                        }
                    }
                    ptx::tc_fence_after_sync();
                    ptx::tmem_st_32x32b_x32(tmem_base + lane_addr + kAStageCol + 64u * as + 32u * grp, a);
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&x_full[i % NX]);   // TMEM stage of step i written
                }
            }
        }
    } else if (warp == kWarpTmaX) {
        // ---------------------------------------------------------------- TMA producer of activation tiles
        test_delay(kDelayActivations);   // the checked build can hold this role back (qlinear_test_delay)
        if (lane == 0) {
            uint32_t i = 0;
            bool ok = true;
            ptx::grid_dependency_wait();               // the activations come from the prepass
            for (int un = blockIdx.x; un < num_units && ok; un += gridDim.x) {
                int t, kb0, kb1;
                unit(un, t, kb0, kb1);
                int t_blk, w_blk;
                tile_coords(t, p.num_w, t_blk, w_blk);
                for (int kb = kb0; kb < kb1; ++kb, ++i) {
                    int s;
                    uint32_t ph;
                    ring_pos<NX>(i, s, ph);
                    if (!ptx::mbar_wait(&x_empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&x_full[s], kXBytes);
                    ptx::tma_load_2d(smem + C::kOffX + s * kXBytes, &map_x, &x_full[s], kb * BK, t_blk * BT);
                }
            }
            // Never leave the CTA with bulk copies still landing in its shared memory:
            // wait for the most recent load of every stage that received one.
            for (uint32_t j = (i > static_cast<uint32_t>(NX) ? i - NX : 0u); j < i; ++j)
                ptx::mbar_wait(&x_full[j % NX], (j / NX) & 1u, nullptr);
        }
    } else if (warp == kWarpTmaC) {
        // ---------------------------------------------------------------- TMA producer of codes and parameters
        test_delay(kDelayCodes);   // the checked build can hold this role back (qlinear_test_delay)
        // (the checked build's stall hook holds it back: no code or parameter load)
        if (lane == 0 && !stalled(kStallFused)) {
            // one code stage: kS K-steps of a tile's 256 rows (in SwiGLU mode 128 gate rows, then the same
            // 128 rows of the up weight); steps past the tensor's K are zero-filled, steps of the next
            // split-K slice are loaded and not used
            auto load_codes = [&](uint8_t* dst, uint64_t* bar, int kc, int w_blk) {
                if constexpr (kSwiGLU) {
                    ptx::tma_load_2d(dst, &map_codes, bar, kc * kCodeWords, w_blk * BWG);
                    ptx::tma_load_2d(dst + C::kCBytes / 2, &map_codes2, bar, kc * kCodeWords, w_blk * BWG);
                } else {
                    ptx::tma_load_2d(dst, &map_codes, bar, kc * kCodeWords, w_blk * BW);
                }
            };
            // The parameter pairs come from the prepass (the transpose, whose completion the conversion
            // just before this kernel on the stream implies; programmatic dependent launch): the code
            // loads of the first NC stages go out at once, their parameter loads (same stage barrier)
            // once the prepass is done.
            uint32_t ci = 0;
            bool ok = true, waited = false;
            int first_kc[NC], first_w[NC];
            for (int un = blockIdx.x; un < num_units && ok; un += gridDim.x) {
                int t, kb0, kb1;
                unit(un, t, kb0, kb1);
                int t_blk, w_blk;
                tile_coords(t, p.num_w, t_blk, w_blk);
                for (int kc = kb0; kc < kb1; kc += C::kS, ++ci) {
                    int s;
                    uint32_t ph;
                    ring_pos<NC>(ci, s, ph);
                    if (ci >= static_cast<uint32_t>(NC) && !waited) {
                        ptx::grid_dependency_wait();
#pragma unroll
                        for (int e = 0; e < NC; ++e)
                            ptx::tma_load_2d(smem + C::kOffP + e * C::kPBytes, &map_params, &c_full[e],
                                             first_w[e] * BW, first_kc[e]);
                        waited = true;
                    }
                    if (!ptx::mbar_wait(&c_empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&c_full[s], C::kCBytes + C::kPBytes);
                    load_codes(smem + C::kOffC + s * C::kCBytes, &c_full[s], kc, w_blk);
                    if (waited) {
                        ptx::tma_load_2d(smem + C::kOffP + s * C::kPBytes, &map_params, &c_full[s], w_blk * BW, kc);
                    } else {
#pragma unroll
                        for (int e = 0; e < NC; ++e) {     // constant indices keep the arrays in registers
                            if (e == s) {
                                first_kc[e] = kc;
                                first_w[e] = w_blk;
                            }
                        }
                    }
                }
            }
            if (!waited) {                             // fewer than NC stages in all
                ptx::grid_dependency_wait();
#pragma unroll
                for (int e = 0; e < NC; ++e)
                    if (static_cast<uint32_t>(e) < ci)
                        ptx::tma_load_2d(smem + C::kOffP + e * C::kPBytes, &map_params, &c_full[e], first_w[e] * BW,
                                         first_kc[e]);
            }
            for (uint32_t j = (ci > static_cast<uint32_t>(NC) ? ci - NC : 0u); j < ci; ++j)
                ptx::mbar_wait(&c_full[j % NC], (j / NC) & 1u, nullptr);
        }
    } else if (warp == kWarpMma || warp == kWarpMma2) {
        // ---------------------------------------------------------------- MMA issuers, one per group
        test_delay(kDelayMma);   // the checked build can hold this role back (qlinear_test_delay)
        const int gsel = warp == kWarpMma ? 0 : 1;
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_f16(BWG, BT, false);
            uint32_t i = 0;
            bool ok = true;
            int j = 0;
            for (int un = blockIdx.x; un < num_units && ok; un += gridDim.x, ++j) {
                int t, kb0, kb1;
                unit(un, t, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++i) {
                    int xs;
                    uint32_t xph;
                    ring_pos<NX>(i, xs, xph);
                    const int as = static_cast<int>(i % NA);
                    if (!ptx::mbar_wait(&x_full[xs], xph, abort_flag)) { ok = false; break; }   // x and A of step i
                    ptx::tc_fence_after_sync();
                    const uint32_t x_addr = ptx::smem_addr(smem + C::kOffX + xs * kXBytes);
                    {
                        const int g = gsel;
                        if (kb == kb0) {
                            // the previous unit's group-g results must have been drained
                            if (!ptx::mbar_wait(&acc_empty[g], (j & 1) ^ 1, abort_flag)) { ok = false; break; }
                            ptx::tc_fence_after_sync();
                        }
                        const uint32_t d = tmem_base + kAccCol + static_cast<uint32_t>(g * BT);
                        const uint32_t a_tm = tmem_base + kAStageCol + 64u * as + 32u * g;
#pragma unroll
                        for (int u = 0; u < BK / UK; ++u) {
                            ptx::mma_f16_ts(d, a_tm + u * (UK / 2), ptx::sdesc_sw128(x_addr + u * UK * 2), idesc,
                                            ((kb - kb0) | u) != 0);
                        }
                    }
                    if (!ok) break;
                    ptx::mma_commit(&x_empty[xs]);         // releases the x stage and the A stage
                }
                if (ok) ptx::mma_commit(&acc_full[0]);
            }
            // Wait until every MMA this thread issued has finished before TMEM is released.
            ptx::mma_commit(drain + gsel);
            ptx::mbar_wait(drain + gsel, 0, nullptr);
        }
    } else if (kSwiGLU && warp >= kWarpEpi0) {
        // ---------------------------------------------------------------- SwiGLU epilogue
        test_delay(kDelayEpilogue);   // the checked build can hold this role back (qlinear_test_delay)
        // Warp (quarter, half) reads the gate and up accumulators of TMEM lanes 32*quarter .. +31 (its
        // 32 intermediate columns) for the token chunks kHalfChunks*half .. +kHalfChunks-1.
        constexpr int kHalfChunks = BT / 32 / 2;
        const int quarter = warp & 3;
        const int half = (warp - kWarpEpi0) >> 2;
        uint8_t* epi_stage = smem + C::kOffEpi + (warp - kWarpEpi0) * C::kNB * C::kStageBytes;
        uint32_t nstore = 0;
        int j = 0;
        ptx::grid_dependency_wait();               // the row scales come from the kernels before this one
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++j) {
            int t_blk, w_blk;
            tile_coords(t, p.num_w, t_blk, w_blk);
            // rs[c] belongs to token t_blk*BT + 32*(kHalfChunks*half + c) + lane
            float rs[kHalfChunks];
#pragma unroll
            for (int c = 0; c < kHalfChunks; ++c) {
                const int m = t_blk * BT + 32 * (kHalfChunks * half + c) + lane;
                rs[c] = (m < p.M) ? p.rowscale[m] : 0.0f;
            }
            const bool got = ptx::mbar_wait(&acc_full[0], j & 1, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            ptx::tc_fence_after_sync();
            const int n_base = w_blk * BWG + quarter * 32;      // this warp's 32 intermediate columns
            const uint32_t tgate = tmem_base + kAccCol + (static_cast<uint32_t>(quarter * 32) << 16);
            const uint32_t tup = tgate + static_cast<uint32_t>(BT);
#pragma unroll
            for (int c = 0; c < kHalfChunks; ++c) {
                const int chunk = kHalfChunks * half + c;
                uint32_t rg[32], ru[32];
                ptx::tmem_ld_32x32b_x32(tgate + chunk * 32, rg);
                ptx::tmem_ld_32x32b_x32(tup + chunk * 32, ru);
                ptx::tmem_wait_ld();
                uint8_t* stage = epi_stage + (nstore % C::kNB) * C::kStageBytes;
                if (lane == 0) ptx::bulk_wait_group_read<C::kNB - 1>();   // the store that used this buffer has read it
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float sc = __shfl_sync(0xFFFFFFFFu, rs[c], k);
                    const float gv = __uint_as_float(rg[k]) * sc;
                    const float uv = __uint_as_float(ru[k]) * sc;
                    // the hardware exponential and reciprocal (a few fp32 ulps, far inside the bf16
                    // rounding that follows); -inf gives NaN and large negative g gives -0 as before
                    const float h = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
                    if constexpr (kBf16Out) {
                        reinterpret_cast<__nv_bfloat16*>(stage)[k * 32 + lane] = __float2bfloat16_rn(h);
                    } else {
                        reinterpret_cast<float*>(stage)[k * 32 + lane] = h;
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    ptx::tma_store_2d(&map_y, stage, n_base, t_blk * BT + chunk * 32);
                    ptx::bulk_commit_group();
                }
                ++nstore;
            }
            ptx::tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&acc_empty[0]);
                ptx::mbar_arrive(&acc_empty[1]);
            }
        }
        if (lane == 0) ptx::bulk_wait_group_all();   // every store has completed before the CTA exits
    } else if (warp >= kWarpEpi0) {
        // ---------------------------------------------------------------- epilogue
        test_delay(kDelayEpilogue);   // the checked build can hold this role back (qlinear_test_delay)
        // All 8 warps drain group 0's accumulator first, then group 1's: warp (quarter, half) takes TMEM
        // lanes 32*quarter .. +31 and the token chunks kHalf*half .. +kHalf-1 of each group, so group 0 is
        // released after half a drain and its MMAs of the next unit run while group 1 is drained.
        constexpr int kHalf = BT / 32 / 2;         // token chunks of 32 per warp and group
        const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
        const int half = (warp - kWarpEpi0) >> 2;
        uint8_t* epi_stage = smem + C::kOffEpi + (warp - kWarpEpi0) * C::kNB * C::kStageBytes;
        uint32_t nstore = 0;
        int j = 0;
        ptx::grid_dependency_wait();               // the row scales come from the kernels before this one
        for (int un = blockIdx.x; un < num_units; un += gridDim.x, ++j) {
            int t, kb0, kb1;
            unit(un, t, kb0, kb1);
            int t_blk, w_blk;
            tile_coords(t, p.num_w, t_blk, w_blk);
            // Row scales of this warp's tokens, fetched before the accumulators are ready:
            // rs[c] belongs to token t_blk*BT + 32*(kHalf*half + c) + lane.
            float rs[kHalf];
#pragma unroll
            for (int c = 0; c < kHalf; ++c) {
                const int m = t_blk * BT + 32 * (kHalf * half + c) + lane;
                rs[c] = (m < p.M) ? p.rowscale[m] : 0.0f;
            }
            const bool got = ptx::mbar_wait(&acc_full[0], j & 1, abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            ptx::tc_fence_after_sync();
#pragma unroll 1
            for (int g = 0; g < NG; ++g) {
                const int n_base = w_blk * BW + g * BWG + quarter * 32;   // this warp's 32 output columns
                const uint32_t taddr = tmem_base + kAccCol + static_cast<uint32_t>(g * BT + 32 * kHalf * half) +
                                       (static_cast<uint32_t>(quarter * 32) << 16);
                // Two register buffers: the TMEM load of chunk c+1 is in flight while chunk c is stored.
                uint32_t r[2][32];
                ptx::tmem_ld_32x32b_x32(taddr, r[0]);
#pragma unroll
                for (int c = 0; c < kHalf; ++c) {
                    const int chunk = kHalf * half + c;
                    ptx::tmem_wait_ld();
                    if (c + 1 < kHalf) ptx::tmem_ld_32x32b_x32(taddr + (c + 1) * 32, r[(c + 1) & 1]);
                    const uint32_t* v = r[c & 1];
                    // staging block [32 tokens][32 columns], C::kNB of them per warp
                    uint8_t* stage = epi_stage + (nstore % C::kNB) * C::kStageBytes;
                    if (lane == 0) ptx::bulk_wait_group_read<C::kNB - 1>();   // the store that used this buffer has read it
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const float val = __uint_as_float(v[k]) * __shfl_sync(0xFFFFFFFFu, rs[c], k);
                        if constexpr (kBf16Out) {
                            reinterpret_cast<__nv_bfloat16*>(stage)[k * 32 + lane] = __float2bfloat16_rn(val);
                        } else {
                            reinterpret_cast<float*>(stage)[k * 32 + lane] = val;
                        }
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (kSplitK) {
                            ptx::tma_store_3d(&map_y, stage, n_base, t_blk * BT + chunk * 32, un / num_tiles);
                        } else {
                            ptx::tma_store_2d(&map_y, stage, n_base, t_blk * BT + chunk * 32);
                        }
                        ptx::bulk_commit_group();
                    }
                    ++nstore;
                }
                ptx::tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&acc_empty[g]);
            }
        }
        if (lane == 0) ptx::bulk_wait_group_all();   // every store has completed before the CTA exits
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
