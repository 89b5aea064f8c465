// C ABI of the qlinear library: argument validation, per-shape dispatch,
// workspace layout, tensor-map encoding and launches.  Every kernel of the
// library is included here so the whole library is one device module.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "ql_common.cuh"
#include "ql_dequant.cuh"
#include "ql_gemv.cuh"
#include "ql_pack.cuh"
#include "ql_pack_fit.cuh"
#include "ql_prepass.cuh"
#include "ql_tc_fused.cuh"
#include "ql_tc_skinny.cuh"

namespace ql {

// Self-test of the bounded waits every pipeline role uses: one CTA, two waiting threads (lane 0 of
// warps 0 and 1) on an mbarrier that nothing arrives on.  One of them gives up after the wait limit,
// records QL_ERR_DEVICE_TIMEOUT and raises the shared abort flag; the other returns on that flag
// (or on its own limit).  The kernel ends about one wait limit after it starts.
__global__ void __launch_bounds__(64) wait_selftest_kernel() {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) ptx::mbar_wait(&bar, 0, &abort_flag);   // phase 0 never completes
    __syncthreads();
}

namespace {

constexpr int32_t kVersion = 100;   // 0.1.0
constexpr int kMaxDevices = 64;

thread_local char t_last_dispatch[192] = "none";
thread_local cudaEvent_t t_prof_start = nullptr;
thread_local cudaEvent_t t_prof_stop = nullptr;

void prof_begin(cudaStream_t st) {
    if (t_prof_start && t_prof_stop) cudaEventRecord(t_prof_start, st);
}
void prof_end(cudaStream_t st) {
    if (t_prof_start && t_prof_stop) cudaEventRecord(t_prof_stop, st);
}

void set_dispatch(const char* fmt, ...) __attribute__((format(printf, 1, 2)));
void set_dispatch(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_dispatch, sizeof(t_last_dispatch), fmt, ap);
    va_end(ap);
}

struct DeviceInfo {
    int sm_count = 0;
    bool fused_attr_set = false;
    bool skinny_attr_set = false;
};

template <int NT, int B>
cudaError_t skinny_smem_attr() {
    return cudaFuncSetAttribute(skinny::skinny_kernel<NT, B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                skinny::Layout<NT, B>::kSmemBytes);
}

template <int B, bool kSwiGLU = false>
cudaError_t fused_smem_attr() {
    using FB = typename fused::PickCfg<B, true>::type;
    using FF = typename fused::PickCfg<B, false>::type;
    const cudaError_t e = cudaFuncSetAttribute(fused::fused_gemm_kernel<true, FB, kSwiGLU>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, FB::kSmemBytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(fused::fused_gemm_kernel<false, FF, kSwiGLU>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, FF::kSmemBytes);
}
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

ql_status device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QL_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (d.sm_count == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return QL_ERR_CUDA;
        d.sm_count = n;
    }
    if (!d.fused_attr_set) {
        if (fused_smem_attr<4>() != cudaSuccess || fused_smem_attr<8>() != cudaSuccess ||
            fused_smem_attr<4, true>() != cudaSuccess ||
            cudaFuncSetAttribute(fused::fused_gemm_kernel<false, fused::PickCfg<4, false>::type, false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fused::PickCfg<4, false>::type::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(fused::fused_gemm_kernel<false, fused::PickCfg<8, false>::type, false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fused::PickCfg<8, false>::type::kSmemBytes) != cudaSuccess)
            return QL_ERR_CUDA;
        d.fused_attr_set = true;
    }
    if (!d.skinny_attr_set) {
        if (skinny_smem_attr<16, 4>() != cudaSuccess || skinny_smem_attr<32, 4>() != cudaSuccess ||
            skinny_smem_attr<16, 8>() != cudaSuccess || skinny_smem_attr<32, 8>() != cudaSuccess ||
            skinny_smem_attr<64, 4>() != cudaSuccess || skinny_smem_attr<64, 8>() != cudaSuccess)
            return QL_ERR_CUDA;
        d.skinny_attr_set = true;
    }
    *out = &d;
    return QL_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

ql_status get_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
    std::call_once(g_encode_once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        }
    });
    *fn = g_encode;
    return g_encode ? QL_OK : QL_ERR_CUDA;
}

// 2-D row-major tensor map: inner extent `cols` elements, `rows` rows, row pitch in bytes.
ql_status encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                    uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    if (get_encoder(&enc) != QL_OK) return QL_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QL_OK : QL_ERR_CUDA;
}

// 3-D row-major tensor map: extents (cols, rows, planes) in elements, row and plane pitches in bytes.
ql_status encode_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                    uint64_t planes, uint64_t row_pitch, uint64_t plane_pitch, uint32_t box_cols, uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    if (get_encoder(&enc) != QL_OK) return QL_ERR_CUDA;
    const cuuint64_t dims[3] = {cols, rows, planes};
    const cuuint64_t strides[2] = {row_pitch, plane_pitch};
    const cuuint32_t box[3] = {box_cols, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QL_OK : QL_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na > 0 && nb > 0 && x < y + nb && y < x + na;
}

ql_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------------ shapes and plans

// Bytes of the packed codes of an [N][K] weight with `bits`-bit codes (4 or 8).
size_t code_bytes(int64_t K, int64_t N, int bits) { return static_cast<size_t>(N) * K * bits / 8; }

ql_status check_shape(int64_t M, int64_t K, int64_t N, int32_t group) {
    if (group != kGroup) return QL_ERR_UNSUPPORTED;
    if (M < 1 || K < kGroup || N < 8 || K % kGroup != 0 || N % 8 != 0) return QL_ERR_INVALID_ARG;
    if (M > (1ll << 31) - 1 || K > (1ll << 30) || N > (1ll << 30)) return QL_ERR_INVALID_ARG;
    return QL_OK;
}

struct Plan {
    int bits = 4;         // code width: 4 (W4 g64) or 8 (W8 g64)
    int path = QL_PATH_GEMV;
    int split_k = 1;
    char why[64] = "forced";      // the dispatcher's reason, reported by qlinear_last_dispatch
    // skinny path: stream-K runs
    int ctas = 0, segmax = 0, nt = 0;
    int64_t units = 0;
    size_t workspace = 0;
    // fused path workspace carve-up (off_part: fp32 partials [split_k][M][N] when the K-steps are split)
    size_t off_xh = 0, off_rs = 0, off_sb = 0, off_part = 0;
    // skinny path workspace carve-up: partials, scaled f16 activations, row exponents, per-slice row maxima
    size_t off_xp = 0, off_re = 0;
};

// Split factor of the fused tensor-core path when the caller leaves it to the dispatcher.  Every K-step
// of a 256 x 192 tile costs about the same (0.56-0.66 us measured on a B200 across the text projection,
// the QKV and the MLP down projection), so a launch of `tiles` tiles cut into S slices takes about
// ceil(tiles * S / SMs) waves of ceil(G / S) K-steps.  Splitting also writes and reads back S fp32
// partials of y and adds the ordered-sum launch.  The S with the lowest estimate wins; a larger S must
// beat the best smaller one by 3%; a slice keeps at least 8 K-steps.  On the measured shapes (text projection M = 96..512,
// QKV M = 64..1024, MLP down M = 64..512) this picks the fastest forced split or one within 5% of it.
int fused_auto_split(int64_t M, int64_t N, int64_t G, int sm_count) {
    constexpr double kStepNs = 600.0;           // one K-step of one tile
    constexpr double kSplitFixedNs = 5000.0;    // the extra launch and the reduction's start
    constexpr double kBytesPerNs = 6000.0;      // HBM rate of the partials' write and read-back
    const int64_t tiles = ((M + fused::BT - 1) / fused::BT) * ((N + fused::BW - 1) / fused::BW);
    const int64_t smax = std::max<int64_t>(1, std::min<int64_t>(16, G / 8));
    int best_s = 1;
    double best = 0.0;
    for (int64_t sk = 1; sk <= smax; ++sk) {
        const double waves = static_cast<double>((tiles * sk + sm_count - 1) / sm_count);
        double t = waves * static_cast<double>((G + sk - 1) / sk) * kStepNs;
        if (sk > 1) t += kSplitFixedNs + 8.0 * static_cast<double>(sk) * M * N / kBytesPerNs;
        if (sk == 1 || t < 0.97 * best) {     // a larger split must win by more than the model's noise
            best = t;
            best_s = static_cast<int>(sk);
        }
    }
    return best_s;
}

// Per-shape choice of QL_PATH_AUTO: the weight-streaming tensor-core kernel up to 64 tokens (its MMA
// N of 16, 32 or 64 tokens covers them; measured on the text projection it takes 50-60 us for
// M = 1..64, where the fused path needs 97 us split 8 ways and 467 us unsplit), the fused kernel above,
// with the split of fused_auto_split.
ql_status make_plan(int64_t M, int64_t K, int64_t N, int path, int split_k, int sm_count, int bits, Plan* plan) {
    const int64_t G = K / kGroup;
    const bool automatic = path == QL_PATH_AUTO;
    if (automatic) {
        path = (M <= 64) ? QL_PATH_TC_SKINNY : QL_PATH_TC_FUSED;
        std::snprintf(plan->why, sizeof(plan->why), "%s", M <= 64 ? "auto:M<=64" : "auto:M>64");
    }
    plan->path = path;
    plan->bits = bits;
    if (path == QL_PATH_GEMV) {
        int s = split_k > 0 ? split_k : gemv_auto_split(K, N, sm_count);
        if (s > G || s > 65535) return QL_ERR_INVALID_ARG;
        plan->split_k = s;
        plan->workspace = s > 1 ? static_cast<size_t>(s) * M * N * sizeof(float) : 0;
        return QL_OK;
    }
    if (path == QL_PATH_TC_SKINNY) {
        // the dispatcher picks this path for M <= 64 (MMA N of 16, 32 or 64 tokens)
        if (M > 64 || split_k > 1) return QL_ERR_UNSUPPORTED;
        plan->nt = M <= 16 ? 16 : M <= 32 ? 32 : 64;
        const int64_t cg = bits == 4 ? skinny::Layout<16, 4>::CG : skinny::Layout<16, 8>::CG;
        const int64_t cpt = (G + cg - 1) / cg;
        plan->units = ((N + skinny::BW - 1) / skinny::BW) * cpt;
        plan->ctas = static_cast<int>(std::min<int64_t>(std::min(sm_count, skinny::kMaxCtas), plan->units));
        const int64_t run = (plan->units + plan->ctas - 1) / plan->ctas;
        plan->segmax = static_cast<int>((run + cpt - 1) / cpt + 1);
        plan->split_k = 1;
        plan->off_xp = round_up(static_cast<size_t>(plan->ctas) * plan->segmax * M * skinny::BW * sizeof(float), 256);
        plan->off_re = plan->off_xp + round_up(static_cast<size_t>(M) * K * 2, 256);
        plan->workspace = plan->off_re + round_up(static_cast<size_t>(plan->nt) * sizeof(int), 256);
        return QL_OK;
    }
    if (path == QL_PATH_TC_FUSED) {
        if (split_k > G || split_k > 1024) return QL_ERR_INVALID_ARG;
        plan->split_k = split_k > 0 ? split_k : fused_auto_split(M, N, G, sm_count);
        if (split_k == 0) {
            const int64_t tiles = ((M + fused::BT - 1) / fused::BT) * ((N + fused::BW - 1) / fused::BW);
            const int sk = plan->split_k;
            std::snprintf(plan->why, sizeof(plan->why), "%s,split:%lldx%lld", automatic ? "auto:M>64" : "forced",
                          static_cast<long long>((tiles * sk + sm_count - 1) / sm_count),
                          static_cast<long long>((G + sk - 1) / sk));
        }
        plan->off_xh = 0;
        plan->off_rs = round_up(static_cast<size_t>(M) * K * 2, 256);
        plan->off_sb = plan->off_rs + round_up(static_cast<size_t>(M) * 4, 256);
        plan->off_part = plan->off_sb + round_up(static_cast<size_t>(G) * N * 4, 256);
        plan->workspace = plan->off_part;
        if (plan->split_k > 1) plan->workspace += round_up(static_cast<size_t>(plan->split_k) * M * N * 4, 256);
        return QL_OK;
    }
    return QL_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ launches

ql_status run_gemv(const Plan& pl, const void* x, const uint32_t* codes, const void* scales, const void* biases,
                   void* y, bool bf16_out, int64_t M, int64_t K, int64_t N, void* ws, cudaStream_t st,
                   int sm_count) {
    const dim3 grid(static_cast<unsigned>(N / kGemvWarps), static_cast<unsigned>(pl.split_k));
    const bool partial = pl.split_k > 1;
    void* out = partial ? ws : y;
    auto xb = static_cast<const __nv_bfloat16*>(x);
    auto sc = static_cast<const __half*>(scales);
    auto bi = static_cast<const __half*>(biases);
    prof_begin(st);
    if (pl.bits == 8) {
        if (bf16_out)
            cc_stream8_kernel<true><<<grid, kGemvWarps * 32, 0, st>>>(xb, codes, sc, bi, out, (int)M, (int)K, (int)N, partial);
        else
            cc_stream8_kernel<false><<<grid, kGemvWarps * 32, 0, st>>>(xb, codes, sc, bi, out, (int)M, (int)K, (int)N, partial);
    } else {
        if (bf16_out)
            cc_stream_kernel<true><<<grid, kGemvWarps * 32, 0, st>>>(xb, codes, sc, bi, out, (int)M, (int)K, (int)N, partial);
        else
            cc_stream_kernel<false><<<grid, kGemvWarps * 32, 0, st>>>(xb, codes, sc, bi, out, (int)M, (int)K, (int)N, partial);
    }
    prof_end(st);
    if (partial) {
        const int64_t count = M * N;
        const int blocks = static_cast<int>(std::min<int64_t>((count / 4 + 255) / 256, 8 * sm_count));
        if (bf16_out)
            ordered_sum_kernel<true><<<blocks, 256, 0, st>>>(static_cast<const float*>(ws), y, count, pl.split_k);
        else
            ordered_sum_kernel<false><<<blocks, 256, 0, st>>>(static_cast<const float*>(ws), y, count, pl.split_k);
    }
    set_dispatch("path=gemv bits=%d warps=%d splitk=%d launches=%d why=%s", pl.bits, kGemvWarps, pl.split_k,
                 partial ? 2 : 1, pl.why);
    return launch_status();
}

// Launches with programmatic stream serialization: the kernel may start while the previous
// kernel on the stream is still running and waits for it (griddepcontrol.wait) where it must.
template <typename... KArgs, typename... Args>
ql_status launch_dependent(void (*kernel)(KArgs...), dim3 grid, int block, size_t smem, cudaStream_t st,
                           Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(static_cast<unsigned>(block));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

#ifdef QL_BOUNDS_CHECK
// Ring-depth variants of the 4-bit bf16 fused kernel (the checked build's qlinear_test_ring_depth):
// (activation stages, code stages, 4-bit codes, bf16 staging, staging blocks per warp).
using RingV1 = fused::Cfg<2, 1, 4, 2, 1>;
using RingV2 = fused::Cfg<3, 1, 4, 2, 2>;
using RingV3 = fused::Cfg<2, 2, 4, 2, 2>;
using RingV4 = fused::Cfg<4, 2, 4, 2, 1>;
using RingV5 = fused::Cfg<6, 1, 4, 2, 2>;
using RingV6 = fused::Cfg<3, 3, 4, 2, 2>;
static_assert(QL_TEST_RING_VARIANTS == 7, "one configuration per variant");
std::atomic<int> g_ring_variant{0};

template <class FC>
ql_status launch_ring(dim3 grid, cudaStream_t st, const CUtensorMap& mx, const CUtensorMap& mc, const CUtensorMap& mp,
                      const CUtensorMap& my, const fused::Params& p) {
    static_assert(FC::kS == fused::PickCfg<4, true>::type::kS, "the parameter boxes are sized for kS K-steps");
    return launch_dependent(fused::fused_gemm_kernel<true, FC>, grid, fused::kThreads, FC::kSmemBytes, st, mx, mc, mc,
                            mp, my, p);
}

ql_status launch_ring_variant(int v, dim3 grid, cudaStream_t st, const CUtensorMap& mx, const CUtensorMap& mc,
                              const CUtensorMap& mp, const CUtensorMap& my, const fused::Params& p) {
    switch (v) {
        case 1: return launch_ring<RingV1>(grid, st, mx, mc, mp, my, p);
        case 2: return launch_ring<RingV2>(grid, st, mx, mc, mp, my, p);
        case 3: return launch_ring<RingV3>(grid, st, mx, mc, mp, my, p);
        case 4: return launch_ring<RingV4>(grid, st, mx, mc, mp, my, p);
        case 5: return launch_ring<RingV5>(grid, st, mx, mc, mp, my, p);
        case 6: return launch_ring<RingV6>(grid, st, mx, mc, mp, my, p);
        default: return QL_ERR_INVALID_ARG;
    }
}

template <class FC>
cudaError_t ring_smem_attr() {
    return cudaFuncSetAttribute(fused::fused_gemm_kernel<true, FC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                FC::kSmemBytes);
}
#endif

// The activation conversion in front of the fused kernel, launched behind the parameter transpose
// under programmatic dependent launch: 128-thread CTAs for rows that fit their registers (K <= 5120),
// 256-thread CTAs for longer rows (the two shapes of convert_x_kernel).
ql_status launch_convert_x(int bits, const __nv_bfloat16* x, __half* xh, float* rs, int64_t M, int64_t K,
                           cudaStream_t st) {
    const dim3 rows(static_cast<unsigned>(M));
    const int k = static_cast<int>(K);
    if (K <= 128 * 5 * 8)
        return bits == 4 ? launch_dependent(convert_x_kernel<4, 128, 5>, rows, 128, 0, st, x, xh, rs, k)
                         : launch_dependent(convert_x_kernel<8, 128, 5>, rows, 128, 0, st, x, xh, rs, k);
    return bits == 4 ? launch_dependent(convert_x_kernel<4, 256, 4>, rows, 256, 0, st, x, xh, rs, k)
                     : launch_dependent(convert_x_kernel<8, 256, 4>, rows, 256, 0, st, x, xh, rs, k);
}

ql_status run_fused(const Plan& pl, const void* x, const uint32_t* codes, const void* scales, const void* biases,
                    void* y, bool bf16_out, int64_t M, int64_t K, int64_t N, void* ws, cudaStream_t st,
                    int sm_count) {
    const int64_t G = K / kGroup;
    auto* base = static_cast<uint8_t*>(ws);
    auto* xh = reinterpret_cast<__half*>(base + pl.off_xh);
    auto* rs = reinterpret_cast<float*>(base + pl.off_rs);
    auto* sb = reinterpret_cast<uint32_t*>(base + pl.off_sb);

    CUtensorMap mx, mc, mp;
    ql_status s;
    if ((s = encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xh, K, M, K * 2, fused::BK, fused::BT,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != QL_OK)
        return s;
    // one code stage per box: 128 bytes of each of 256 rows (4 K-steps of 4-bit codes, 2 of 8-bit codes),
    // 128-byte swizzle, which the dequantizers undo; the (scale, bias) pairs of the same K-steps
    const int bits = pl.bits;
    const int cfg_steps = bits == 4 ? fused::PickCfg<4, true>::type::kS : fused::PickCfg<8, true>::type::kS;
    if ((s = encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, codes, K * bits / 32, N, K * bits / 8,
                       fused::kCodeRowBytes / 4, fused::BW, CU_TENSOR_MAP_SWIZZLE_128B)) != QL_OK)
        return s;
    if ((s = encode_2d(&mp, CU_TENSOR_MAP_DATA_TYPE_UINT32, sb, N, G, N * 4, fused::BW, cfg_steps,
                       CU_TENSOR_MAP_SWIZZLE_NONE)) != QL_OK)
        return s;
    CUtensorMap my;
    const bool split = pl.split_k > 1;
    float* part = reinterpret_cast<float*>(base + pl.off_part);
    if (split) {
        // fp32 partials [split_k][M][N]: 32 x 32 blocks, clipped at M and N within every slice
        if ((s = encode_3d(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, part, N, M, pl.split_k, N * 4,
                           static_cast<uint64_t>(M) * N * 4, 32, 32)) != QL_OK)
            return s;
    } else if ((s = encode_2d(&my, bf16_out ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, y, N,
                              M, N * (bf16_out ? 2 : 4), 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE)) != QL_OK) {
        return s;
    }

    // The parameter transpose first (a plain launch: it follows the caller's earlier work), then the
    // conversion and the fused kernel under programmatic dependent launch: the conversion runs beside the
    // transpose, its last CTA waits for it, and the fused kernel waits for the conversion where it reads
    // the outputs of both.
    const dim3 tgrid(static_cast<unsigned>((G + 31) / 32), static_cast<unsigned>((N + kTransposeCols - 1) / kTransposeCols));
    transpose_params_kernel<<<tgrid, 256, 0, st>>>(static_cast<const __half*>(scales), static_cast<const __half*>(biases),
                                                   sb, static_cast<int>(N), static_cast<int>(G));
    if ((s = launch_status()) != QL_OK) return s;
    if ((s = launch_convert_x(bits, static_cast<const __nv_bfloat16*>(x), xh, rs, M, K, st)) != QL_OK) return s;
    fused::Params p;
    p.rowscale = rs;
    p.y = y;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.G = static_cast<int>(G);
    p.num_t = static_cast<int>((M + fused::BT - 1) / fused::BT);
    p.num_w = static_cast<int>((N + fused::BW - 1) / fused::BW);
    p.splits = pl.split_k;
    const int tiles = p.num_t * p.num_w;
    const int grid = static_cast<int>(std::min<int64_t>(static_cast<int64_t>(tiles) * pl.split_k, sm_count));
    prof_begin(st);
    const dim3 fgrid(static_cast<unsigned>(grid));
    using F4 = fused::PickCfg<4, false>::type;
    using F8 = fused::PickCfg<8, false>::type;
    if (split) {
        s = bits == 4 ? launch_dependent(fused::fused_gemm_kernel<false, F4, false, true>, fgrid, fused::kThreads,
                                         F4::kSmemBytes, st, mx, mc, mc, mp, my, p)
                      : launch_dependent(fused::fused_gemm_kernel<false, F8, false, true>, fgrid, fused::kThreads,
                                         F8::kSmemBytes, st, mx, mc, mc, mp, my, p);
        if (s != QL_OK) return s;
        prof_end(st);
        // ordered sum of the slices, rounded once (a plain launch: it reads what the kernel above wrote)
        const int64_t count = M * N;
        const int blocks = static_cast<int>(std::min<int64_t>((count / 4 + 255) / 256, 8 * sm_count));
        if (bf16_out)
            ordered_sum_kernel<true><<<blocks, 256, 0, st>>>(part, y, count, pl.split_k);
        else
            ordered_sum_kernel<false><<<blocks, 256, 0, st>>>(part, y, count, pl.split_k);
        const int nc = bits == 4 ? F4::kNC : F8::kNC;
        const int nx = bits == 4 ? F4::kNX : F8::kNX;
        set_dispatch("path=tc_fused bits=%d tile=%dw x %dt x %dk stages=x%d/c%dx%d/a%d ctas=%d splitk=%d launches=4 why=%s",
                     bits, fused::BW, fused::BT, fused::BK, nx, nc, cfg_steps, fused::NA, grid, pl.split_k, pl.why);
        return launch_status();
    }
    using B4 = fused::PickCfg<4, true>::type;
    using B8 = fused::PickCfg<8, true>::type;
#ifdef QL_BOUNDS_CHECK
    if (const int v = g_ring_variant.load(); v != 0 && bits == 4 && bf16_out) {
        if ((s = launch_ring_variant(v, fgrid, st, mx, mc, mp, my, p)) != QL_OK) return s;
        prof_end(st);
        set_dispatch("path=tc_fused bits=4 ring_variant=%d ctas=%d splitk=1 launches=3 why=%s", v, grid, pl.why);
        return launch_status();
    }
#endif
    if (bits == 4) {
        s = bf16_out ? launch_dependent(fused::fused_gemm_kernel<true, B4>, fgrid, fused::kThreads, B4::kSmemBytes, st,
                                        mx, mc, mc, mp, my, p)
                     : launch_dependent(fused::fused_gemm_kernel<false, F4>, fgrid, fused::kThreads, F4::kSmemBytes, st,
                                        mx, mc, mc, mp, my, p);
    } else {
        s = bf16_out ? launch_dependent(fused::fused_gemm_kernel<true, B8>, fgrid, fused::kThreads, B8::kSmemBytes, st,
                                        mx, mc, mc, mp, my, p)
                     : launch_dependent(fused::fused_gemm_kernel<false, F8>, fgrid, fused::kThreads, F8::kSmemBytes, st,
                                        mx, mc, mc, mp, my, p);
    }
    if (s != QL_OK) return s;
    prof_end(st);
    const int nc = bits == 4 ? (bf16_out ? B4::kNC : F4::kNC) : (bf16_out ? B8::kNC : F8::kNC);
    const int nx = bits == 4 ? (bf16_out ? B4::kNX : F4::kNX) : (bf16_out ? B8::kNX : F8::kNX);
    set_dispatch("path=tc_fused bits=%d tile=%dw x %dt x %dk stages=x%d/c%dx%d/a%d ctas=%d splitk=1 launches=3 why=%s",
                 bits, fused::BW, fused::BT, fused::BK, nx, nc, cfg_steps, fused::NA, grid, pl.why);
    (void)codes;
    return launch_status();
}

ql_status run_skinny(const Plan& pl, const void* x, const uint32_t* codes, const void* scales, const void* biases,
                     void* y, bool bf16_out, int64_t M, int64_t K, int64_t N, void* ws, cudaStream_t st,
                     int sm_count) {
    const int64_t G = K / kGroup;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    void* xp = wsb + pl.off_xp;
    int* rowexp = reinterpret_cast<int*>(wsb + pl.off_re);
    CUtensorMap mc, mx;
    ql_status s;
    const int bits = pl.bits;
    // code boxes: 128 bytes (32 words) of each of 128 rows, 128-byte swizzle, for either code width
    if ((s = encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, codes, K * bits / 32, N, K * bits / 8,
                       skinny::kBoxBytes / skinny::BW / 4, skinny::BW, CU_TENSOR_MAP_SWIZZLE_128B)) != QL_OK)
        return s;
    if ((s = encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xp, K, M, K * 2, skinny::BK, pl.nt,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != QL_OK)
        return s;
    // scale/bias boxes of 8 groups by TMA need a 16-byte row pitch (G % 8 == 0); every chunk then
    // lies inside one box
    const bool param_tma = (G % skinny::kParGroups) == 0;
    CUtensorMap ms = mc, mb = mc;
    if (param_tma) {
        if ((s = encode_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, scales, G, N, G * 2, skinny::kParGroups, skinny::BW,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != QL_OK)
            return s;
        if ((s = encode_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, biases, G, N, G * 2, skinny::kParGroups, skinny::BW,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != QL_OK)
            return s;
    }
    skinny::Params p;
    p.param_tma = param_tma ? 1 : 0;
    p.partial = reinterpret_cast<float*>(wsb);
    p.scales = static_cast<const __half*>(scales);
    p.biases = static_cast<const __half*>(biases);
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.G = static_cast<int>(G);
    p.num_w = static_cast<int>((N + skinny::BW - 1) / skinny::BW);
    const int cg = bits == 4 ? skinny::Layout<16, 4>::CG : skinny::Layout<16, 8>::CG;
    p.cpt = static_cast<int>((G + cg - 1) / cg);
    p.units = pl.units;
    p.segmax = pl.segmax;
    p.partial_elems = static_cast<int64_t>(pl.ctas) * pl.segmax * M * skinny::BW;
    // row exponents and scaled, reordered f16 activations (one cluster of CTAs per row)
    const dim3 pre_grid(static_cast<unsigned>(skinny::kPrepCluster), static_cast<unsigned>(M));
    if (bits == 4)
        skinny::skinny_prepass_kernel<4><<<pre_grid, skinny::kPrepThreads, 0, st>>>(
            static_cast<const uint4*>(x), static_cast<uint4*>(xp), rowexp, static_cast<int>(K));
    else
        skinny::skinny_prepass_kernel<8><<<pre_grid, skinny::kPrepThreads, 0, st>>>(
            static_cast<const uint4*>(x), static_cast<uint4*>(xp), rowexp, static_cast<int>(K));
    if ((s = launch_status()) != QL_OK) return s;
    prof_begin(st);
    const dim3 sgrid(static_cast<unsigned>(pl.ctas));
    if (bits == 4 && pl.nt == 16)
        s = launch_dependent(skinny::skinny_kernel<16, 4>, sgrid, skinny::kThreads, skinny::Layout<16, 4>::kSmemBytes, st,
                             mc, mx, ms, mb, p);
    else if (bits == 4 && pl.nt == 32)
        s = launch_dependent(skinny::skinny_kernel<32, 4>, sgrid, skinny::kThreads, skinny::Layout<32, 4>::kSmemBytes, st,
                             mc, mx, ms, mb, p);
    else if (bits == 4)
        s = launch_dependent(skinny::skinny_kernel<64, 4>, sgrid, skinny::kThreads, skinny::Layout<64, 4>::kSmemBytes, st,
                             mc, mx, ms, mb, p);
    else if (pl.nt == 16)
        s = launch_dependent(skinny::skinny_kernel<16, 8>, sgrid, skinny::kThreads, skinny::Layout<16, 8>::kSmemBytes, st,
                             mc, mx, ms, mb, p);
    else if (pl.nt == 32)
        s = launch_dependent(skinny::skinny_kernel<32, 8>, sgrid, skinny::kThreads, skinny::Layout<32, 8>::kSmemBytes, st,
                             mc, mx, ms, mb, p);
    else
        s = launch_dependent(skinny::skinny_kernel<64, 8>, sgrid, skinny::kThreads, skinny::Layout<64, 8>::kSmemBytes, st,
                             mc, mx, ms, mb, p);
    if (s != QL_OK) return s;
    prof_end(st);
    const float* part = p.partial;
    const int* rexp = rowexp;
    const dim3 red_grid(static_cast<unsigned>(p.num_w), static_cast<unsigned>((M + 1) / 2));
    if (bf16_out)
        s = launch_dependent(skinny::skinny_reduce_kernel<true>, red_grid, 256, 0, st, part, rexp, y, p.M, p.N, p.cpt,
                             p.units, pl.ctas, pl.segmax, p.partial_elems);
    else
        s = launch_dependent(skinny::skinny_reduce_kernel<false>, red_grid, 256, 0, st, part, rexp, y, p.M, p.N, p.cpt,
                             p.units, pl.ctas, pl.segmax, p.partial_elems);
    if (s != QL_OK) return s;
    (void)sm_count;
    set_dispatch("path=tc_skinny bits=%d nt=%d ctas=%d segmax=%d units=%lld launches=3 why=%s", bits, pl.nt, pl.ctas,
                 pl.segmax, static_cast<long long>(pl.units), pl.why);
    return launch_status();
}

// ------------------------------------------------------------------ SwiGLU pair (gate and up in one GEMM)

struct SwigluPlan {
    int num_w = 0;            // tiles of 128 intermediate columns
    int64_t ncols = 0;        // columns of the interleaved parameter array: 256 per tile
    size_t off_rs = 0, off_sb = 0, workspace = 0;
};

SwigluPlan swiglu_plan(int64_t M, int64_t K, int64_t I) {
    SwigluPlan pl;
    const int64_t G = K / kGroup;
    pl.num_w = static_cast<int>((I + fused::BWG - 1) / fused::BWG);
    pl.ncols = static_cast<int64_t>(pl.num_w) * fused::BW;
    pl.off_rs = round_up(static_cast<size_t>(M) * K * 2, 256);
    pl.off_sb = pl.off_rs + round_up(static_cast<size_t>(M) * 4, 256);
    pl.workspace = pl.off_sb + round_up(static_cast<size_t>(G) * pl.ncols * 4, 256);
    return pl;
}

ql_status run_swiglu(const SwigluPlan& pl, const void* x, const uint32_t* gc, const void* gs, const void* gb,
                     const uint32_t* uc, const void* us, const void* ub, void* h, bool bf16_out, int64_t M, int64_t K,
                     int64_t I, void* ws, cudaStream_t st, int sm_count) {
    const int64_t G = K / kGroup;
    auto* base = static_cast<uint8_t*>(ws);
    auto* xh = reinterpret_cast<__half*>(base);
    auto* rs = reinterpret_cast<float*>(base + pl.off_rs);
    auto* sb = reinterpret_cast<uint32_t*>(base + pl.off_sb);
    CUtensorMap mx, mcg, mcu, mp, my;
    ql_status s;
    if ((s = encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xh, K, M, K * 2, fused::BK, fused::BT,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != QL_OK)
        return s;
    // 128-row code boxes of one code stage (128 bytes per row, 128-byte swizzle): a tile's gate rows,
    // then the same rows of the up weight
    using FB = fused::PickCfg<4, true>::type;
    using FF = fused::PickCfg<4, false>::type;
    if ((s = encode_2d(&mcg, CU_TENSOR_MAP_DATA_TYPE_UINT32, gc, K / 8, I, K / 2, fused::kCodeRowBytes / 4, fused::BWG,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != QL_OK)
        return s;
    if ((s = encode_2d(&mcu, CU_TENSOR_MAP_DATA_TYPE_UINT32, uc, K / 8, I, K / 2, fused::kCodeRowBytes / 4, fused::BWG,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != QL_OK)
        return s;
    if ((s = encode_2d(&mp, CU_TENSOR_MAP_DATA_TYPE_UINT32, sb, pl.ncols, G, pl.ncols * 4, fused::BW, FB::kS,
                       CU_TENSOR_MAP_SWIZZLE_NONE)) != QL_OK)
        return s;
    if ((s = encode_2d(&my, bf16_out ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, h, I, M,
                       I * (bf16_out ? 2 : 4), 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE)) != QL_OK)
        return s;
    // pair transpose, then conversion and fused kernel under programmatic dependent launch (as run_fused)
    const dim3 tgrid(static_cast<unsigned>((G + 31) / 32), static_cast<unsigned>(pl.ncols / kTransposeCols));
    transpose_params_pair_kernel<<<tgrid, 256, 0, st>>>(static_cast<const __half*>(gs), static_cast<const __half*>(gb),
                                                        static_cast<const __half*>(us), static_cast<const __half*>(ub),
                                                        sb, static_cast<int>(I), static_cast<int>(G),
                                                        static_cast<int>(pl.ncols));
    if ((s = launch_status()) != QL_OK) return s;
    if ((s = launch_convert_x(4, static_cast<const __nv_bfloat16*>(x), xh, rs, M, K, st)) != QL_OK) return s;
    fused::Params p;
    p.rowscale = rs;
    p.y = h;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(I);
    p.G = static_cast<int>(G);
    p.num_t = static_cast<int>((M + fused::BT - 1) / fused::BT);
    p.num_w = pl.num_w;
    p.splits = 1;
    const int tiles = p.num_t * p.num_w;
    const int grid = std::min(tiles, sm_count);
    const dim3 fgrid(static_cast<unsigned>(grid));
    prof_begin(st);
    s = bf16_out ? launch_dependent(fused::fused_gemm_kernel<true, FB, true>, fgrid, fused::kThreads, FB::kSmemBytes,
                                    st, mx, mcg, mcu, mp, my, p)
                 : launch_dependent(fused::fused_gemm_kernel<false, FF, true>, fgrid, fused::kThreads, FF::kSmemBytes,
                                    st, mx, mcg, mcu, mp, my, p);
    if (s != QL_OK) return s;
    prof_end(st);
    set_dispatch("path=tc_fused_swiglu bits=4 tile=%dg+%du x %dt x %dk stages=x%d/c%dx%d/a%d ctas=%d launches=3",
                 fused::BWG, fused::BWG, fused::BT, fused::BK, bf16_out ? FB::kNX : FF::kNX,
                 bf16_out ? FB::kNC : FF::kNC, FB::kS, fused::NA, grid);
    return launch_status();
}

ql_status swiglu_impl(const void* x, const uint32_t* gc, const void* gs, const void* gb, const uint32_t* uc,
                      const void* us, const void* ub, void* h, ql_dtype out_dtype, int64_t M, int64_t K, int64_t I,
                      int32_t group, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    ql_status s = check_shape(M, K, I, group);
    if (s != QL_OK) return s;
    if (!x || !gc || !gs || !gb || !uc || !us || !ub || !h) return QL_ERR_INVALID_ARG;
    if (out_dtype != QL_BF16 && out_dtype != QL_F32) return QL_ERR_INVALID_ARG;
    const void* in[7] = {x, gc, gs, gb, uc, us, ub};
    for (const void* q : in)
        if (!aligned16(q)) return QL_ERR_ALIGNMENT;
    if (!aligned16(h)) return QL_ERR_ALIGNMENT;
    const int64_t G = K / kGroup;
    const size_t xb = static_cast<size_t>(M) * K * 2, cb = code_bytes(K, I, 4), pb = static_cast<size_t>(I) * G * 2,
                 hb = static_cast<size_t>(M) * I * (out_dtype == QL_BF16 ? 2 : 4);
    const size_t in_bytes[7] = {xb, cb, pb, pb, cb, pb, pb};
    for (int i = 0; i < 7; ++i)
        if (overlap(h, hb, in[i], in_bytes[i])) return QL_ERR_INVALID_ARG;
    const SwigluPlan pl = swiglu_plan(M, K, I);
    if (!workspace || workspace_bytes < pl.workspace) return QL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QL_ERR_ALIGNMENT;
    if (overlap(workspace, pl.workspace, h, hb)) return QL_ERR_INVALID_ARG;
    for (int i = 0; i < 7; ++i)
        if (overlap(workspace, pl.workspace, in[i], in_bytes[i])) return QL_ERR_INVALID_ARG;
    DeviceInfo* dev = nullptr;
    if ((s = device_info(&dev)) != QL_OK) return s;
    return run_swiglu(pl, x, gc, gs, gb, uc, us, ub, h, out_dtype == QL_BF16, M, K, I, workspace, stream,
                      dev->sm_count);
}

ql_status forward_impl(const void* x, const uint32_t* codes, const void* scales, const void* biases, void* y,
                       ql_dtype out_dtype, int64_t M, int64_t K, int64_t N, int32_t group, int32_t path,
                       int32_t split_k, void* workspace, size_t workspace_bytes, cudaStream_t stream, int bits) {
    ql_status s = check_shape(M, K, N, group);
    if (s != QL_OK) return s;
    if (!x || !codes || !scales || !biases || !y) return QL_ERR_INVALID_ARG;
    if (out_dtype != QL_BF16 && out_dtype != QL_F32) return QL_ERR_INVALID_ARG;
    if (path < QL_PATH_AUTO || path > QL_PATH_TC_FUSED || split_k < 0) return QL_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases) || !aligned16(y))
        return QL_ERR_ALIGNMENT;
    const int64_t G = K / kGroup;
    const size_t xb = static_cast<size_t>(M) * K * 2, cb = code_bytes(K, N, bits),
                 pb = static_cast<size_t>(N) * G * 2,
                 yb = static_cast<size_t>(M) * N * (out_dtype == QL_BF16 ? 2 : 4);
    if (overlap(y, yb, x, xb) || overlap(y, yb, codes, cb) || overlap(y, yb, scales, pb) || overlap(y, yb, biases, pb))
        return QL_ERR_INVALID_ARG;
    DeviceInfo* dev = nullptr;
    if ((s = device_info(&dev)) != QL_OK) return s;
    Plan pl;
    if ((s = make_plan(M, K, N, path, split_k, dev->sm_count, bits, &pl)) != QL_OK) return s;
    if (pl.workspace > 0) {
        if (!workspace || workspace_bytes < pl.workspace) return QL_ERR_WORKSPACE;
        if (!aligned16(workspace)) return QL_ERR_ALIGNMENT;
        if (overlap(workspace, pl.workspace, x, xb) || overlap(workspace, pl.workspace, y, yb) ||
            overlap(workspace, pl.workspace, codes, cb) || overlap(workspace, pl.workspace, scales, pb) ||
            overlap(workspace, pl.workspace, biases, pb))
            return QL_ERR_INVALID_ARG;
    }
    const bool bf16 = out_dtype == QL_BF16;
    if (pl.path == QL_PATH_GEMV)
        return run_gemv(pl, x, codes, scales, biases, y, bf16, M, K, N, workspace, stream, dev->sm_count);
    if (pl.path == QL_PATH_TC_SKINNY)
        return run_skinny(pl, x, codes, scales, biases, y, bf16, M, K, N, workspace, stream, dev->sm_count);
    return run_fused(pl, x, codes, scales, biases, y, bf16, M, K, N, workspace, stream, dev->sm_count);
}

size_t workspace_impl(int64_t M, int64_t K, int64_t N, int32_t group, int32_t path, int32_t split_k, int bits) {
    if (check_shape(M, K, N, group) != QL_OK) return static_cast<size_t>(-1);
    DeviceInfo* dev = nullptr;
    int sms = 148;
    if (device_info(&dev) == QL_OK) sms = dev->sm_count;
    Plan pl;
    if (make_plan(M, K, N, path, split_k, sms, bits, &pl) != QL_OK) return static_cast<size_t>(-1);
    return pl.workspace;
}

ql_status dequant_impl(const uint32_t* codes, const void* scales, const void* biases, int64_t K, int64_t N,
                       int32_t group, void* out, ql_dtype out_dtype, cudaStream_t stream, int bits) {
    ql_status s = check_shape(1, K, N, group);
    if (s != QL_OK) return s;
    if (!codes || !scales || !biases || !out) return QL_ERR_INVALID_ARG;
    if (out_dtype != QL_BF16 && out_dtype != QL_F32) return QL_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(biases) || !aligned16(out)) return QL_ERR_ALIGNMENT;
    const int64_t G = K / kGroup;
    const size_t ob = static_cast<size_t>(N) * K * (out_dtype == QL_BF16 ? 2 : 4);
    if (overlap(out, ob, codes, code_bytes(K, N, bits)) || overlap(out, ob, scales, static_cast<size_t>(N) * G * 2) ||
        overlap(out, ob, biases, static_cast<size_t>(N) * G * 2))
        return QL_ERR_INVALID_ARG;
    DeviceInfo* dev = nullptr;
    if ((s = device_info(&dev)) != QL_OK) return s;
    const int64_t words = N * K * bits / 32;
    const int blocks = static_cast<int>(std::min<int64_t>((words + 255) / 256, 16 * dev->sm_count));
    auto sc = static_cast<const __half*>(scales);
    auto bi = static_cast<const __half*>(biases);
    if (bits == 8) {
        if (out_dtype == QL_BF16)
            dequant8_kernel<true><<<blocks, 256, 0, stream>>>(codes, sc, bi, out, words);
        else
            dequant8_kernel<false><<<blocks, 256, 0, stream>>>(codes, sc, bi, out, words);
    } else {
        if (out_dtype == QL_BF16)
            dequant_kernel<true><<<blocks, 256, 0, stream>>>(codes, sc, bi, out, words);
        else
            dequant_kernel<false><<<blocks, 256, 0, stream>>>(codes, sc, bi, out, words);
    }
    return launch_status();
}

ql_status pack_impl(const float* w, const float* imatrix, int64_t K, int64_t N, int32_t group, uint32_t* codes,
                    void* scales, void* biases, cudaStream_t stream, int bits) {
    ql_status s = check_shape(1, K, N, group);
    if (s != QL_OK) return s;
    if (!w || !codes || !scales || !biases) return QL_ERR_INVALID_ARG;
    if (imatrix != nullptr && bits != 4) return QL_ERR_UNSUPPORTED;   // the weighted fit is built for 4-bit codes
    if (N > 65535ll * kFitThreads || K / kGroup > 2147483647ll) return QL_ERR_UNSUPPORTED;   // fit grid limits
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases)) return QL_ERR_ALIGNMENT;
    const int64_t G = K / kGroup;
    const size_t wb = static_cast<size_t>(N) * K * 4, cb = code_bytes(K, N, bits),
                 pb = static_cast<size_t>(N) * G * 2;
    if (overlap(w, wb, codes, cb) || overlap(w, wb, scales, pb) || overlap(w, wb, biases, pb) ||
        overlap(codes, cb, scales, pb) || overlap(codes, cb, biases, pb) || overlap(scales, pb, biases, pb))
        return QL_ERR_INVALID_ARG;
    if (imatrix != nullptr) {
        const size_t ib = static_cast<size_t>(K) * 4;
        if (overlap(imatrix, ib, codes, cb) || overlap(imatrix, ib, scales, pb) || overlap(imatrix, ib, biases, pb))
            return QL_ERR_INVALID_ARG;
        const dim3 grid(static_cast<unsigned>(K / kGroup), static_cast<unsigned>((N + kFitThreads - 1) / kFitThreads));
        pack_fit_kernel<<<grid, kFitThreads, 0, stream>>>(w, imatrix, codes, static_cast<__half*>(scales),
                                                          static_cast<__half*>(biases), static_cast<int>(K),
                                                          static_cast<int>(N));
        return launch_status();
    }
    DeviceInfo* dev = nullptr;
    if ((s = device_info(&dev)) != QL_OK) return s;
    const int64_t groups = N * G;
    const int blocks = static_cast<int>(std::min<int64_t>((groups + 7) / 8, 32 * dev->sm_count));
    if (bits == 8)
        pack8_rtn_kernel<<<blocks, 256, 0, stream>>>(w, codes, static_cast<__half*>(scales),
                                                     static_cast<__half*>(biases), groups);
    else
        pack_rtn_kernel<<<blocks, 256, 0, stream>>>(w, codes, static_cast<__half*>(scales),
                                                    static_cast<__half*>(biases), groups);
    return launch_status();
}

}  // namespace
}  // namespace ql

using namespace ql;

extern "C" {

size_t qlinear_workspace_size(int64_t M, int64_t K, int64_t N, int32_t group) {
    return workspace_impl(M, K, N, group, QL_PATH_AUTO, 0, 4);
}

size_t qlinear_workspace_size_config(int64_t M, int64_t K, int64_t N, int32_t group, int32_t path, int32_t split_k) {
    return workspace_impl(M, K, N, group, path, split_k, 4);
}

ql_status qlinear_forward(const void* x, const uint32_t* codes, const void* scales, const void* biases, void* y,
                          int64_t M, int64_t K, int64_t N, int32_t group, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
    return forward_impl(x, codes, scales, biases, y, QL_BF16, M, K, N, group, QL_PATH_AUTO, 0, workspace,
                        workspace_bytes, stream, 4);
}

ql_status qlinear_forward_config(const void* x, const uint32_t* codes, const void* scales, const void* biases,
                                 void* y, ql_dtype out_dtype, int64_t M, int64_t K, int64_t N, int32_t group,
                                 int32_t path, int32_t split_k, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
    return forward_impl(x, codes, scales, biases, y, out_dtype, M, K, N, group, path, split_k, workspace,
                        workspace_bytes, stream, 4);
}

ql_status qlinear_dequant(const uint32_t* codes, const void* scales, const void* biases, int64_t K, int64_t N,
                          int32_t group, void* out, ql_dtype out_dtype, cudaStream_t stream) {
    return dequant_impl(codes, scales, biases, K, N, group, out, out_dtype, stream, 4);
}

ql_status qlinear_pack(const float* w, const float* imatrix, int64_t K, int64_t N, int32_t group, uint32_t* codes,
                       void* scales, void* biases, cudaStream_t stream) {
    return pack_impl(w, imatrix, K, N, group, codes, scales, biases, stream, 4);
}

ql_status qlinear_selftest_bounded_wait(cudaStream_t stream) {
    wait_selftest_kernel<<<1, 64, 0, stream>>>();
    return launch_status();
}

ql_status qlinear_test_stall(int32_t kernel_mask, uint64_t wait_limit_ns) {
#ifdef QL_BOUNDS_CHECK
    if (kernel_mask < 0 || kernel_mask > (kStallFused | kStallSkinny) || wait_limit_ns == 0) return QL_ERR_INVALID_ARG;
    const unsigned long long limit = wait_limit_ns;
    if (cudaMemcpyToSymbol(g_stall_mask, &kernel_mask, sizeof(kernel_mask)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_wait_limit_ns, &limit, sizeof(limit)) != cudaSuccess)
        return QL_ERR_CUDA;
    return QL_OK;
#else
    (void)kernel_mask;
    (void)wait_limit_ns;
    return QL_ERR_UNSUPPORTED;
#endif
}

ql_status qlinear_test_delay(int32_t role_mask, uint64_t max_ns) {
#ifdef QL_BOUNDS_CHECK
    constexpr int kAll = kDelayActivations | kDelayCodes | kDelayDequant | kDelayMma | kDelayEpilogue;
    if (role_mask < 0 || (role_mask & ~kAll) != 0 || max_ns > 1000000) return QL_ERR_INVALID_ARG;
    const unsigned long long ns = max_ns;
    if (cudaMemcpyToSymbol(g_delay_mask, &role_mask, sizeof(role_mask)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_delay_ns, &ns, sizeof(ns)) != cudaSuccess)
        return QL_ERR_CUDA;
    return QL_OK;
#else
    (void)role_mask;
    (void)max_ns;
    return QL_ERR_UNSUPPORTED;
#endif
}

ql_status qlinear_test_ring_depth(int32_t variant) {
#ifdef QL_BOUNDS_CHECK
    if (variant < 0 || variant >= QL_TEST_RING_VARIANTS) return QL_ERR_INVALID_ARG;
    if (ring_smem_attr<RingV1>() != cudaSuccess || ring_smem_attr<RingV2>() != cudaSuccess ||
        ring_smem_attr<RingV3>() != cudaSuccess || ring_smem_attr<RingV4>() != cudaSuccess ||
        ring_smem_attr<RingV5>() != cudaSuccess || ring_smem_attr<RingV6>() != cudaSuccess)
        return QL_ERR_CUDA;
    g_ring_variant.store(variant);
    return QL_OK;
#else
    (void)variant;
    return QL_ERR_UNSUPPORTED;
#endif
}

ql_status qlinear_reduce_partials(const float* partials, int32_t S, int64_t count, void* y, ql_dtype out_dtype,
                                  cudaStream_t stream) {
    if (!partials || !y || S < 1 || count < 4 || count % 4 != 0) return QL_ERR_INVALID_ARG;
    if (out_dtype != QL_BF16 && out_dtype != QL_F32) return QL_ERR_INVALID_ARG;
    if (!aligned16(partials) || !aligned16(y)) return QL_ERR_ALIGNMENT;
    const size_t yb = static_cast<size_t>(count) * (out_dtype == QL_BF16 ? 2 : 4);
    if (overlap(y, yb, partials, static_cast<size_t>(S) * count * 4)) return QL_ERR_INVALID_ARG;
    DeviceInfo* dev = nullptr;
    ql_status s;
    if ((s = device_info(&dev)) != QL_OK) return s;
    const int blocks = static_cast<int>(std::min<int64_t>((count / 4 + 255) / 256, 8 * dev->sm_count));
    if (out_dtype == QL_BF16)
        ordered_sum_kernel<true><<<blocks, 256, 0, stream>>>(partials, y, count, S);
    else
        ordered_sum_kernel<false><<<blocks, 256, 0, stream>>>(partials, y, count, S);
    return launch_status();
}

size_t qlinear_swiglu_workspace_size(int64_t M, int64_t K, int64_t I, int32_t group) {
    if (check_shape(M, K, I, group) != QL_OK) return static_cast<size_t>(-1);
    return swiglu_plan(M, K, I).workspace;
}

ql_status qlinear_swiglu_forward(const void* x, const uint32_t* gate_codes, const void* gate_scales,
                                 const void* gate_biases, const uint32_t* up_codes, const void* up_scales,
                                 const void* up_biases, void* h, ql_dtype out_dtype, int64_t M, int64_t K, int64_t I,
                                 int32_t group, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return swiglu_impl(x, gate_codes, gate_scales, gate_biases, up_codes, up_scales, up_biases, h, out_dtype, M, K, I,
                       group, workspace, workspace_bytes, stream);
}

size_t qlinear8_workspace_size(int64_t M, int64_t K, int64_t N, int32_t group) {
    return workspace_impl(M, K, N, group, QL_PATH_AUTO, 0, 8);
}

size_t qlinear8_workspace_size_config(int64_t M, int64_t K, int64_t N, int32_t group, int32_t path, int32_t split_k) {
    return workspace_impl(M, K, N, group, path, split_k, 8);
}

ql_status qlinear8_forward(const void* x, const uint32_t* codes, const void* scales, const void* biases, void* y,
                           int64_t M, int64_t K, int64_t N, int32_t group, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    return forward_impl(x, codes, scales, biases, y, QL_BF16, M, K, N, group, QL_PATH_AUTO, 0, workspace,
                        workspace_bytes, stream, 8);
}

ql_status qlinear8_forward_config(const void* x, const uint32_t* codes, const void* scales, const void* biases,
                                  void* y, ql_dtype out_dtype, int64_t M, int64_t K, int64_t N, int32_t group,
                                  int32_t path, int32_t split_k, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream) {
    return forward_impl(x, codes, scales, biases, y, out_dtype, M, K, N, group, path, split_k, workspace,
                        workspace_bytes, stream, 8);
}

ql_status qlinear8_dequant(const uint32_t* codes, const void* scales, const void* biases, int64_t K, int64_t N,
                           int32_t group, void* out, ql_dtype out_dtype, cudaStream_t stream) {
    return dequant_impl(codes, scales, biases, K, N, group, out, out_dtype, stream, 8);
}

ql_status qlinear8_pack(const float* w, const float* imatrix, int64_t K, int64_t N, int32_t group, uint32_t* codes,
                        void* scales, void* biases, cudaStream_t stream) {
    return pack_impl(w, imatrix, K, N, group, codes, scales, biases, stream, 8);
}

ql_status qlinear_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return QL_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return QL_ERR_CUDA;
    const unsigned int zero = 0;
    if (v != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return QL_ERR_CUDA;
    return static_cast<ql_status>(v);
}

ql_status qlinear_last_dispatch(char* buf, size_t len) {
    if (!buf || len == 0) return QL_ERR_INVALID_ARG;
    std::strncpy(buf, t_last_dispatch, len - 1);
    buf[len - 1] = '\0';
    return QL_OK;
}

ql_status qlinear_set_profile_events(cudaEvent_t start, cudaEvent_t stop) {
    if ((start == nullptr) != (stop == nullptr)) return QL_ERR_INVALID_ARG;
    t_prof_start = start;
    t_prof_stop = stop;
    return QL_OK;
}

const char* qlinear_status_string(ql_status status) {
    switch (status) {
        case QL_OK: return "QL_OK";
        case QL_ERR_INVALID_ARG: return "QL_ERR_INVALID_ARG";
        case QL_ERR_ALIGNMENT: return "QL_ERR_ALIGNMENT";
        case QL_ERR_UNSUPPORTED: return "QL_ERR_UNSUPPORTED";
        case QL_ERR_WORKSPACE: return "QL_ERR_WORKSPACE";
        case QL_ERR_CUDA: return "QL_ERR_CUDA";
        case QL_ERR_DEVICE_TIMEOUT: return "QL_ERR_DEVICE_TIMEOUT";
        case QL_ERR_BOUNDS: return "QL_ERR_BOUNDS";
    }
    return "QL_ERR_UNKNOWN";
}

int32_t qlinear_version(void) { return kVersion; }

}  // extern "C"
