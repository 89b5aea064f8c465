// qlinear_forward_noalloc: the small-M weight-streaming forward for callers
// that cannot allocate device memory.
//
// Who needs it: code that may not call cudaMalloc (or any allocator) at the
// point where it runs the layer -- a plugin invoked inside another engine's
// fixed memory pool, a driver loop that is forbidden to allocate once serving
// has started, or a runtime that hands the layer only its inputs and outputs
// and no workspace.  For them this entry point takes its split-K scratch from
// a fixed array compiled into the library instead of from a caller workspace.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds QL_NOALLOC_SCRATCH_BYTES of it until the process exits.  In
// host code its name is only a host-side stand-in; the device address is
// obtained with cudaGetSymbolAddress once per device (with that device
// current) by the first call made on that device, which is why that first
// call should happen before any stream capture.  All calls share the array:
// calls that overlap on the GPU (different streams, or several host threads)
// race on it and must be serialized by the caller.  Nothing in it needs to
// start at zero -- each call writes every partial it later reads.
//
// The cached address belongs to the device's context as it was at the first
// call: after cudaDeviceReset on that device the cached address is stale, so
// this entry point must not be used across a device reset.
//
// Size bound: the split factor keeps S * N / 8 below 8 * SMs (it stops
// doubling once the grid has four waves of 8-row CTAs), so the partials of a
// call need S * M * N * 4 < 256 * SMs * M bytes: 2.4 MB at M = 64 on the 148
// SMs of a B200.  Parts with more than 256 SMs could exceed the array; such a
// shape is refused with QL_ERR_WORKSPACE before anything is launched.
#include <algorithm>
#include <mutex>

#include "ql_common.cuh"
#include "ql_gemv.cuh"

namespace {

constexpr size_t kScratchBytes = QL_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
static_assert(kScratchBytes >= size_t(256) * 148 * QL_NOALLOC_MAX_M,
              "the scratch array holds the largest partials of a B200 (148 SMs) at the maximum M");

static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

float* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (set up once per device).
ql_status scratch_address(float** out, int* sm_count) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QL_ERR_CUDA;
    if (cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QL_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QL_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_ptr[dev];
    return QL_OK;
}

template <bool kBf16Out>
__global__ void __launch_bounds__(ql::kGemvWarps * 32) noalloc_stream_kernel(
    const __nv_bfloat16* __restrict__ x, const uint32_t* __restrict__ codes, const __half* __restrict__ scales,
    const __half* __restrict__ biases, void* __restrict__ out, int M, int K, int N, bool partial_out) {
    ql::gemv_body<kBf16Out>(x, codes, scales, biases, out, M, K, N, partial_out);
}

template <bool kBf16Out>
__global__ void __launch_bounds__(256) noalloc_reduce_kernel(const float* __restrict__ partial, void* __restrict__ y,
                                                             int64_t count, int S) {
    ql::ordered_sum_body<kBf16Out>(partial, y, count, S);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t u = reinterpret_cast<uintptr_t>(a), v = reinterpret_cast<uintptr_t>(b);
    return na > 0 && nb > 0 && u < v + nb && v < u + na;
}

}  // namespace

extern "C" {

QL_API ql_status qlinear_forward_noalloc(const void* x, const uint32_t* codes, const void* scales, const void* biases,
                                         void* y, int64_t M, int64_t K, int64_t N, int32_t group, cudaStream_t stream) {
    if (group != ql::kGroup) return QL_ERR_UNSUPPORTED;
    if (M < 1 || K < ql::kGroup || N < 8 || K % ql::kGroup != 0 || N % 8 != 0 || K > (1ll << 30) || N > (1ll << 30))
        return QL_ERR_INVALID_ARG;
    if (M > QL_NOALLOC_MAX_M) return QL_ERR_UNSUPPORTED;
    if (!x || !codes || !scales || !biases || !y) return QL_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases) || !aligned16(y))
        return QL_ERR_ALIGNMENT;
    const int64_t G = K / ql::kGroup;
    const size_t xb = static_cast<size_t>(M) * K * 2, cb = static_cast<size_t>(N) * K / 2,
                 pb = static_cast<size_t>(N) * G * 2, yb = static_cast<size_t>(M) * N * 2;
    if (overlap(y, yb, x, xb) || overlap(y, yb, codes, cb) || overlap(y, yb, scales, pb) || overlap(y, yb, biases, pb))
        return QL_ERR_INVALID_ARG;

    // An error left pending by some earlier launch is not this call's: report it without launching
    // (and without clearing it), so that the error read after the launches below is this call's own.
    if (cudaPeekAtLastError() != cudaSuccess) return QL_ERR_CUDA;

    float* scratch = nullptr;
    int sms = 0;
    ql_status s = scratch_address(&scratch, &sms);
    if (s != QL_OK) return s;
    const int S = ql::gemv_auto_split(K, N, sms);
    const size_t need = S > 1 ? static_cast<size_t>(S) * M * N * sizeof(float) : 0;
    if (need > kScratchBytes) return QL_ERR_WORKSPACE;

    auto xp = static_cast<const __nv_bfloat16*>(x);
    auto sp = static_cast<const __half*>(scales);
    auto bp = static_cast<const __half*>(biases);
    const dim3 grid(static_cast<unsigned>(N / ql::kGemvWarps), static_cast<unsigned>(S));
    noalloc_stream_kernel<true><<<grid, ql::kGemvWarps * 32, 0, stream>>>(xp, codes, sp, bp, S > 1 ? scratch : y,
                                                                        (int)M, (int)K, (int)N, S > 1);
    if (S > 1) {
        const int64_t count = M * N;
        const int blocks = static_cast<int>(std::min<int64_t>((count / 4 + 255) / 256, 8 * sms));
        noalloc_reduce_kernel<true><<<blocks, 256, 0, stream>>>(scratch, y, count, S);
    }
    return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

}  // extern "C"
