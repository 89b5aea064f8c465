// Shared device helpers of the qlinear library: status word, bounded waits,
// conversions.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/qlinear.h"

namespace ql {

constexpr int kGroup = 64;

// First error recorded by any kernel since the host last read it (0 = none).
// One per translation unit and device; qlinear_get_device_status() reads the
// one of ql_api.cu, whose kernels are the ones that record errors.
static __device__ unsigned int g_device_status;

__device__ __forceinline__ void record_status(unsigned int code) {
    atomicCAS(&g_device_status, 0u, code);
}

// Index checks of the bounds-checked build (compiled with QL_BOUNDS_CHECK, the stand-in for a memory
// checker): an index outside [0, n) records QL_ERR_BOUNDS and the access is skipped.  In the normal
// build every check is the constant true.
#ifdef QL_BOUNDS_CHECK
__device__ __forceinline__ bool in_bounds(int64_t i, int64_t n) {
    if (i >= 0 && i < n) return true;
    record_status(QL_ERR_BOUNDS);
    return false;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(int64_t, int64_t) { return true; }
#endif

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Every wait on another thread, warp or async unit gives up after this long,
// records QL_ERR_DEVICE_TIMEOUT and lets the kernel unwind.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;   // 1 s

// Kernels whose code producer the checked build can hold back (qlinear_test_stall).
constexpr int kStallFused = 1, kStallSkinny = 2;

#ifdef QL_BOUNDS_CHECK
// Test hooks of the checked build (the index-checked variant): the host can shorten the wait limit and
// hold back the code producer of the kernels in a mask, so that a real pipeline's waits expire with no
// copy or MMA in flight and its unwinding can be tested.  The shipped build has neither: its limit is
// the constant above and nothing is held back.
static __device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;
static __device__ int g_stall_mask;
__device__ __forceinline__ uint64_t wait_limit_ns() { return g_wait_limit_ns; }
__device__ __forceinline__ bool stalled(int kernel_bit) { return (g_stall_mask & kernel_bit) != 0; }
#else
__device__ __forceinline__ constexpr uint64_t wait_limit_ns() { return kWaitLimitNs; }
__device__ __forceinline__ constexpr bool stalled(int) { return false; }
#endif

// Roles of the tensor-core kernels that the checked build can hold back at their start (qlinear_test_delay):
// the activation producer, the code producer, the dequantizers (builders), the MMA issuers and the
// epilogue (drain) warps.
constexpr int kDelayActivations = 1, kDelayCodes = 2, kDelayDequant = 4, kDelayMma = 8, kDelayEpilogue = 16;

#ifdef QL_BOUNDS_CHECK
// Test hook of the checked build: a role in the mask spins at its start for a CTA- and warp-dependent
// part (0/7 .. 7/7) of g_delay_ns, bounded by the time read, so that every hand-off between roles meets
// other orders of arrival; a race between roles then shows up as differing output bytes.
static __device__ int g_delay_mask;
static __device__ unsigned long long g_delay_ns;
__device__ __forceinline__ void test_delay(int role_bit) {
    if ((g_delay_mask & role_bit) == 0) return;
    const uint64_t d = g_delay_ns * ((blockIdx.x * 7u + (threadIdx.x >> 5) * 3u) % 8u) / 7u;
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < d) {
    }
}
#else
__device__ __forceinline__ void test_delay(int) {}
#endif

__device__ __forceinline__ uint32_t bits_of(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 half2_of(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace ql
