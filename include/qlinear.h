/*
 * qlinear.h -- C ABI of the group-wise affine W4 g64 quantized linear layer (sm_100a),
 * with its W8 g64 variant (qlinear8_*, at the end).
 *
 * The packed format (aimarketly "Ideogram-4-IQ4_M", intro: one f16 scale and one
 * f16 bias per 64 weights on top of 4-bit codes, 4.5 bits per weight;
 * huggingface "SceneWorks/ideogram-4-mlx", Versions: group-wise affine, group
 * size 64) and its uniform affine grid w = scale * q + bias (aimarketly
 * "Ideogram-4-IQ4_M", "What IQ4 means here").
 *
 * Layout of every tensor (all row-major, dense, no padding):
 *   x       bf16     [M][K]      activations
 *   codes   uint32   [N][K/8]    code (n, k) = (codes[n][k/8] >> 4*(k%8)) & 0xF, low nibble first
 *   scales  f16      [N][K/64]   group scale  s(n, k/64)
 *   biases  f16      [N][K/64]   group bias   b(n, k/64)
 *   y       bf16     [M][N]      y[m][n] = sum_k x[m][k] * (s * q(n, k) + b)
 * W is logically [N][K] (a PyTorch Linear weight): y = x . W^T.
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller owns every buffer.  Tensor arguments are DEVICE
 *     pointers on the current CUDA device.  The library allocates no device
 *     memory; scratch comes from the caller's workspace.
 *   - Asynchrony: work is enqueued on `stream` (0 = legacy default stream).
 *     QL_OK means "validated and launched"; launch failures return QL_ERR_CUDA.
 *     Faults detected inside kernels (non-finite pack input, a bounded wait that
 *     expired) are recorded in a per-device status word read by
 *     qlinear_get_device_status().
 *   - Validation happens before any launch; on any error nothing is launched.
 *     Required: group == 64 (else QL_ERR_UNSUPPORTED); K % 64 == 0, N % 8 == 0,
 *     M >= 1, K >= 64, N >= 8, non-null tensors (else QL_ERR_INVALID_ARG); every
 *     pointer 16-byte aligned (else QL_ERR_ALIGNMENT); outputs must not overlap
 *     inputs (else QL_ERR_INVALID_ARG).
 *   - Non-finite activations or parameters propagate through the arithmetic
 *     IEEE-style.
 *   - Thread safety: calls are reentrant; the last-dispatch record is
 *     thread-local.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define QL_API __attribute__((visibility("default")))
#else
#define QL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QL_OK = 0,
    QL_ERR_INVALID_ARG = 1,     /* bad size, null pointer, overlap, non-finite pack input */
    QL_ERR_ALIGNMENT = 2,       /* a pointer is not 16-byte aligned */
    QL_ERR_UNSUPPORTED = 3,     /* group != 64, or a feature not built (see each call) */
    QL_ERR_WORKSPACE = 4,       /* workspace missing or smaller than qlinear_workspace_size() */
    QL_ERR_CUDA = 5,            /* a CUDA runtime call or kernel launch failed */
    QL_ERR_DEVICE_TIMEOUT = 6,  /* a bounded wait inside a kernel expired; the kernel returned early */
    QL_ERR_BOUNDS = 7           /* a kernel's own index check failed (debug builds) */
} ql_status;

typedef enum { QL_F32 = 0, QL_BF16 = 1 } ql_dtype;

/* Kernel paths of qlinear_forward, for qlinear_forward_config() and qlinear_last_dispatch(). */
typedef enum {
    QL_PATH_AUTO = 0,       /* per-shape choice of the dispatcher */
    QL_PATH_GEMV = 1,       /* CUDA-core split-K weight streaming (any M; meant for M <= 4) */
    QL_PATH_TC_SKINNY = 2,  /* tcgen05 weight streaming for small M: stream-K over K, fp32 partials
                               reduced in a fixed order; the dispatcher uses it for M <= 32, forced it
                               runs M <= 64 (QL_ERR_UNSUPPORTED above) */
    QL_PATH_TC_FUSED = 3    /* tcgen05 fused-dequant GEMM for large M */
    /* Both tcgen05 paths multiply f16 operands with fp32 accumulation in tensor memory: each
     * weight is rounded once, RN_f16(s * q + b), and each activation row is scaled by a power of
     * two into f16 (exact for entries above 2^-28 of the row's largest magnitude) and scaled back
     * after the accumulation.  QL_PATH_GEMV multiplies the exact codes in fp32. */
} ql_path;

/*
 * Bytes of device workspace qlinear_forward() needs for this shape (0 is
 * possible).  Returns (size_t)-1 when the shape is invalid.
 */
QL_API size_t qlinear_workspace_size(int64_t M, int64_t K, int64_t N, int32_t group);

/*
 * y = x . W^T for the packed W (the layer the pages describe: bf16
 * activations, fp32 accumulation, bf16 output).  Preconditions and errors as in
 * the conventions above; additionally `workspace` must hold at least
 * qlinear_workspace_size(M, K, N, group) bytes (QL_ERR_WORKSPACE otherwise)
 * and must not overlap any tensor.  The dispatcher picks the kernel path from
 * (M, K, N); qlinear_last_dispatch() reports the choice.
 */
QL_API ql_status qlinear_forward(const void* x, const uint32_t* codes, const void* scales,
                          const void* biases, void* y, int64_t M, int64_t K, int64_t N,
                          int32_t group, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/*
 * qlinear_forward with the path and split-K factor forced (testing and tuning).
 * path: a ql_path; split_k: 0 = the dispatcher's choice, else the number of K
 * slices, 1 <= split_k <= K/64 (and <= 1024 on the fused path; QL_ERR_INVALID_ARG otherwise); slice z covers the
 * groups [z*G/split_k, (z+1)*G/split_k), G = K/64.
 * out_dtype: QL_BF16 = the layer's output; QL_F32 writes y as fp32 [M][N]
 * (the same arithmetic without the final rounding, for numerical tests).
 * Split-K: QL_PATH_GEMV and QL_PATH_TC_FUSED take split_k > 1 (the fused path then writes one fp32
 * partial per slice into the workspace and sums them in slice order, for shapes with fewer output
 * tiles than SMs); QL_PATH_TC_SKINNY balances K itself and returns QL_ERR_UNSUPPORTED for it.
 * A path that cannot run the shape returns QL_ERR_UNSUPPORTED.
 */
QL_API ql_status qlinear_forward_config(const void* x, const uint32_t* codes, const void* scales,
                                 const void* biases, void* y, ql_dtype out_dtype,
                                 int64_t M, int64_t K, int64_t N, int32_t group,
                                 int32_t path, int32_t split_k,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes for qlinear_forward_config() with the same path and split_k. */
QL_API size_t qlinear_workspace_size_config(int64_t M, int64_t K, int64_t N, int32_t group,
                                     int32_t path, int32_t split_k);

/*
 * Standalone dequantization: out[n][k] = RN_fp32(s * q + b), rounded once more
 * to bf16 (nearest even) when out_dtype == QL_BF16.  Bit-exact by definition:
 * s*q + b is formed with one fused multiply-add.  out is [N][K] of out_dtype.
 */
QL_API ql_status qlinear_dequant(const uint32_t* codes, const void* scales, const void* biases,
                          int64_t K, int64_t N, int32_t group, void* out, ql_dtype out_dtype,
                          cudaStream_t stream);

/*
 * Quantize fp32 w [N][K] into codes/scales/biases.
 * imatrix == NULL: min/max round-to-nearest (MLX's own solution, candidate 0
 * of the search in aimarketly "Ideogram-4-IQ4_M", "What IQ4 means here"):
 * per group of 64, s = RN32(RN32(max-min)/15), scale = RN_f16(s),
 * bias = RN_f16(min), q = clamp(rint(RN32(RN32(w-bias)/scale)), 0, 15)
 * (ties to even), q = 0 when scale == 0.  Deterministic: equal inputs give
 * equal bytes.
 * imatrix != NULL: importance-weighted fit.  imatrix is fp32 [K], the per-channel
 * E[x^2] of the layer's activations (device memory, read only).  Per group the
 * candidates are the RTN triple, then 80 range shrinks (lo = min + a r,
 * hi = max - c r, a, c in {0, 0.025, ..., 0.2}), each refined by up to two
 * weighted least-squares refits of (scale, bias) with the codes fixed; the
 * triple with the lowest sum_j imp_j (w_j - RN32(s q_j + b))^2 (float64,
 * imp = imatrix + 1e-6 * mean(imatrix)) wins, ties to the earliest, so the fit
 * is never worse than RTN on that objective.  Deterministic: every float64 sum
 * is taken in index order with correctly rounded operations.  A negative or
 * non-finite imatrix entry is an argument error reported through the device
 * status word (all groups written as zeros).
 * A group holding a non-finite value or |w| > 65504 is written as codes 0,
 * scale 0, bias 0, and the device status word records QL_ERR_INVALID_ARG.
 */
QL_API ql_status qlinear_pack(const float* w, const float* imatrix, int64_t K, int64_t N, int32_t group,
                       uint32_t* codes, void* scales, void* biases, cudaStream_t stream);

/*
 * Synchronizes `stream`, then reads and clears the current device's status word
 * (the first error a kernel recorded since the last read).  Returns QL_OK when
 * no kernel recorded anything, QL_ERR_CUDA if the synchronization fails.
 */
QL_API ql_status qlinear_get_device_status(cudaStream_t stream);

/*
 * Writes a NUL-terminated description of the calling thread's last
 * qlinear_forward dispatch, e.g. "path=tc_fused bits=4 tile=256w x 192t x 64k stages=x5/c2x4/a2
 * ctas=148 splitk=1 launches=3 why=auto:M>64,split:9x72" (stages: activation, code x K-steps per
 * code stage, tensor-memory weight stages; launches = kernels that call enqueued; why = the rule or
 * the caller's forced path behind the choice),
 * truncated to len bytes.  QL_ERR_INVALID_ARG if buf is NULL or len == 0.
 */
QL_API ql_status qlinear_last_dispatch(char* buf, size_t len);

/*
 * Test hook of the checked build (libqlinear_bounds.so, compiled with QL_BOUNDS_CHECK); the pages have no
 * counterpart.  kernel_mask bit 0 holds back the code producer of the fused tensor-core kernel
 * (QL_PATH_TC_FUSED), bit 1 that of the weight-streaming kernel (QL_PATH_TC_SKINNY): they issue no code
 * or parameter load, so the kernel's other roles wait until the limit, record QL_ERR_DEVICE_TIMEOUT and
 * unwind (nothing of theirs in flight, tensor memory freed).  wait_limit_ns replaces the one-second
 * limit of every bounded wait in the library's kernels (> 0); call with kernel_mask 0 and 1000000000
 * to restore the defaults.  Synchronous (two small host-to-device copies on the legacy stream).
 * The shipped library returns QL_ERR_UNSUPPORTED and changes nothing; QL_ERR_INVALID_ARG for an
 * unknown bit or a zero limit.
 */
QL_API ql_status qlinear_test_stall(int32_t kernel_mask, uint64_t wait_limit_ns);

/*
 * Test hook of the checked build (libqlinear_bounds.so); the pages have no counterpart.  Selects the ring
 * depths of the fused tensor-core kernel that later 4-bit, bf16-output, unsplit qlinear_forward calls
 * (QL_PATH_TC_FUSED or the dispatcher's choice of it) launch on this process: variant 0 is the shipped
 * configuration, variants 1 .. QL_TEST_RING_VARIANTS-1 other (activation stages, code stages, epilogue
 * staging blocks per warp) triples.  Every ring position is a function of the step count alone, so the
 * output must be the same bytes for every variant.  The shipped library returns QL_ERR_UNSUPPORTED;
 * QL_ERR_INVALID_ARG for a variant out of range; QL_ERR_CUDA if the variant's shared-memory size
 * cannot be set on the current device.
 */
#define QL_TEST_RING_VARIANTS 7
QL_API ql_status qlinear_test_ring_depth(int32_t variant);

/*
 * Test hook of the checked build (libqlinear_bounds.so); the pages have no counterpart.  Holds back the
 * roles of the tensor-core kernels in role_mask at their start, each CTA's and warp's by a different part
 * (0/7 .. 7/7) of max_ns, so that every hand-off between roles (TMA rings, tensor-memory stages,
 * accumulators, partials) meets other orders of arrival; the output must not change.  Bits: 1 the
 * activation producer, 2 the code producer, 4 the dequantizers, 8 the MMA issuers, 16 the epilogue or
 * drain warps.  role_mask 0 turns it off.  Synchronous (two small host-to-device copies on the legacy
 * stream).  The shipped library returns QL_ERR_UNSUPPORTED; QL_ERR_INVALID_ARG for an unknown bit or
 * max_ns above 1 ms.
 */
QL_API ql_status qlinear_test_delay(int32_t role_mask, uint64_t max_ns);

/*
 * Allocation-free forward for small M.  The pages have no counterpart of this
 * call; it exists for callers that cannot allocate device memory where they
 * run the layer (a plugin living inside another engine's fixed memory pool, a
 * serving loop that must not allocate after start-up, a runtime that passes
 * only inputs and outputs and no workspace).
 *
 * Same arithmetic and arguments as qlinear_forward (bf16 y), restricted to
 * M <= QL_NOALLOC_MAX_M (QL_ERR_UNSUPPORTED above), and it allocates nothing:
 * its split-K partials live in a fixed scratch array of
 * QL_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library holds until the process exits.  A shape whose partials
 * would not fit returns QL_ERR_WORKSPACE.  The first call on a device looks up
 * that device's address of the array (cudaGetSymbolAddress with the device
 * current), so make the first call on each device before any stream capture.
 * All calls share the one array and it keeps the last call's contents: calls
 * that overlap on the GPU (other streams or host threads) race and must be
 * serialized by the caller.  No cudaMalloc, cudaFree or allocating library
 * routine is called.  The cached address is that of the context current at
 * the first call: do not use this entry point across cudaDeviceReset.  A
 * launch error already pending on the calling thread when the call is made
 * returns QL_ERR_CUDA before anything is launched and is left pending.
 * It runs the CUDA-core split-K path (QL_PATH_GEMV), whose cost grows with M
 * (each 4-row block of activations streams the weights again).
 */
#define QL_NOALLOC_SCRATCH_BYTES (4u << 20)
#define QL_NOALLOC_MAX_M 64
QL_API ql_status qlinear_forward_noalloc(const void* x, const uint32_t* codes, const void* scales,
                                         const void* biases, void* y, int64_t M, int64_t K, int64_t N,
                                         int32_t group, cudaStream_t stream);

/*
 * Measurement hook.  While set (both non-NULL), every qlinear_forward* call
 * made by the calling thread records `start` on its stream immediately before
 * its main kernel (the tensor-core GEMM or the weight-streaming kernel) and
 * `stop` immediately after it, so the main kernel can be timed alone.  The
 * caller owns both events; NULL, NULL turns the hook off.  Thread-local.
 */
QL_API ql_status qlinear_set_profile_events(cudaEvent_t start, cudaEvent_t stop);

/*
 * W8 g64: the 8-bit variant of the same format.  The pages ship an 8-bit pack beside the 4-bit one
 * (huggingface "SceneWorks/ideogram-4-mlx", Versions: Q8) and keep the modulation and conditioning
 * projections at 8 bits (aimarketly "Ideogram-4-IQ4_M", Conversion); the scale and bias stay one f16
 * pair per 64 weights, so a weight costs 8.5 bits.
 *
 *   codes   uint32   [N][K/4]    code (n, k) = (codes[n][k/4] >> 8*(k%4)) & 0xFF, low byte first
 *   scales, biases, x, y          as for the 4-bit calls; w = s * q + b with q in [0, 255]
 *
 * Each qlinear8_* call has the arguments, preconditions, errors and arithmetic of the 4-bit call of
 * the same name, with the code tensor above in place of the 4-bit one:
 *   qlinear8_forward / _config   y = x . W^T; the same kernel paths (QL_PATH_GEMV multiplies exact
 *                                codes in fp32; both tcgen05 paths multiply RN_f16(s * q + b) by f16
 *                                activations scaled per row by a power of two, fp32 accumulation)
 *   qlinear8_workspace_size[_config]
 *   qlinear8_dequant             out = RN_fp32(s * q + b) (bf16: rounded once more), bit-exact
 *   qlinear8_pack                min/max round-to-nearest with 255 levels:
 *                                s = RN32(RN32(max-min)/255), scale = RN_f16(s), bias = RN_f16(min),
 *                                q = clamp(rint(RN32(RN32(w-bias)/scale)), 0, 255) (ties to even),
 *                                q = 0 when scale == 0; imatrix must be NULL (QL_ERR_UNSUPPORTED
 *                                otherwise: the importance-weighted fit is built for 4-bit codes)
 */
QL_API size_t qlinear8_workspace_size(int64_t M, int64_t K, int64_t N, int32_t group);
QL_API size_t qlinear8_workspace_size_config(int64_t M, int64_t K, int64_t N, int32_t group,
                                             int32_t path, int32_t split_k);
QL_API ql_status qlinear8_forward(const void* x, const uint32_t* codes, const void* scales,
                                  const void* biases, void* y, int64_t M, int64_t K, int64_t N,
                                  int32_t group, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);
QL_API ql_status qlinear8_forward_config(const void* x, const uint32_t* codes, const void* scales,
                                         const void* biases, void* y, ql_dtype out_dtype,
                                         int64_t M, int64_t K, int64_t N, int32_t group,
                                         int32_t path, int32_t split_k,
                                         void* workspace, size_t workspace_bytes, cudaStream_t stream);
QL_API ql_status qlinear8_dequant(const uint32_t* codes, const void* scales, const void* biases,
                                  int64_t K, int64_t N, int32_t group, void* out, ql_dtype out_dtype,
                                  cudaStream_t stream);
QL_API ql_status qlinear8_pack(const float* w, const float* imatrix, int64_t K, int64_t N, int32_t group,
                               uint32_t* codes, void* scales, void* biases, cudaStream_t stream);

/*
 * SwiGLU up/gate pair in one call: h = silu(x . W_gate^T) * (x . W_up^T) elementwise, with
 * silu(z) = z / (1 + e^-z) (the DiT block's MLP is a SwiGLU of three Linears, jimmysue "Ideogram 4"
 * notes, sec. 2.1 and 2.8; this call covers the first two and the gating, the third is an ordinary
 * qlinear_forward of h).
 *
 *   x                                   bf16 [M][K]
 *   gate_codes / up_codes               uint32 [I][K/8], 4-bit codes as above
 *   gate_scales, gate_biases, up_...    f16 [I][K/64]
 *   h                                   [M][I], bf16 (QL_BF16) or fp32 (QL_F32, for numerical tests)
 *
 * Arithmetic of the tcgen05 path (QL_PATH_TC_FUSED): g and u accumulate in fp32 from f16 operands
 * (weights RN_f16(s * q + b), activations scaled per row by a power of two), then
 * h = g / (1 + expf(-g)) * u in fp32, rounded once to the output type.  One GEMM computes both: each
 * tile holds 128 rows of the gate weight and the same 128 rows of the up weight, so g and u of an
 * output element meet in the epilogue and never travel through memory.
 * Preconditions as for qlinear_forward with N = I (I % 8 == 0), all eight tensors 16-byte aligned,
 * h overlapping no input and the workspace overlapping nothing; `workspace` must hold
 * qlinear_swiglu_workspace_size(M, K, I, group) bytes (QL_ERR_WORKSPACE otherwise).
 */
QL_API size_t qlinear_swiglu_workspace_size(int64_t M, int64_t K, int64_t I, int32_t group);
QL_API ql_status qlinear_swiglu_forward(const void* x, const uint32_t* gate_codes, const void* gate_scales,
                                        const void* gate_biases, const uint32_t* up_codes,
                                        const void* up_scales, const void* up_biases, void* h,
                                        ql_dtype out_dtype, int64_t M, int64_t K, int64_t I, int32_t group,
                                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * y[i] = sum_{z=0}^{S-1} partials[z][i], summed in z order in fp32 and rounded once to out_dtype.
 * partials is fp32 [S][count] (device, read only), y is [count] of out_dtype; count % 4 == 0.
 * This is the combination step of a K-sharded (row-parallel) layer: the ranks' fp32 partial
 * outputs (qlinear_forward_config with QL_F32), gathered in rank order, reduce to the same bytes on
 * every rank.  Errors: QL_ERR_INVALID_ARG (null pointer, S < 1, count not a positive multiple of 4,
 * y overlapping partials, bad out_dtype), QL_ERR_ALIGNMENT (a pointer not 16-byte aligned).
 */
QL_API ql_status qlinear_reduce_partials(const float* partials, int32_t S, int64_t count, void* y,
                                         ql_dtype out_dtype, cudaStream_t stream);

/*
 * Self-test of the bounded waits inside the library's kernels.  Enqueues one small kernel that waits
 * on a barrier nothing ever completes, with the same bounded wait every pipeline role uses: it gives
 * up after the library's wait limit (about one second), records QL_ERR_DEVICE_TIMEOUT in the device
 * status word and returns, leaving the context usable.  A following qlinear_get_device_status()
 * therefore returns QL_ERR_DEVICE_TIMEOUT.  Returns QL_ERR_CUDA if the launch fails.
 */
QL_API ql_status qlinear_selftest_bounded_wait(cudaStream_t stream);

/* Static, human-readable name of a status code. */
QL_API const char* qlinear_status_string(ql_status status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
QL_API int32_t qlinear_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */
