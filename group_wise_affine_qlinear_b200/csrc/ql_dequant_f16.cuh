// Code unpack and affine dequantization to f16, shared by the tensor-core kernels.
#pragma once

#include "ql_common.cuh"

namespace ql {

// Dequantize one code word (8 codes, k order 0..7) into 4 f16x2 words holding the
// pairs (0,4), (1,5), (2,6), (3,7).  A nibble at bits 0-3 / 16-19 ORed into 1024.0
// (0x6400, unit in the last place 1) gives 1024 + q exactly; a nibble at bits
// 4-7 / 20-23 ORed into 64.0 (0x5400, unit 1/16) gives 64 + q exactly.
// Subtracting the magic leaves q exactly; one fused f16x2 FMA then forms
// RN_f16(s*q + b).
__device__ __forceinline__ void dequant_word(uint32_t v, __half2 s2, __half2 b2, uint32_t* o) {
    const uint32_t v8 = v >> 8;
    uint32_t p0, p1, p2, p3;
    asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(p0) : "r"(v));
    asm("lop3.b32 %0, %1, 0x00F000F0, 0x54005400, 0xEA;" : "=r"(p1) : "r"(v));
    asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(p2) : "r"(v8));
    asm("lop3.b32 %0, %1, 0x00F000F0, 0x54005400, 0xEA;" : "=r"(p3) : "r"(v8));
    const __half2 m1024 = half2_of(0x64006400u);
    const __half2 m64 = half2_of(0x54005400u);
    o[0] = bits_of(__hfma2(__hsub2(half2_of(p0), m1024), s2, b2));
    o[1] = bits_of(__hfma2(__hsub2(half2_of(p1), m64), s2, b2));
    o[2] = bits_of(__hfma2(__hsub2(half2_of(p2), m1024), s2, b2));
    o[3] = bits_of(__hfma2(__hsub2(half2_of(p3), m64), s2, b2));
}

// Dequantize one word of 8-bit codes (4 codes, k order 0..3) into 2 f16x2 words holding the
// pairs (0,2) and (1,3).  A code byte placed under the byte 0x64 is the f16 1024 + q exactly
// (1024.0 = 0x6400, unit in the last place 1, and q <= 255); one byte permute per pair builds it
// from the word and the magic byte.  Subtracting 1024 leaves q exactly; one fused f16x2 FMA then
// forms RN_f16(s*q + b).
__device__ __forceinline__ void dequant_word8(uint32_t v, __half2 s2, __half2 b2, uint32_t* o) {
    const uint32_t p0 = __byte_perm(v, 0x64646464u, 0x4240u);    // bytes: q0, 0x64, q2, 0x64
    const uint32_t p1 = __byte_perm(v, 0x64646464u, 0x4341u);    // bytes: q1, 0x64, q3, 0x64
    const __half2 m1024 = half2_of(0x64006400u);
    o[0] = bits_of(__hfma2(__hsub2(half2_of(p0), m1024), s2, b2));
    o[1] = bits_of(__hfma2(__hsub2(half2_of(p1), m1024), s2, b2));
}

}  // namespace ql
