// int4 (and 8-bit) -> fp16 decoding of the tiled weight layouts (include/w4a16.h): each
// 32-bit word holds eight signed codes of one column, nibble i holding
// k_local {0,2,4,6,1,3,5,7}[i], so that the decoder below yields (k, k+1)
// pairs in natural order.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "ptx.cuh"

namespace w4a16 {

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }
__device__ __forceinline__ __half2 bits_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }

// Eight int4 codes of one word (nibble i = k_local {0,2,4,6,1,3,5,7}[i]) ->
// eight fp16 weights q*s in natural k order. Each code c is read as the fp16
// number 1024 + (c ^ 8) (or 1024 + 16*(c ^ 8) for the high nibble of a byte)
// by OR-ing it under the exponent of 1024; subtracting the bias then gives the
// signed code exactly, and one multiply applies the group scale.
__device__ __forceinline__ uint4 dequant_word(uint32_t x, __half2 s2) {
    const __half2 bias_lo = bits_h2(0x64086408u);  // 1032, 1032
    const __half2 sixteenth = bits_h2(0x2C002C00u);  // 1/16, 1/16
    const __half2 bias_hi = bits_h2(0xD480D480u);  // -72, -72
    const uint32_t b0 = lop3_and_xor(x, 0x000F000Fu, 0x64086408u);
    const uint32_t t0 = lop3_and_xor(x, 0x00F000F0u, 0x64806480u);
    const uint32_t x8 = x >> 8;
    const uint32_t b1 = lop3_and_xor(x8, 0x000F000Fu, 0x64086408u);
    const uint32_t t1 = lop3_and_xor(x8, 0x00F000F0u, 0x64806480u);
    const __half2 q01 = __hsub2(bits_h2(b0), bias_lo);
    const __half2 q23 = __hfma2(bits_h2(t0), sixteenth, bias_hi);
    const __half2 q45 = __hsub2(bits_h2(b1), bias_lo);
    const __half2 q67 = __hfma2(bits_h2(t1), sixteenth, bias_hi);
    uint4 out;
    out.x = h2_bits(__hmul2(q01, s2));
    out.y = h2_bits(__hmul2(q23, s2));
    out.z = h2_bits(__hmul2(q45, s2));
    out.w = h2_bits(__hmul2(q67, s2));
    return out;
}

// The same decode without the scale: the signed codes themselves, exactly.
__device__ __forceinline__ uint4 decode_word(uint32_t x) {
    const __half2 bias_lo = bits_h2(0x64086408u);
    const __half2 sixteenth = bits_h2(0x2C002C00u);
    const __half2 bias_hi = bits_h2(0xD480D480u);
    const uint32_t b0 = lop3_and_xor(x, 0x000F000Fu, 0x64086408u);
    const uint32_t t0 = lop3_and_xor(x, 0x00F000F0u, 0x64806480u);
    const uint32_t x8 = x >> 8;
    const uint32_t b1 = lop3_and_xor(x8, 0x000F000Fu, 0x64086408u);
    const uint32_t t1 = lop3_and_xor(x8, 0x00F000F0u, 0x64806480u);
    uint4 out;
    out.x = h2_bits(__hsub2(bits_h2(b0), bias_lo));
    out.y = h2_bits(__hfma2(bits_h2(t0), sixteenth, bias_hi));
    out.z = h2_bits(__hsub2(bits_h2(b1), bias_lo));
    out.w = h2_bits(__hfma2(bits_h2(t1), sixteenth, bias_hi));
    return out;
}

// Four signed 8-bit codes of one word (byte b = k_local b) -> two fp16 pairs
// (q0, q1) * s and (q2, q3) * s. Flipping the sign bit of each byte gives
// c + 128 in [0, 255]; placed under the exponent byte of 1024 (0x64) it reads as
// the fp16 number 1024 + c + 128, exactly, and subtracting 1152 leaves c.
__device__ __forceinline__ uint2 dequant_word8(uint32_t x, __half2 s2) {
    const uint32_t u = x ^ 0x80808080u;
    const uint32_t lo = __byte_perm(u, 0x64646464u, 0x4140u);  // bytes (u0, 0x64, u1, 0x64)
    const uint32_t hi = __byte_perm(u, 0x64646464u, 0x4342u);  // bytes (u2, 0x64, u3, 0x64)
    const __half2 bias = bits_h2(0x64806480u);                 // 1152, 1152
    uint2 out;
    out.x = h2_bits(__hmul2(__hsub2(bits_h2(lo), bias), s2));
    out.y = h2_bits(__hmul2(__hsub2(bits_h2(hi), bias), s2));
    return out;
}

}  // namespace w4a16
