// Per-element helpers of the per-token int8 quantizer, shared by the
// quantize kernel and the fused decode kernel ("Quantization" notes,
// Symmetric Quantization: q = clip(round(x / s), -127, 127), round half to
// even, x / s one IEEE fp32 division).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace w4a8 {
namespace quant {

// 16 consecutive elements of a row as fp32.
template <typename T>
__device__ __forceinline__ void load16(const T* src, float (&v)[16]);

template <>
__device__ __forceinline__ void load16<float>(const float* src, float (&v)[16]) {
    const float4* s = reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 f = s[i];
        v[4 * i + 0] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
    }
}

template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16* src, float (&v)[16]) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 u = s[i];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // bf16 -> fp32 is a 16-bit shift
            v[8 * i + 2 * j + 0] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

// Code for one element: rne(fl32(x / s)) clamped to [-127, 127].
// Fast path: x * fl32(1/s) is within 2^-23 |x/s| <= 1.6e-5 of x/s, and the
// correctly rounded quotient within 3.9e-6, so when the product is farther
// than 2^-14 from a half-integer both round to the same integer.  Otherwise
// (or for tiny s, whose reciprocal would overflow) take the IEEE division.
__device__ __forceinline__ int code_i8(float x, float s, float rcp, bool exact_only) {
    float t = __fmul_rn(x, rcp);
    float r = rintf(t);
    if (exact_only || fabsf(t - r) > 0.49993896484375f) {
        t = __fdiv_rn(x, s);
        r = rintf(t);
    }
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    return int(r);
}

// The same code, returned in the low byte of a 32-bit word (the other bytes
// are unspecified), with the rounding done by adding 1.5 * 2^23: for |t| <
// 2^22 the sum's round-to-nearest-even drops t's fraction exactly as rint
// does, and its low mantissa bits are the integer in two's complement.  No
// clamp on the fast path: s = fl32(max|x| / 127) and the product's error
// keep |t| below 127.5, so the code already lies in [-127, 127].
__device__ __forceinline__ uint32_t code_i8_byte(float x, float s, float rcp, bool exact_only) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const float t = __fmul_rn(x, rcp);
    const float m = __fadd_rn(t, kMagic);
    const float r = __fsub_rn(m, kMagic);
    if (!exact_only && fabsf(__fsub_rn(t, r)) <= 0.49993896484375f) return __float_as_uint(m);
    return uint32_t(code_i8(x, s, rcp, exact_only));
}

// Four codes (low bytes of a, b, c, d) as one word: byte 0 = a, ..., byte 3 = d.
__device__ __forceinline__ uint32_t pack4_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

}  // namespace quant
}  // namespace w4a8
