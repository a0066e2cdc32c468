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

}  // namespace quant
}  // namespace w4a8
