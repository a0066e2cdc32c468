// Offline weight preparation for sm_100a: per-group int4 quantization, nibble
// packing, the amplifier search and the integer group scales.
//
// 探秘Transformer系列之（34）量化基礎 §2.3.3 逐组量化 (one scale per group of
// consecutive K entries of a weight column); "Quantization" notes, Symmetric
// Quantization (s = max|w| / qmax, z = 0), here with qmax = 7 (codes [-7, 7]),
// or the full signed 4-bit range [-8, 7] of 极致量化 其他子4位整数格式 with
// s = max|w| / 8; Integer Scale
// summary §4 (amplifier search, S = round(s_g * alpha)); 极致量化 数据打包.
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "kernels.h"

namespace w4a8 {
namespace pack {

constexpr int kThreads = 256;

__device__ __forceinline__ float pos_inf() { return __int_as_float(0x7f800000); }

// s_g[g, n] = fl32(max_{k in g} |w[k, n]| / qdiv), qdiv = 7 for codes in
// [-7, 7] or 8 for the full two's-complement range [-8, 7].  One thread per
// column n and group g; threads of a warp read consecutive columns of one row.
__global__ void __launch_bounds__(kThreads) group_scales_kernel(const float* __restrict__ w, int64_t K, int64_t N,
                                                                int32_t group, float qdiv, float* __restrict__ s_g) {
    const int64_t n = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t g = blockIdx.y;
    if (n >= N) return;
    const float* col = w + g * group * N + n;
    float a = 0.0f;
    for (int32_t k = 0; k < group; ++k) a = fmaxf(a, fabsf(col[int64_t(k) * N]));
    s_g[g * N + n] = (a == 0.0f) ? 0.0f : __fdiv_rn(a, qdiv);
}

// Per-block smallest positive and largest scale.
__global__ void __launch_bounds__(kThreads) minmax_kernel(const float* __restrict__ s, int64_t count,
                                                          float2* __restrict__ partial) {
    __shared__ float smin[kThreads / 32], smax[kThreads / 32];
    float mn = pos_inf();
    float mx = 0.0f;
    for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < count; i += int64_t(gridDim.x) * kThreads) {
        const float v = s[i];
        if (v > 0.0f) mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if ((threadIdx.x & 31) == 0) {
        smin[threadIdx.x >> 5] = mn;
        smax[threadIdx.x >> 5] = mx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) {
            mn = fminf(mn, smin[w]);
            mx = fmaxf(mx, smax[w]);
        }
        mn = fminf(mn, smin[0]);
        mx = fmaxf(mx, smax[0]);
        partial[blockIdx.x] = make_float2(mn, mx);
    }
}

// Combine the partials and choose the amplifier: the smallest power of two
// that lifts the smallest positive scale to at least 1 (1 when every scale is
// already >= 1 or none is positive), or the caller's fixed amplifier.
__global__ void amplifier_kernel(const float2* __restrict__ partial, int nblocks, int32_t alpha_in,
                                 Results* __restrict__ out) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    float mn = pos_inf();
    float mx = 0.0f;
    for (int i = 0; i < nblocks; ++i) {
        mn = fminf(mn, partial[i].x);
        mx = fmaxf(mx, partial[i].y);
    }
    int32_t alpha = 1;
    int32_t err = 0;
    if (alpha_in > 0) {
        alpha = alpha_in;
    } else if (mn <= FLT_MAX) {
        int shifts = 0;
        float amplified = mn;  // mn * 2^shifts, exact
        while (amplified < 1.0f) {
            amplified *= 2.0f;
            ++shifts;
            if (shifts > 30) {
                err = 1;
                break;
            }
        }
        alpha = err ? 0 : int32_t(1u << shifts);
    }
    out->alpha = alpha;
    out->error = err;
    out->s_min_pos = mn;
    out->s_max = mx;
    out->colsum_max = 0ull;
}

// Codes, nibble packing and integer scales.  One thread per column n and
// 32-wide K chunk: it reads w[k0..k0+31, n] (coalesced across the warp's
// consecutive n) and writes 16 packed bytes packed[n, k0/2 ..].
__global__ void __launch_bounds__(kThreads) quantize_pack_kernel(const float* __restrict__ w,
                                                                 const float* __restrict__ s_g, int32_t alpha,
                                                                 int64_t K, int64_t N, int32_t group, float qmin,
                                                                 uint8_t* __restrict__ packed,
                                                                 int16_t* __restrict__ S) {
    const int64_t n = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t k0 = int64_t(blockIdx.y) * 32;
    if (n >= N) return;
    const int64_t g = k0 / group;
    const float s = s_g[g * N + n];
    uint32_t words[4] = {0u, 0u, 0u, 0u};
    if (s != 0.0f) {
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const float t = __fdiv_rn(w[(k0 + i) * N + n], s);
            const float r = fminf(fmaxf(rintf(t), qmin), 7.0f);  // qmin: -7 or -8
            const uint32_t nib = uint32_t(int(r)) & 0xFu;
            // code j = i mod 8 of its word: byte j mod 4, high nibble for j >= 4
            words[i >> 3] |= nib << (8 * (i & 3) + 4 * ((i >> 2) & 1));
        }
    }
    *reinterpret_cast<uint4*>(packed + n * (K / 2) + k0 / 2) = make_uint4(words[0], words[1], words[2], words[3]);
    if (S != nullptr && (k0 % group) == 0) S[g * N + n] = int16_t(rintf(s * float(alpha)));  // s * alpha exact
}

// 8-bit weight codes (the W8A8 variant): q = clip(rne(fl32(w / s_g)), -127, 127)
// with s_g = max|w| / 127, stored K-contiguous per column, w8[n, k].  One
// thread per column n and 32-wide K chunk, 32 bytes written per thread.
__global__ void __launch_bounds__(kThreads) quantize_w8_kernel(const float* __restrict__ w,
                                                               const float* __restrict__ s_g, int32_t alpha,
                                                               int64_t K, int64_t N, int32_t group,
                                                               int8_t* __restrict__ w8, int16_t* __restrict__ S) {
    const int64_t n = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t k0 = int64_t(blockIdx.y) * 32;
    if (n >= N) return;
    const int64_t g = k0 / group;
    const float s = s_g[g * N + n];
    uint32_t words[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (s != 0.0f) {
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const float t = __fdiv_rn(w[(k0 + i) * N + n], s);
            const float r = fminf(fmaxf(rintf(t), -127.0f), 127.0f);
            words[i >> 2] |= (uint32_t(int(r)) & 0xFFu) << (8 * (i & 3));
        }
    }
    uint4* dst = reinterpret_cast<uint4*>(w8 + n * K + k0);
    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
    dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    if (S != nullptr && (k0 % group) == 0) S[g * N + n] = int16_t(rintf(s * float(alpha)));  // s * alpha exact
}

// max over columns of sum_g |S[g, n]|.
__global__ void __launch_bounds__(kThreads) colsum_kernel(const int16_t* __restrict__ S, int64_t G, int64_t N,
                                                          unsigned long long* __restrict__ out) {
    const int64_t n = int64_t(blockIdx.x) * kThreads + threadIdx.x;
    unsigned long long t = 0ull;
    if (n < N)
        for (int64_t g = 0; g < G; ++g) {
            const int v = S[g * N + n];
            t += unsigned(v < 0 ? -v : v);
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long u = __shfl_xor_sync(0xffffffffu, t, o);
        t = u > t ? u : t;
    }
    if ((threadIdx.x & 31) == 0) atomicMax(out, t);
}

// Weight-side zero-point term of an asymmetric activation ("Quantization"
// notes, quantized matmul expansion: with Z_W = 0 the term Z_X q_W depends on
// the weights alone and is precomputed; with integer group scales it is
// zc[n] = sum_g S[g, n] * sum_{k in g} q[k, n]).  One warp per column; each
// lane sums whole 16-byte chunks of the packed row, 32 codes of one group (the
// order of the nibbles inside a chunk does not matter to a sum).  Sums wrap in
// 32 bits like the GEMM's accumulator, which subtracts z[m] * zc[n].
__global__ void __launch_bounds__(kThreads) zero_point_term_kernel(const uint8_t* __restrict__ packed,
                                                                   const int16_t* __restrict__ S, int64_t K,
                                                                   int64_t N, int32_t group,
                                                                   int32_t* __restrict__ zc) {
    constexpr int kWarps = kThreads / 32;
    const int lane = threadIdx.x & 31;
    const int64_t chunks = K / 32;
    const int64_t chunks_per_group = group / 32;
    const int64_t stride = int64_t(gridDim.x) * kWarps;
    for (int64_t n = int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5); n < N; n += stride) {
        const uint4* row = reinterpret_cast<const uint4*>(packed + n * (K / 2));
        uint32_t t = 0u;
        for (int64_t c = lane; c < chunks; c += 32) {
            const uint4 v = row[c];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            int32_t sum = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) sum += int32_t(w[i] << (28 - 4 * j)) >> 28;  // nibble j, sign-extended
            t += uint32_t(int32_t(S[(c / chunks_per_group) * N + n])) * uint32_t(sum);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == 0) zc[n] = int32_t(t);
    }
}

cudaError_t zero_point_term(const uint8_t* packed, const int16_t* S, int64_t K, int64_t N, int32_t group,
                            int32_t* zc, cudaStream_t stream, int num_sms) {
    const int64_t per_block = kThreads / 32;
    int64_t blocks = (N + per_block - 1) / per_block;
    if (blocks > int64_t(num_sms) * 8) blocks = int64_t(num_sms) * 8;
    zero_point_term_kernel<<<unsigned(blocks), kThreads, 0, stream>>>(packed, S, K, N, group, zc);
    return cudaGetLastError();
}

cudaError_t group_scales(const float* w, int64_t K, int64_t N, int32_t group, int32_t qmin, float* s_g,
                         cudaStream_t stream) {
    return group_scales_div(w, K, N, group, qmin == -8 ? 8.0f : 7.0f, s_g, stream);
}

cudaError_t group_scales_div(const float* w, int64_t K, int64_t N, int32_t group, float qdiv, float* s_g,
                             cudaStream_t stream) {
    dim3 grid(unsigned((N + kThreads - 1) / kThreads), unsigned(K / group));
    group_scales_kernel<<<grid, kThreads, 0, stream>>>(w, K, N, group, qdiv, s_g);
    return cudaGetLastError();
}

cudaError_t amplifier(const float* scales, int64_t count, int32_t alpha_in, void* workspace, cudaStream_t stream,
                      int num_sms) {
    auto* res = static_cast<Results*>(workspace);
    auto* partial = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + kPartialsOffset);
    int64_t blocks = (count + kThreads - 1) / kThreads;
    const int64_t cap = int64_t(num_sms) * 4 < kMaxPartialBlocks ? int64_t(num_sms) * 4 : kMaxPartialBlocks;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    minmax_kernel<<<unsigned(blocks), kThreads, 0, stream>>>(scales, count, partial);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    amplifier_kernel<<<1, 32, 0, stream>>>(partial, int(blocks), alpha_in, res);
    return cudaGetLastError();
}

cudaError_t quantize_w8(const float* w, const float* s_g, int32_t alpha, int64_t K, int64_t N, int32_t group,
                       int8_t* w8, int16_t* S, void* workspace, cudaStream_t stream) {
    dim3 grid(unsigned((N + kThreads - 1) / kThreads), unsigned(K / 32));
    quantize_w8_kernel<<<grid, kThreads, 0, stream>>>(w, s_g, alpha, K, N, group, w8, S);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || S == nullptr) return e;
    auto* res = static_cast<Results*>(workspace);
    colsum_kernel<<<unsigned((N + kThreads - 1) / kThreads), kThreads, 0, stream>>>(S, K / group, N,
                                                                                   &res->colsum_max);
    return cudaGetLastError();
}

cudaError_t quantize_pack(const float* w, const float* s_g, int32_t alpha, int64_t K, int64_t N, int32_t group,
                          int32_t qmin, uint8_t* packed, int16_t* S, void* workspace, cudaStream_t stream) {
    dim3 grid(unsigned((N + kThreads - 1) / kThreads), unsigned(K / 32));
    quantize_pack_kernel<<<grid, kThreads, 0, stream>>>(w, s_g, alpha, K, N, group, float(qmin), packed, S);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || S == nullptr) return e;
    auto* res = static_cast<Results*>(workspace);
    colsum_kernel<<<unsigned((N + kThreads - 1) / kThreads), kThreads, 0, stream>>>(S, K / group, N,
                                                                                   &res->colsum_max);
    return cudaGetLastError();
}

}  // namespace pack
}  // namespace w4a8
