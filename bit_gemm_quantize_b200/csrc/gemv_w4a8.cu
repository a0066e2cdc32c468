// Decode-shaped W4A8 layer (M <= 4 tokens) on the CUDA cores: the weight
// stream is the whole cost, so the kernel is built for HBM bandwidth, not for
// the tensor cores.  A 128-row int8 MMA takes about 95 cycles even with 16
// tokens (measured with the library's tensor-pipe probe), which caps a
// tensor-core pass over packed weights near the HBM rate; here each weight
// byte costs a few integer instructions and the loads stream at full rate.
//
// Integer Scale: A Free Lunch for Faster Fine-grained Quantization of LLMs
// (summary), Fig. 3(c) and §4 (integer group scales, one rescale at the end)
// and §3.2 / Fig. 3(b) (the float-scale comparison path); "Quantization"
// notes, Symmetric Quantization (the token codes).
//
// Layout: a CTA owns 32 consecutive output columns n (lane = column) and
// splits K over its warps.  Every lane streams its column's packed weights,
// 64 bytes (one group of 128 K) at a time with four 16-byte loads; the int4
// codes become 16 * q in int8 lanes (three integer ops per 8 weights) and
// dp4a multiplies them with the token codes, which sit in shared memory and
// are read by all lanes at once (broadcast).  Per group and token:
//   P_g = (sum of dp4a) >> 4            (exact: every product is 16 q x)
//   acc += S[g,n] * P_g                 (integer scale: one IMAD)
//   accf += s_g[g,n] * float(P_g)       (float scale: one I2F and one FMA)
// The warps' partial sums are added in a fixed order through shared memory,
// and y = acc * s_a[m] / alpha (or accf * s_a[m]) is stored once per output.
//
// FUSED: the CTA quantizes the tokens itself (per-token absmax over all of K,
// then the codes), so one launch takes bf16 / fp32 tokens to the output: the
// quantize step of the path fused into the GEMM's prologue.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "gemm_common.cuh"
#include "gemm_w4a8.h"
#include "kernels.h"
#include "quant_common.cuh"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace gemv {

constexpr int kCols = 32;  // output columns per CTA (one per lane)

// Shared memory of a CTA: the token codes [mt][K], their output scales, and
// the warps' partial sums [ks][mt][32].
int smem_bytes(int mt, int K, int ks) { return mt * K + 16 + ks * mt * kCols * 4; }

// x: the tokens, either their int8 codes (MT rows used of M) or bf16 / fp32 values
template <int MT, int PATH, typename XT>
__global__ void __launch_bounds__(512) gemv_kernel(const GemvParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int K = p.K;
    int8_t* codes = reinterpret_cast<int8_t*>(smem);                                   // [MT][K]
    float* scl = reinterpret_cast<float*>(smem + MT * K);                              // [MT] output scales
    int32_t* red = reinterpret_cast<int32_t*>(smem + MT * K + 16);                     // [ks][MT][32]
    float* redf = reinterpret_cast<float*>(red);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ks = blockDim.x >> 5;
    const int nthreads = blockDim.x;
    if (threadIdx.x == 0) griddep_launch_dependents();
    griddep_wait();  // the tokens may be the previous kernel's output, y its input

    // ---- the token codes of rows 0..MT-1 (rows past M: zero codes, scale 0)
    constexpr bool kFused = !std::is_same<XT, int8_t>::value;
    if constexpr (kFused) {
        __shared__ float wmax[16];
        for (int m = 0; m < MT; ++m) {
            const bool live = m < p.M;
            const XT* row = reinterpret_cast<const XT*>(p.x) + int64_t(m) * p.ldx;
            float a = 0.0f;
            if (live) {
                for (int c = threadIdx.x; c < K / 16; c += nthreads) {
                    float v[16];
                    quant::load16<XT>(row + c * 16, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            if (lane == 0) wmax[warp] = a;
            __syncthreads();
            float amax = 0.0f;
            for (int w = 0; w < ks; ++w) amax = fmaxf(amax, wmax[w]);
            const float s = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
            const bool zero = (s == 0.0f);
            const bool exact_only = s < 1e-30f;
            const float rcp = zero ? 0.0f : __frcp_rn(s);
            for (int c = threadIdx.x; c < K / 16; c += nthreads) {
                uint32_t packed[4] = {0u, 0u, 0u, 0u};
                if (live && !zero) {
                    float v[16];
                    quant::load16<XT>(row + c * 16, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        packed[i >> 2] |= (uint32_t(quant::code_i8(v[i], s, rcp, exact_only)) & 0xFFu) << (8 * (i & 3));
                }
                const uint4 q4 = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                *reinterpret_cast<uint4*>(codes + m * K + c * 16) = q4;
                if (live && blockIdx.x == 0 && p.q_out)  // the codes and scales, for a caller that keeps them
                    *reinterpret_cast<uint4*>(p.q_out + int64_t(m) * K + c * 16) = q4;
            }
            if (threadIdx.x == 0) {
                scl[m] = PATH == gemm::kIntScale ? __fmul_rn(s, p.inv_alpha) : s;
                if (live && blockIdx.x == 0 && p.s_out) p.s_out[m] = s;
            }
            __syncthreads();  // wmax is reused by the next row
        }
    } else {
        const int8_t* q = reinterpret_cast<const int8_t*>(p.x);
        for (int c = threadIdx.x; c < MT * (K / 16); c += nthreads) {
            const int m = c / (K / 16), cc = c - m * (K / 16);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (m < p.M) v = *reinterpret_cast<const uint4*>(q + int64_t(m) * K + cc * 16);
            *reinterpret_cast<uint4*>(codes + m * K + cc * 16) = v;
        }
        if (threadIdx.x < MT) {
            const float s = threadIdx.x < p.M ? p.s_a[threadIdx.x] : 0.0f;
            scl[threadIdx.x] = PATH == gemm::kIntScale ? __fmul_rn(s, p.inv_alpha) : s;
        }
    }
    __syncthreads();

    // ---- this warp's groups of this lane's column
    const int n = blockIdx.x * kCols + lane;
    const bool nvalid = n < p.N;
    const int n_ld = nvalid ? n : 0;  // a column past N reads column 0 (never stored)
    const int G = p.G;
    const int gpw = G / ks;           // groups per warp (ks divides G)
    const int g0 = warp * gpw;
    const int kbpg = p.group >> 7;    // 128-wide K blocks per group
    const uint8_t* wrow = p.w + int64_t(n_ld) * (K / 2);
    int32_t acc[MT];
    float accf[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        acc[m] = 0;
        accf[m] = 0.0f;
    }
    // loads of the first K block, then one block ahead
    const int kb0 = g0 * kbpg, kb1 = (g0 + gpw) * kbpg;
    uint4 cur[4], nxt[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cur[i] = __ldg(reinterpret_cast<const uint4*>(wrow + kb0 * 64) + i);
    int32_t pg[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) pg[m] = 0;
    // this column's scales, loaded two groups ahead of their use
    auto ld_scale = [&](int g) -> uint32_t {
        if (g >= g0 + gpw) return 0u;
        const int64_t si = int64_t(g) * p.N + n_ld;
        if constexpr (PATH == gemm::kIntScale)
            return uint32_t(int32_t(__ldg(p.S + si)));
        else
            return __float_as_uint(__ldg(p.s_g + si));
    };
    uint32_t sc0 = ld_scale(g0), sc1 = ld_scale(g0 + 1);
    int g_cur = g0;
    for (int kb = kb0; kb < kb1; ++kb) {
        if (kb + 1 < kb1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) nxt[i] = __ldg(reinterpret_cast<const uint4*>(wrow + (kb + 1) * 64) + i);
        }
        // 128 weights: 16 packed words -> 32 words of four 16 q each, K order
        uint32_t wq[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint2 a = gemm::unpack_int4x8_x16(cur[i].x), b = gemm::unpack_int4x8_x16(cur[i].y);
            const uint2 c = gemm::unpack_int4x8_x16(cur[i].z), d = gemm::unpack_int4x8_x16(cur[i].w);
            wq[8 * i + 0] = a.x; wq[8 * i + 1] = a.y; wq[8 * i + 2] = b.x; wq[8 * i + 3] = b.y;
            wq[8 * i + 4] = c.x; wq[8 * i + 5] = c.y; wq[8 * i + 6] = d.x; wq[8 * i + 7] = d.y;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint4* xr = reinterpret_cast<const uint4*>(codes + m * K + kb * 128);
            int32_t s = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // 16 token codes per shared-memory load (all lanes read the same)
                const uint4 x4 = xr[j];
                s = __dp4a(int(wq[4 * j + 0]), int(x4.x), s);
                s = __dp4a(int(wq[4 * j + 1]), int(x4.y), s);
                s = __dp4a(int(wq[4 * j + 2]), int(x4.z), s);
                s = __dp4a(int(wq[4 * j + 3]), int(x4.w), s);
            }
            pg[m] += s;
        }
        if ((kb + 1) % kbpg == 0) {  // the group ends: apply its scale
            const uint32_t sraw = sc0;
            sc0 = sc1;
            sc1 = ld_scale(g_cur + 2);
            ++g_cur;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int32_t P = pg[m] >> 4;  // exact: 16 P_g
                if constexpr (PATH == gemm::kIntScale)
                    acc[m] += int32_t(sraw) * P;
                else
                    accf[m] = __fmaf_rn(__uint_as_float(sraw), __int2float_rn(P), accf[m]);
                pg[m] = 0;
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    }

    // ---- the warps' partial sums, added in warp order, and the output
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if constexpr (PATH == gemm::kIntScale)
            red[(warp * MT + m) * kCols + lane] = acc[m];
        else
            redf[(warp * MT + m) * kCols + lane] = accf[m];
    }
    __syncthreads();
    if (warp < MT && warp < p.M && nvalid) {
        const int m = warp;
        int32_t a = 0;
        float af = 0.0f;
        for (int w = 0; w < ks; ++w) {
            if constexpr (PATH == gemm::kIntScale)
                a += red[(w * MT + m) * kCols + lane];
            else
                af = __fadd_rn(af, redf[(w * MT + m) * kCols + lane]);
        }
        const float v = __fmul_rn(PATH == gemm::kIntScale ? __int2float_rn(a) : af, scl[m]);
        const int64_t o = int64_t(m) * p.N + n;
        if (p.y_dtype == gemm::kOutI32)
            reinterpret_cast<int32_t*>(p.y)[o] = a;
        else if (p.y_dtype == gemm::kOutF16)
            reinterpret_cast<__half*>(p.y)[o] = __float2half_rn(v);
        else
            reinterpret_cast<float*>(p.y)[o] = v;
    }
}

template <int MT, int PATH, typename XT>
static cudaError_t launch_t(const GemvParams& p, int ks, cudaStream_t stream) {
    constexpr auto kern = gemv_kernel<MT, PATH, XT>;
    const int smem = smem_bytes(MT, p.K, ks);
    const cudaError_t e = configure_once<kern>(32 * ks, smem_bytes(MT, kMaxK, 16));
    if (e != cudaSuccess) return e;
    const unsigned grid = unsigned((p.N + kCols - 1) / kCols);
    const LaunchPdl lc(grid, unsigned(32 * ks), size_t(smem), stream);
    return cudaLaunchKernelEx(&lc.cfg, kern, p);
}

template <int PATH, typename XT>
static cudaError_t launch_path(const GemvParams& p, int ks, cudaStream_t stream) {
    switch (p.M) {
        case 1: return launch_t<1, PATH, XT>(p, ks, stream);
        case 2: return launch_t<2, PATH, XT>(p, ks, stream);
        default: return launch_t<4, PATH, XT>(p, ks, stream);
    }
}

}  // namespace gemv

namespace gemv {

// Warps per CTA: enough CTAs x warps to keep every SM streaming (about 32
// warps per SM, each with two 2 KB K blocks of loads in flight), at most 16,
// and a divisor of the group count.
int warps_for(int64_t N, int64_t G, int num_sms) {
    const int64_t blocks = (N + kCols - 1) / kCols;
    int ks = 1;
    while (ks < 16 && blocks * ks < int64_t(num_sms) * 32 && G % (2 * ks) == 0) ks *= 2;
    return ks;
}

cudaError_t launch(const GemvParams& p, int path, int x_kind, int num_sms, cudaStream_t stream) {
    const int ks = warps_for(p.N, p.G, num_sms);
    if (path == gemm::kIntScale) {
        if (x_kind == kXCodes) return launch_path<gemm::kIntScale, int8_t>(p, ks, stream);
        if (x_kind == kXBf16) return launch_path<gemm::kIntScale, __nv_bfloat16>(p, ks, stream);
        return launch_path<gemm::kIntScale, float>(p, ks, stream);
    }
    if (x_kind == kXCodes) return launch_path<gemm::kFloatScale, int8_t>(p, ks, stream);
    if (x_kind == kXBf16) return launch_path<gemm::kFloatScale, __nv_bfloat16>(p, ks, stream);
    return launch_path<gemm::kFloatScale, float>(p, ks, stream);
}

}  // namespace gemv
}  // namespace w4a8
