// Per-token symmetric int8 activation quantization for sm_100a.
//
// "Quantization" notes, Symmetric Quantization: s = max|x| / 127, z = 0,
// q = clip(round(x / s), -127, 127); 探秘Transformer系列之（34）量化基礎
// §2.3.3 (one scale per token row).  round() is half to even and x / s is one
// IEEE fp32 division, so codes match a plain CPU evaluation bit for bit.
//
// HBM-bound: every input byte is read once and every code written once.
// A persistent grid (SMs x resident CTAs) walks the rows; each CTA stages one
// row in shared memory with a bulk async copy while it quantizes the previous
// row (two buffers), reduces |x| with warp shuffles, and writes the codes with
// 16-byte stores.  Rows too long for two shared-memory buffers take a second
// kernel that re-reads the row (from L2) instead of staging it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "kernels.h"
#include "quant_common.cuh"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace quant {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r = fmaxf(r, red[w]);
    return r;
}

template <typename T>
__device__ __forceinline__ void quantize_row(const T* row, int64_t K, float s, int8_t* qrow) {
    const bool zero = (s == 0.0f);
    const bool exact_only = s < 1e-30f;
    const float rcp = zero ? 0.0f : __frcp_rn(s);
    for (int64_t c = threadIdx.x; c < K / 16; c += kThreads) {
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
        if (!zero) {
            float v[16];
            load16<T>(row + c * 16, v);
            uint32_t cb[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) cb[i] = code_i8_byte(v[i], s, rcp, exact_only);
#pragma unroll
            for (int w = 0; w < 4; ++w)
                packed[w] = pack4_low_bytes(cb[4 * w], cb[4 * w + 1], cb[4 * w + 2], cb[4 * w + 3]);
        }
        *reinterpret_cast<uint4*>(qrow + c * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

template <typename T>
__device__ __forceinline__ float row_absmax(const T* row, int64_t K, float* red) {
    float a = 0.0f;
    for (int64_t c = threadIdx.x; c < K / 16; c += kThreads) {
        float v[16];
        load16<T>(row + c * 16, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
    }
    return block_max(a, red);
}

// Source row of output row `row`: the row itself, or rows[row] when the
// caller routes rows (then `ok` says whether it lies in [0, T_src); an
// invalid source reads row 0 and its outputs are zeroed).
__device__ __forceinline__ int64_t source_row(const int32_t* rows, int64_t row, int64_t T_src, bool& ok) {
    if (rows == nullptr) {
        ok = true;
        return row;
    }
    const int64_t t = rows[row];
    ok = t >= 0 && t < T_src;
    return ok ? t : 0;
}

// Row staged in shared memory by a bulk async copy; two buffers.
template <typename T>
__global__ void __launch_bounds__(kThreads) quant_rows_staged(const T* __restrict__ x, int64_t M, int64_t K,
                                                              int64_t ldx, int8_t* __restrict__ q,
                                                              float* __restrict__ s_a, int* status,
                                                              const int32_t* __restrict__ rows, int64_t T_src) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t row_bytes = uint32_t(K * sizeof(T));
    const uint32_t buf_bytes = (row_bytes + 127u) & ~127u;
    T* buf[2] = {reinterpret_cast<T*>(smem), reinterpret_cast<T*>(smem + buf_bytes)};
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * buf_bytes);
    float* red = reinterpret_cast<float*>(bars + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(red + kWarps);

    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
        griddep_launch_dependents();
    }
    // x may be the previous kernel's output, q and s_a its input
    griddep_wait();
    __syncthreads();

    int64_t row = blockIdx.x;
    bool inflight[2] = {false, false};  // meaningful in thread 0, which issues the copies
    bool ok_src = true;
    if (threadIdx.x == 0 && row < M) {
        const int64_t src = source_row(rows, row, T_src, ok_src);
        mbar_arrive_expect_tx(&bars[0], row_bytes);
        bulk_load(buf[0], x + src * ldx, row_bytes, &bars[0]);
        inflight[0] = true;
    }
    uint32_t phase[2] = {0u, 0u};
    int st = 0;
    for (; row < M; row += gridDim.x) {
        const int64_t next = row + gridDim.x;
        if (threadIdx.x == 0 && next < M) {  // prefetch the next row into the other buffer
            const int64_t src = source_row(rows, next, T_src, ok_src);
            mbar_arrive_expect_tx(&bars[st ^ 1], row_bytes);
            bulk_load(buf[st ^ 1], x + src * ldx, row_bytes, &bars[st ^ 1]);
            inflight[st ^ 1] = true;
        }
        if (!mbar_wait(&bars[st], phase[st], abort_flag, status)) break;
        inflight[st] = false;
        phase[st] ^= 1u;
        source_row(rows, row, T_src, ok_src);
        const float a = row_absmax<T>(buf[st], K, red);
        const float s = (a == 0.0f || !ok_src) ? 0.0f : __fdiv_rn(a, 127.0f);
        if (threadIdx.x == 0) {
            s_a[row] = s;
            if (!ok_src) atomicExch(status, kStatusInvalidArg);
        }
        quantize_row<T>(buf[st], K, s, q + row * K);
        __syncthreads();  // buffer and reduction scratch are free again
        st ^= 1;
    }
    // after a timeout, let copies in flight land before leaving
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            if (!inflight[b]) continue;
            const long long t0 = clock64();
            while (!mbar_try_wait(&bars[b], phase[b]) && clock64() - t0 < kWaitLimitCycles) {
            }
        }
    }
}

// Long rows: read the row twice from global memory (the second pass hits L2).
template <typename T>
__global__ void __launch_bounds__(kThreads) quant_rows_direct(const T* __restrict__ x, int64_t M, int64_t K,
                                                              int64_t ldx, int8_t* __restrict__ q,
                                                              float* __restrict__ s_a, int* status,
                                                              const int32_t* __restrict__ rows, int64_t T_src) {
    __shared__ float red[kWarps];
    if (threadIdx.x == 0) griddep_launch_dependents();
    griddep_wait();  // x may be the previous kernel's output, q and s_a its input
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
        bool ok_src = true;
        const T* r = x + source_row(rows, row, T_src, ok_src) * ldx;
        const float a = row_absmax<T>(r, K, red);
        const float s = (a == 0.0f || !ok_src) ? 0.0f : __fdiv_rn(a, 127.0f);
        if (threadIdx.x == 0) {
            s_a[row] = s;
            if (!ok_src) atomicExch(status, kStatusInvalidArg);
        }
        quantize_row<T>(r, K, s, q + row * K);
        __syncthreads();
    }
}

// ---- asymmetric codes ("Quantization" notes, Asymmetric Quantization): the
// row's range [x_min, x_max] maps onto the int8 codes [-128, 127]:
// s = (x_max - x_min) / 255, z = clip(rne(-128 - x_min / s), -128, 127),
// q = clip(rne(x / s) + z, -128, 127).  Each step is one IEEE fp32 operation
// (true division), so the codes match a plain CPU evaluation bit for bit.  A
// constant row's empty range is widened to include zero; a row whose scale is
// 0 gets z = 0 and codes 0.  Inputs are finite.  Two passes over the row (the
// second from L2): the min / max reduction, then the codes.

__device__ __forceinline__ void block_minmax(float& lo, float& hi, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        red[warp] = lo;
        red[kWarps + warp] = hi;
    }
    __syncthreads();
    lo = red[0];
    hi = red[kWarps];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        lo = fminf(lo, red[w]);
        hi = fmaxf(hi, red[kWarps + w]);
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) quant_rows_asym(const T* __restrict__ x, int64_t M, int64_t K,
                                                            int64_t ldx, int8_t* __restrict__ q,
                                                            float* __restrict__ s_a, int32_t* __restrict__ z_a) {
    __shared__ float red[2 * kWarps];
    if (threadIdx.x == 0) griddep_launch_dependents();
    griddep_wait();  // x may be the previous kernel's output, q, s_a and z_a its input
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
        const T* r = x + row * ldx;
        float lo = INFINITY, hi = -INFINITY;
        for (int64_t c = threadIdx.x; c < K / 16; c += kThreads) {
            float v[16];
            load16<T>(r + c * 16, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                lo = fminf(lo, v[i]);
                hi = fmaxf(hi, v[i]);
            }
        }
        block_minmax(lo, hi, red);
        if (hi == lo) {  // empty range: widen it to include zero
            lo = fminf(lo, 0.0f);
            hi = fmaxf(hi, 0.0f);
        }
        const float s = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
        const bool zero = (s == 0.0f);
        const float zf = zero ? 0.0f : fminf(fmaxf(rintf(__fsub_rn(-128.0f, __fdiv_rn(lo, s))), -128.0f), 127.0f);
        if (threadIdx.x == 0) {
            s_a[row] = s;
            z_a[row] = int32_t(zf);
        }
        int8_t* qrow = q + row * K;
        for (int64_t c = threadIdx.x; c < K / 16; c += kThreads) {
            uint32_t packed[4] = {0u, 0u, 0u, 0u};
            if (!zero) {
                float v[16];
                load16<T>(r + c * 16, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    // rne(x / s) + z is exact below 2^24; above it the clip decides alone
                    const float t = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(v[i], s)), zf), -128.0f), 127.0f);
                    packed[i >> 2] |= (uint32_t(int(t)) & 0xFFu) << (8 * (i & 3));
                }
            }
            *reinterpret_cast<uint4*>(qrow + c * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        __syncthreads();  // the reduction scratch is free again
    }
}

constexpr size_t kMaxStagedSmem = 200 * 1024;

// Resident CTAs per SM of the staged kernel for a given shared-memory size,
// with the shared-memory opt-in set once per device and kernel; cached.
template <typename K>
static cudaError_t staged_blocks_per_sm(K kern, size_t smem, int* per_sm) {
    struct Entry {
        int dev;
        size_t smem;
        int blocks;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& c : cache)
        if (c.dev == dev && c.smem == smem) {
            *per_sm = c.blocks;
            return cudaSuccess;
        }
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kMaxStagedSmem + 1024));
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = true;
    }
    int blocks = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (blocks < 1) blocks = 1;
    if (cache.size() < 256) cache.push_back({dev, smem, blocks});
    *per_sm = blocks;
    return cudaSuccess;
}

template <typename T>
static cudaError_t launch_t(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* s_a, int* status,
                            cudaStream_t stream, int num_sms, const int32_t* rows, int64_t T_src) {
    const uint32_t row_bytes = uint32_t(K * sizeof(T));
    const uint32_t buf_bytes = (row_bytes + 127u) & ~127u;
    const size_t smem = 2 * size_t(buf_bytes) + 2 * sizeof(uint64_t) + kWarps * sizeof(float) + 16;
    if (smem <= kMaxStagedSmem) {
        auto kern = quant_rows_staged<T>;
        int per_sm = 0;
        cudaError_t e = staged_blocks_per_sm(kern, smem, &per_sm);
        if (e != cudaSuccess) return e;
        const int64_t grid = M < int64_t(num_sms) * per_sm ? M : int64_t(num_sms) * per_sm;
        const LaunchPdl lc(unsigned(grid), kThreads, smem, stream);
        return cudaLaunchKernelEx(&lc.cfg, kern, x, M, K, ldx, q, s_a, status, rows, T_src);
    }
    auto kern = quant_rows_direct<T>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int64_t grid = M < int64_t(num_sms) * per_sm ? M : int64_t(num_sms) * per_sm;
    const LaunchPdl lc(unsigned(grid), kThreads, 0, stream);
    return cudaLaunchKernelEx(&lc.cfg, kern, x, M, K, ldx, q, s_a, status, rows, T_src);
}

cudaError_t launch(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* s_a,
                   int* status, cudaStream_t stream, int num_sms, const int32_t* rows, int64_t T_src) {
    if (bf16)
        return launch_t<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), M, K, ldx, q, s_a, status, stream,
                                       num_sms, rows, T_src);
    return launch_t<float>(static_cast<const float*>(x), M, K, ldx, q, s_a, status, stream, num_sms, rows, T_src);
}

cudaError_t launch_asym(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* s_a,
                        int32_t* z_a, cudaStream_t stream, int num_sms) {
    int per_sm = 0;
    cudaError_t e = bf16 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_rows_asym<__nv_bfloat16>,
                                                                         kThreads, 0)
                         : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_rows_asym<float>, kThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int64_t grid = M < int64_t(num_sms) * per_sm ? M : int64_t(num_sms) * per_sm;
    const LaunchPdl lc(unsigned(grid), kThreads, 0, stream);
    if (bf16)
        return cudaLaunchKernelEx(&lc.cfg, quant_rows_asym<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(x), M,
                                  K, ldx, q, s_a, z_a);
    return cudaLaunchKernelEx(&lc.cfg, quant_rows_asym<float>, static_cast<const float*>(x), M, K, ldx, q, s_a, z_a);
}

}  // namespace quant
}  // namespace w4a8
