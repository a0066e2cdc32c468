// Tensor-pipe throughput probe: back-to-back tcgen05.mma.kind::i8 on operands
// resident on chip, with no loads, no epilogue and nothing else on the SM.
// It measures the int8 tensor rate a GEMM on this GPU can at best reach, the
// denominator of the large-M roofline fraction.
//
// One CTA per SM.  Each CTA fills its operands once (the weight-side operand
// A either in shared memory, 128 rows x 128 bytes in the 128-byte-swizzled
// K-major layout, or in TMEM like the GEMM's unpacked weights; the token-side
// operand B, n rows x 128 bytes, in shared memory), then one elected thread
// issues `iters` x 4 MMAs of shape 128 x n x 32 into one TMEM accumulator and
// commits them to an mbarrier that the CTA waits on (bounded).  int8 ops per
// launch: 2 * 128 * n * 128 * iters * grid.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace peak {

constexpr int kThreads = 128;
constexpr int kABytes = 128 * 128;         // 128 rows x 128 B (one K = 128 block)
constexpr int kBMaxBytes = 256 * 128;      // up to 256 rows x 128 B
constexpr int kSmemBytes = kABytes + kBMaxBytes + 1024;

__global__ void __launch_bounds__(kThreads, 1)
    i8_mma_peak_kernel(int64_t iters, int n, int a_in_tmem, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t done;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // operands: a fixed pseudo-random byte pattern (nonzero, so that the
    // tensor pipe sees ordinary data)
    uint32_t* words = reinterpret_cast<uint32_t*>(smem);
    for (int i = threadIdx.x; i < (kABytes + kBMaxBytes) / 4; i += kThreads) {
        uint32_t h = uint32_t(i) * 2654435761u + 0x9e3779b9u;
        h ^= h >> 15;
        words[i] = h * 2246822519u;
    }
    if (threadIdx.x == 0) {
        mbar_init(&done, 1);
        abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_base_s, 512);
    fence_proxy_async_smem();  // generic-proxy writes of the operands, visible to the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const uint32_t a_tmem = tmem;            // columns [0, 32): A, 4 int8 K values per column
    const uint32_t d_tmem = tmem + 256;      // columns [256, 256 + n): the accumulator

    if (a_in_tmem) {
        // every warp writes its 32 lanes of A: 32 columns (K = 128) per lane
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) r[c] = words[(warp * 32 + lane) * 32 + c];
        tmem_st32(a_tmem + (uint32_t(warp * 32) << 16), r);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(128 >> 4) << 24);
        const uint32_t a_lo = smem_desc_sw128_lo(smem_u32(smem));
        const uint32_t b_lo = smem_desc_sw128_lo(smem_u32(smem + kABytes));
        for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t acc = (it > 0 || k > 0) ? 1u : 0u;
                if (a_in_tmem)
                    mma_i8_tmem_a_one(d_tmem, a_tmem + uint32_t(8 * k), smem_desc_from_lo(b_lo + 2u * k), idesc, acc);
                else
                    mma_i8_ss_one(d_tmem, smem_desc_from_lo(a_lo + 2u * k), smem_desc_from_lo(b_lo + 2u * k), idesc,
                                  acc);
            }
        }
        mma_commit_one(&done);
        __syncwarp();
    }
    // every thread waits for the MMAs (bounded) before TMEM is released
    if (!mbar_wait(&done, 0, &abort_s, status)) {
        // timed out: still wait for the MMAs in flight before freeing TMEM
        const long long t0 = clock64();
        while (!mbar_try_wait(&done, 0) && clock64() - t0 < kWaitLimitCycles) {
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

cudaError_t launch(int64_t iters, int n, bool a_in_tmem, int grid, int* status, cudaStream_t stream) {
    const cudaError_t e = configure_once<i8_mma_peak_kernel>(kThreads, kSmemBytes);
    if (e != cudaSuccess) return e;
    i8_mma_peak_kernel<<<grid, kThreads, kSmemBytes, stream>>>(iters, n, a_in_tmem ? 1 : 0, status);
    return cudaGetLastError();
}

}  // namespace peak
}  // namespace w4a8
