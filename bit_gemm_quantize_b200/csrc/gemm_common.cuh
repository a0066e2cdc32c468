// Device helpers shared by the GEMM kernels: int4 -> int8 unpack, TMEM
// loads, named barriers, bounded waits, GPU-scope counters, ring indices.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace w4a8 {
namespace gemm {

// int4 two's-complement nibbles -> int8, 8 values per 32-bit word.  Byte j
// of the word holds K position j (low nibble) and j + 4 (high nibble), so the
// low nibbles give output word 0 (K 0..3) and the high nibbles word 1 (K 4..7)
// in MMA order with no byte permute.
// Exact: per byte ((v ^ 8) + 0x78) ^ 0x80 maps nibble v to its sign-extended
// byte without carries between bytes.
__device__ __forceinline__ uint2 unpack_int4x8(uint32_t w) {
    uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
    uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
    lo = (lo + 0x78787878u) ^ 0x80808080u;
    hi = (hi + 0x78787878u) ^ 0x80808080u;
    return make_uint2(lo, hi);
}

// Scaled: each nibble lands in the high half of its byte, which read as int8
// is 16 * q exactly.
__device__ __forceinline__ uint2 unpack_int4x8_x16(uint32_t w) {
    return make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
}

template <bool X16>
__device__ __forceinline__ uint2 unpack8(uint32_t w) {
    if constexpr (X16)
        return unpack_int4x8_x16(w);
    else
        return unpack_int4x8(w);
}

__device__ __forceinline__ void epi_bar_sync(int threads) {
    asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 8) {
        tmem_ld8(taddr, r);
    } else if constexpr (N == 16) {
        tmem_ld16(taddr, r);
    } else {
        static_assert(N % 32 == 0, "columns per load");
#pragma unroll
        for (int i = 0; i < N / 32; ++i)
            tmem_ld32(taddr + uint32_t(32 * i), *reinterpret_cast<uint32_t(*)[32]>(&r[32 * i]));
    }
}

// Bounded wait without the abort short-cut, for draining copies in flight.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) break;
    }
}

// Acquire load at GPU scope (the arrival counter of a split tile).
__device__ __forceinline__ int ld_acquire_gpu(const int* addr) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
    return v;
}

// Release add at GPU scope: the CTA's writes ordered before it (by a CTA
// barrier) become visible to a thread that acquires the counter.
__device__ __forceinline__ void red_release_gpu_add(int* addr, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

struct Ring {
    int idx = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void advance(int n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

}  // namespace gemm
}  // namespace w4a8
