// Internal launch entry points of the library's kernels (host side).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace w4a8 {

// The dynamic shared-memory opt-in of a kernel is a per-device function
// attribute: set it (and check that one CTA fits) once per (kernel, device),
// the first time the kernel is launched on the device.  Thread-safe; later
// launches only read the recorded result.  The kernel is a template argument,
// so every kernel has flags of its own.
template <auto kern>
cudaError_t configure_once(int threads, int smem) {
    constexpr int kDevs = 64;
    static std::once_flag once[kDevs];
    static cudaError_t result[kDevs];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kDevs) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        int resident = 0;
        if (r == cudaSuccess) r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kern, threads, smem);
        if (r == cudaSuccess && resident < 1) r = cudaErrorLaunchOutOfResources;
        result[dev] = r;
    });
    return result[dev];
}

// Launch configuration with programmatic stream serialization: the kernel
// may start while the previous kernel in the stream is still running; it
// orders its own accesses with griddepcontrol.wait (see sm100_ptx.cuh).
struct LaunchPdl {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1]{};
    LaunchPdl(unsigned grid, unsigned threads, size_t smem, cudaStream_t stream) {
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(threads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    LaunchPdl(const LaunchPdl&) = delete;
    LaunchPdl& operator=(const LaunchPdl&) = delete;
};

namespace quant {
// rows: NULL (row m of x gives row m of q) or [M] source rows (row m of q is
// row rows[m] of x, which has T_src rows; a source outside [0, T_src) gives
// zero codes and scale and sets W4A8_ERR_INVALID_ARG in *status)
cudaError_t launch(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* s_a,
                   int* status, cudaStream_t stream, int num_sms, const int32_t* rows = nullptr, int64_t T_src = 0);
// asymmetric codes in [-128, 127] with a zero point z_a[m] per row
cudaError_t launch_asym(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, int8_t* q, float* s_a,
                        int32_t* z_a, cudaStream_t stream, int num_sms);
}


namespace peak {
// Back-to-back int8 MMAs (128 x n x 32, n % 16 == 0, 16 <= n <= 256) on
// on-chip operands, iters x 4 per CTA, one CTA per SM of `grid`.
cudaError_t launch(int64_t iters, int n, bool a_in_tmem, int grid, int* status, cudaStream_t stream);
}  // namespace peak

namespace pack {
// Layout of the pack workspace (device bytes).
struct Results {
    int32_t alpha;         // chosen amplifier
    int32_t error;         // nonzero: no power of two up to 2^30 suffices
    float s_min_pos;       // smallest positive scale (+inf when none)
    float s_max;           // largest scale
    unsigned long long colsum_max;  // max_n sum_g |S[g,n]|
};
constexpr int64_t kPartialsOffset = 256;  // per-block (min, max) pairs start here
constexpr int kMaxPartialBlocks = 4096;

// qmin: the lowest code, -7 (codes [-7, 7], s = max|w| / 7) or -8 (codes
// [-8, 7], s = max|w| / 8)
cudaError_t group_scales(const float* w, int64_t K, int64_t N, int32_t group, int32_t qmin, float* s_g,
                         cudaStream_t stream);
// s_g = fl32(max|w| / qdiv) for any divisor (127 for 8-bit weight codes)
cudaError_t group_scales_div(const float* w, int64_t K, int64_t N, int32_t group, float qdiv, float* s_g,
                             cudaStream_t stream);
// min / max reduction + amplifier search (alpha_in > 0: fixed amplifier)
cudaError_t amplifier(const float* scales, int64_t count, int32_t alpha_in, void* workspace,
                      cudaStream_t stream, int num_sms);
cudaError_t quantize_pack(const float* w, const float* s_g, int32_t alpha, int64_t K, int64_t N, int32_t group,
                          int32_t qmin, uint8_t* packed, int16_t* S, void* workspace, cudaStream_t stream);
// 8-bit codes clip(rne(w / s_g), -127, 127) stored as w8 [N, K] int8, and S
cudaError_t quantize_w8(const float* w, const float* s_g, int32_t alpha, int64_t K, int64_t N, int32_t group,
                        int8_t* w8, int16_t* S, void* workspace, cudaStream_t stream);
// zc[n] = sum_g S[g,n] * sum_{k in g} q[k,n] from the packed int4 codes (the
// weight-side zero-point term of an asymmetric activation)
cudaError_t zero_point_term(const uint8_t* packed, const int16_t* S, int64_t K, int64_t N, int32_t group,
                            int32_t* zc, cudaStream_t stream, int num_sms);
}  // namespace pack

}  // namespace w4a8
