// Routed-row gather of the mixture-of-experts path.
//
// The Integer Scale summary applies the method to Mixtral 8x7B (§5.3): every
// expert's linear layer is a fine-grained W4A8 GEMM with integer scales.  A
// token's int8 codes and scale do not depend on the expert, so tokens are
// quantized once; this kernel copies the routed rows (a token appears once per
// expert it is routed to) into expert-contiguous rows of codes and scales, the
// operands of one integer-scale GEMM per expert.
//
// Grid: blockIdx.y = expert, blockIdx.x strides over the expert's rows; each
// CTA copies a whole row of K codes with 16-byte loads and stores (HBM-bound:
// K + 4 bytes read and written per routed row).  A routed row whose token
// index is out of range is written as zeros and reported in the device status
// word (W4A8_ERR_INVALID_ARG).
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace moe {

constexpr int kThreads = 256;
constexpr int kStatusInvalidArg = 1;  // mirrors W4A8_ERR_INVALID_ARG

__global__ void __launch_bounds__(kThreads) gather_rows_kernel(const __grid_constant__ GatherParams p) {
    if (threadIdx.x == 0) griddep_launch_dependents();
    griddep_wait();  // q_x and s_a may be the previous kernel's output, the gathered rows its input
    const int e = blockIdx.y;
    const int lo = p.off[e], hi = p.off[e + 1];
    const int64_t chunks = p.K / 16;
    for (int i = lo + int(blockIdx.x); i < hi; i += int(gridDim.x)) {
        const int t = p.row_index[i];
        const bool ok = t >= 0 && int64_t(t) < p.T;
        if (!ok && threadIdx.x == 0) atomicExch(p.status, kStatusInvalidArg);
        uint4* dst = reinterpret_cast<uint4*>(p.xg + int64_t(i) * p.K);
        if (ok) {
            const uint4* src = reinterpret_cast<const uint4*>(p.q_x + int64_t(t) * p.K);
            for (int64_t c = threadIdx.x; c < chunks; c += kThreads) dst[c] = src[c];
        } else {
            for (int64_t c = threadIdx.x; c < chunks; c += kThreads) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (threadIdx.x == 0) p.sg[p.sbase[e] + (i - lo)] = ok ? p.s_a[t] : 0.0f;
    }
}

cudaError_t gather(const GatherParams& p, int max_rows, cudaStream_t stream) {
    const unsigned bx = unsigned(max_rows < 64 ? (max_rows < 1 ? 1 : max_rows) : 64);
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1]{};
    cfg.gridDim = dim3(bx, unsigned(p.E));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gather_rows_kernel, p);
}

}  // namespace moe
}  // namespace w4a8
