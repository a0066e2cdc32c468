// Setup kernel of a grouped (mixture-of-experts) call.  Integer Scale
// summary §5.3 applies the method to Mixtral 8x7B; here every expert's GEMM
// runs in one persistent launch (the tiles of gemm_w4a8.cu in grouped mode),
// and everything the routing decides is read on the device.  This kernel turns
// the device routing offsets into the launch's schedule and builds each
// expert's weight tensor map, so no host round trip sits between a router
// kernel and the GEMM.
//
// Schedule layout (int32, in the caller's workspace): W (steps), W / g,
// W % g, g (CTAs that take ranges), then m_tiles[E+1], first tile[E+1],
// first routed row[E+1].
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm_w4a8.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace gemm {
namespace {

__global__ void __launch_bounds__(256) moe_setup_kernel(const __grid_constant__ CUtensorMap tmpl,
                                                        const int64_t* offsets, const void* const* w_ptrs,
                                                        const void* const* s_ptrs, int32_t E, int64_t R,
                                                        int32_t bt, int32_t n_tiles, int32_t G, int32_t grid,
                                                        int32_t* sched, CUtensorMap* maps, int* status) {
    __shared__ alignas(128) uint8_t smap[8][128];
    __shared__ int bad_s;
    griddep_wait();  // the offsets and pointers may be the previous kernel's output
    int32_t* mt = sched + 4;
    int32_t* tstart = mt + (E + 1);
    int32_t* rstart = tstart + (E + 1);
    if (threadIdx.x == 0) {
        int bad = offsets[0] != 0 || offsets[E] != R;
        int64_t tiles = 0;
        for (int32_t e = 0; e < E && !bad; ++e) {
            const int64_t m = offsets[e + 1] - offsets[e];
            if (m < 0) {
                bad = 1;
                break;
            }
            // an expert with rows needs its weights 16-byte aligned (a TMA base)
            // and its integer scales 2-byte aligned
            if (m > 0 && (w_ptrs[e] == nullptr || s_ptrs[e] == nullptr ||
                          (reinterpret_cast<uintptr_t>(w_ptrs[e]) & 15u) != 0 ||
                          (reinterpret_cast<uintptr_t>(s_ptrs[e]) & 1u) != 0)) {
                bad = 1;
                break;
            }
            const int64_t mte = (m + bt - 1) / bt;
            mt[e] = int32_t(mte);
            tstart[e] = int32_t(tiles);
            rstart[e] = int32_t(offsets[e]);
            tiles += mte * n_tiles;
            if (tiles * G >= (int64_t(1) << 31)) bad = 1;
        }
        if (bad) {
            tiles = 0;
            atomicExch(status, 1);  // W4A8_ERR_INVALID_ARG
        } else {
            mt[E] = 1;
            tstart[E] = int32_t(tiles);
            rstart[E] = int32_t(R);
        }
        // Fewer steps than CTAs: only the first W CTAs take a (one-step)
        // range, so that every CTA between a split tile's first and last
        // contributor is a contributor; the others exit at once.
        const uint32_t W = uint32_t(tiles * G);
        const uint32_t g_eff = W == 0 ? 1u : (W < uint32_t(grid) ? W : uint32_t(grid));
        sched[0] = int32_t(W);
        sched[1] = int32_t(W / g_eff);
        sched[2] = int32_t(W % g_eff);
        sched[3] = int32_t(g_eff);
        bad_s = bad;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (!bad_s) {
        for (int32_t e = warp; e < E; e += 8) {
            if (offsets[e + 1] == offsets[e]) continue;  // no rows: its map is never used

            reinterpret_cast<uint32_t*>(smap[warp])[lane] = reinterpret_cast<const uint32_t*>(&tmpl)[lane];
            __syncwarp();
            if (lane == 0) tensormap_replace_address(smap[warp], w_ptrs[e]);
            __syncwarp();
            tensormap_publish(maps + e, smap[warp]);
            __syncwarp();
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) griddep_launch_dependents();
}

}  // namespace

cudaError_t launch_grouped_setup(const CUtensorMap& tm_w_template, const int64_t* offsets, const void* const* w_ptrs,
                                 const void* const* s_ptrs, int32_t E, int64_t R, int32_t bt, int32_t n_tiles,
                                 int32_t G, int32_t grid, int32_t* sched, CUtensorMap* maps, int* status,
                                 cudaStream_t stream) {
    const LaunchPdl lc(1u, 256, 0, stream);
    return cudaLaunchKernelEx(&lc.cfg, moe_setup_kernel, tm_w_template, offsets, w_ptrs, s_ptrs, E, R, bt, n_tiles, G,
                              grid, sched, maps, status);
}

}  // namespace gemm
}  // namespace w4a8
