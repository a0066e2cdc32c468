// Host/device interface of the W4A8 GEMM kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace w4a8 {
namespace gemm {

enum Path { kIntScale = 0, kFloatScale = 1 };
enum OutType { kOutF32 = 0, kOutF16 = 1, kOutI32 = 3 };

struct Params {
    const float* s_a;    // [M] token scales
    const int16_t* S;    // [G, N] integer group scales (integer-scale path)
    const float* s_g;    // [G, N] float group scales (float-scale path)
    void* y;             // [M, N] output
    int32_t* ws_part;    // [grid][128 * BT] partial sums of split tiles (one per contributing CTA)
    int32_t* ws_count;   // [grid] arrival counters (index: first contributing CTA), zero between calls
    int* status;         // device status word for timeouts
    int64_t M, N;
    int64_t G;           // groups along K
    int32_t kb_per_group;  // 128-wide K blocks per group
    int64_t m_tiles;
    int64_t W;           // total (tile, group) steps, < 2^31
    int64_t grid;        // CTAs
    uint32_t w_q, w_r;   // W / grid, W % grid
    float inv_alpha;     // 1 / alpha (exact, alpha is a power of two)
    int32_t y_dtype;     // OutType
};

// Parameters of the kernels for asymmetric token codes (a separate type, so
// that the other kernels' parameter block stays as it is)
struct ParamsZp : Params {
    const int32_t* z_a;  // [M] token zero points
    const int32_t* zc;   // [N] zero-point term zc[n] = sum_g S[g,n] sum_{k in g} q[k,n]
};

struct Plan {
    int BT;              // tokens per tile (MMA N)
    int64_t n_tiles, m_tiles, tiles, G, W, grid;
    int64_t count_bytes;  // bytes of the fixed counter region at the start of the workspace
    int64_t ws_bytes;     // total workspace bytes
};

// w8: int8 weight codes (the W8A8 variant); its CTAs run one per SM
Plan make_plan(int64_t M, int64_t N, int64_t K, int32_t group, int num_sms, bool w8 = false);

// tm_w: packed weights [N][K/2] u8, box 128 B x 128 rows, 128-byte swizzle
// tm_x: token codes [M][K] u8, box 128 B x BT rows, 128-byte swizzle
// tm_y: output y [M][N] (f16, f32 or i32 as Params::y_dtype), box 128 columns x BT rows
// The group scales are read through Params::S / Params::s_g.
// w8: tm_w covers int8 weights w8 [N][K] (box 128 B x 128 rows, 128-byte swizzle); integer-scale path only
cudaError_t launch(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const CUtensorMap& tm_y, const Params& p, int BT,
                   int path, cudaStream_t stream, bool w8 = false);
// asymmetric token codes (zero points p.z_a, weight-side term p.zc): the
// integer-scale path with int4 weights
cudaError_t launch_zp(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const CUtensorMap& tm_y, const ParamsZp& p,
                      int BT, cudaStream_t stream);

int token_tile_rows();

// Bytes per row of one packed-weight TMA box (one pipeline stage of K).
int weight_box_bytes();

}  // namespace gemm
}  // namespace w4a8
