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
    const uint8_t* wq;   // [N, K/2] packed codes, read when a scale of 17 or 18 may be folded (null: never)
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
    long long wait_limit;  // SM cycles a pipeline or split-tile wait may last before it gives up
};

// Parameters of the kernels for asymmetric token codes (a separate type, so
// that the other kernels' parameter block stays as it is)
struct ParamsZp : Params {
    const int32_t* z_a;  // [M] token zero points
    const int32_t* zc;   // [N] zero-point term zc[n] = sum_g S[g,n] sum_{k in g} q[k,n]
};

// Parameters of a grouped (mixture-of-experts) call on the tiles of
// gemm_w4a8.cu: the token rows are routed-order codes (row i = routed row i),
// the partition and the per-expert schedule come from the workspace.
struct ParamsGr : Params {
    const int32_t* grp_sched;       // W, W / g, W % g, g, then m_tiles[E+1], first tile[E+1], first row[E+1]
    const CUtensorMap* grp_maps;    // [E] weight tensor maps (built by the setup kernel)
    const void* const* grp_scales;  // [E] device pointers to each expert's S [G, N]
    const int32_t* out_row;         // [R] output row of each routed row, or null (row i)
    const int32_t* row_index;       // [R] token of each routed row (rows gathered from q_x), or null (row i of q_x)
    int64_t y_rows;                 // rows of y: an output row must lie below it
    int32_t E;
    int32_t n_tiles;
    int32_t T;                      // rows of q_x / s_a: a token index must lie in [0, T)
};


}  // namespace gemm

namespace gemv {
// Decode-shaped layers on the CUDA cores (gemv_w4a8.cu): M <= 4 tokens,
// K <= kMaxK, one CTA per 32 output columns, K split over its warps.
constexpr int kMaxM = 4;
constexpr int kMinK = 256;
constexpr int kMaxK = 16384;
#ifndef W4A8_GEMV_BOX_M4
#define W4A8_GEMV_BOX_M4 64
#endif
// The weight box of the kernel for M tokens: box_bytes(M) x 32 rows (two
// 128-wide K blocks per box for one or two tokens; for three or four, where
// the kernel does four times the arithmetic per byte, the smaller box lets
// more warps share the SM).
constexpr int box_bytes(int M, bool w8 = false) { return (M <= 2 || w8) ? 128 : W4A8_GEMV_BOX_M4; }
enum XKind { kXCodes = 0, kXBf16 = 1, kXF32 = 2 };

struct GemvParams {
    const void* x;         // int8 codes [M][K] (kXCodes) or bf16 / fp32 tokens [M][ldx] (quantized here)
    const float* s_a;      // [M] token scales (kXCodes)
    int64_t ldx;           // row pitch of x in elements (bf16 / fp32 tokens)
    const uint8_t* w;      // packed int4 weights [N][K/2] (or 8-bit codes [N][K])
    const int16_t* S;      // [G][N] integer scales (integer-scale path)
    const float* s_g;      // [G][N] float scales (float-scale path)
    void* y;               // [M][N]
    int32_t y_dtype;       // gemm::OutType
    int32_t M, N, K, G, group;
    float inv_alpha;       // 1 / alpha (integer-scale path)
    int8_t* q_out;         // optional: the codes the kernel computed [M][K] (fused tokens)
    float* s_out;          // optional: their scales [M]
    int* status;           // device status word (a ring wait that runs out)
    long long wait_limit;  // SM cycles a ring wait may last
    int32_t stages;        // ring slots per warp (set by the launcher)
    const int32_t* z_a;    // asymmetric token codes: [M] zero points (with zc; integer-scale path), or null
    const int32_t* zc;     // [N] zero-point term of each column
};

int smem_bytes(int mt, int K, int ks, int stages, int sub);
// tm_w: packed weights [N][K/2] u8, box box_bytes(M) x 32 rows, swizzled by the box width
cudaError_t launch(const CUtensorMap& tm_w, const GemvParams& p, int path, int x_kind, int num_sms,
                   cudaStream_t stream);
// 8-bit weight codes (the W8A8 variant, integer scale, int8 token codes):
// tm_w: w8 [N][K] int8, box 128 B x 32 rows, 128-byte swizzle
cudaError_t launch_w8(const CUtensorMap& tm_w, const GemvParams& p, int num_sms, cudaStream_t stream);
}  // namespace gemv

namespace gemm {

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

// A grouped call on the tiles of gemm_w4a8.cu (token tile 128): the setup
// kernel, then the GEMM, chained with programmatic dependent launch.
// tm_w_template: a packed-weight map of the tiles' box (128 rows x 128 B,
// 128-byte swizzle) whose address the setup kernel replaces per expert;
// tm_x: the codes [T][K], box 128 B x 128 rows (routed-order codes) or
// 128 B x 1 row (rows gathered by p.row_index, four per copy).
cudaError_t launch_grouped(const CUtensorMap& tm_w_template, const CUtensorMap& tm_x, const int64_t* offsets,
                           const void* const* w_ptrs, int64_t R, const ParamsGr& p, int32_t* sched,
                           CUtensorMap* maps, cudaStream_t stream);
// The setup kernel of a grouped call (grouped_setup.cu), for token tiles of `bt`.
cudaError_t launch_grouped_setup(const CUtensorMap& tm_w_template, const int64_t* offsets, const void* const* w_ptrs,
                                 const void* const* s_ptrs, int32_t E, int64_t R, int32_t bt, int32_t n_tiles,
                                 int32_t G, int32_t grid, int32_t* sched, CUtensorMap* maps, int* status,
                                 cudaStream_t stream);

int token_tile_rows();

// Bytes per row of one packed-weight TMA box (one pipeline stage of K).
int weight_box_bytes();

}  // namespace gemm
}  // namespace w4a8
