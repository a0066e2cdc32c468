// C ABI of the library: argument checks on the host, tensor maps, launches.
// The operations and their sources are documented in include/w4a8_intscale.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "w4a8_intscale.h"
#include "gemm_w4a8.h"
#include "kernels.h"

namespace {

// One status word per device that loads the library; bounded waits that run
// out write W4A8_ERR_TIMEOUT into it.
__device__ int g_status_word;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int* status = nullptr;
};

DeviceInfo g_devices[kMaxDevices];
std::mutex g_devices_mutex;

// Workspace of w4a8_gemm_intscale_static_ws: one fixed array per device,
// shared by every call of that entry point on the device.  Its first 4096
// bytes are the split-tile arrival counters, zero at module load (device
// globals without an initializer are zero-filled) and left zero by every
// call that completes; the rest holds partial sums and needs no clearing.
__device__ __align__(256) uint8_t g_static_workspace[W4A8_STATIC_WORKSPACE_BYTES];

struct StaticWorkspace {
    bool ready = false;
    void* ptr = nullptr;
};

StaticWorkspace g_static_ws[kMaxDevices];
std::mutex g_static_ws_mutex;

// Device address of the current device's static workspace, looked up once per
// device (the first call on a device does this set-up).
w4a8_status static_workspace(void** out);

// How long (SM cycles) a GEMM's pipeline and split-tile waits may last before
// the kernel gives up with W4A8_ERR_TIMEOUT; w4a8_set_wait_limit changes it.
constexpr long long kDefaultWaitLimit = 1ll << 31;
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

// Last CUDA runtime error seen by this thread's library calls.
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

w4a8_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = e;
    return W4A8_ERR_CUDA;
}

#define W4A8_CUDA_TRY(expr)                           \
    do {                                              \
        const cudaError_t w4a8_e_ = (expr);           \
        if (w4a8_e_ != cudaSuccess) return cuda_fail(w4a8_e_); \
    } while (0)

w4a8_status static_workspace(void** out) {
    int dev = 0;
    W4A8_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return W4A8_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    StaticWorkspace& w = g_static_ws[dev];
    if (!w.ready) {
        W4A8_CUDA_TRY(cudaGetSymbolAddress(&w.ptr, g_static_workspace));
        w.ready = true;
    }
    *out = w.ptr;
    return W4A8_OK;
}

w4a8_status current_device(DeviceInfo& out) {
    int dev = 0;
    W4A8_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return W4A8_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_devices_mutex);
    DeviceInfo& d = g_devices[dev];
    if (!d.ready) {
        W4A8_CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        W4A8_CUDA_TRY(cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_status_word));
        d.ready = true;
    }
    out = d;
    return W4A8_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D tensor map: [rows][cols] elements of `type` with row pitch `pitch` bytes.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType type, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t pitch, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch, uint32_t box_cols,
                 uint32_t box_rows, CUtensorMapSwizzle swz) {
    return make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, cols, rows, pitch, box_cols, box_rows, swz);
}

// Whether the stream-K partition of `pl` cuts any tile (then a workspace is needed).
bool plan_splits_tiles(const w4a8::gemm::Plan& pl) {
    for (int64_t b = 1; b < pl.grid; ++b)
        if ((b * pl.W / pl.grid) % pl.G != 0) return true;
    return false;
}

w4a8_status check_gemm_shape(int64_t M, int64_t N, int64_t K, int32_t group) {
    if (M < 0 || N <= 0 || K <= 0 || group <= 0) return W4A8_ERR_SHAPE;
    if (N % 8 != 0 || K % 128 != 0 || group % 128 != 0 || K % group != 0) return W4A8_ERR_SHAPE;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return W4A8_ERR_SHAPE;
    if ((K / group) * N >= (int64_t(1) << 31)) return W4A8_ERR_SHAPE;  // scale indices are 32-bit
    return W4A8_OK;
}

// Decode-shaped calls (a few tokens) run on the CUDA cores (gemv_w4a8.cu):
// one or two tokens always; three or four while the weights take at most
// 32 MB (measured with 4-bit weights: past that the tensor-core tiles, which
// do a quarter of the instructions per weight byte, are faster at four
// tokens).  8-bit weight codes (w8) take the same kernel without the unpack.
bool gemv_fits(int64_t M, int64_t K, bool w8, bool zp) {
    (void)zp;  // asymmetric token codes: the kernel subtracts z[m] * zc[n] from each accumulator
    (void)w8;
    return M >= 1 && M <= w4a8::gemv::kMaxM && K >= w4a8::gemv::kMinK && K <= w4a8::gemv::kMaxK;
}
bool gemv_path(int64_t M, int64_t N, int64_t K, bool w8, bool zp) {
    return gemv_fits(M, K, w8, zp) && (M <= 2 || N * (w8 ? K : K / 2) <= (int64_t(32) << 20));
}

// The decode kernel's weight map for M tokens: [N][K/2] bytes (4-bit) or
// [N][K] bytes (w8), boxes of 32 rows x box_bytes(M, w8) (one or two 128-wide
// K blocks of 32 columns), swizzled by the box width.
bool gemv_weight_map(CUtensorMap* m, const uint8_t* w_packed, int64_t N, int64_t K, int64_t M, bool w8 = false) {
    const int box = w4a8::gemv::box_bytes(int(M), w8);
    const uint64_t row = uint64_t(w8 ? K : K / 2);
    return make_map_u8(m, w_packed, row, uint64_t(N), row, uint32_t(box), 32,
                       box == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

w4a8_status run_gemm(int path, const int8_t* q_x, const float* s_a, const uint8_t* w_packed, const int16_t* S,
                     const float* s_g, int32_t alpha, int64_t M, int64_t N, int64_t K, int32_t group, void* y,
                     int32_t y_dtype, void* workspace, int64_t workspace_bytes, void* stream, bool w8 = false,
                     const int32_t* z_a = nullptr, const int32_t* zc = nullptr, bool zp = false) {
    w4a8_status st = check_gemm_shape(M, N, K, group);
    if (st != W4A8_OK) return st;
    if (path == w4a8::gemm::kIntScale) {
        if (y_dtype != W4A8_F16 && y_dtype != W4A8_F32 && y_dtype != W4A8_I32) return W4A8_ERR_DTYPE;
        if (!is_pow2(alpha) || alpha > (1 << 30)) return W4A8_ERR_INVALID_ARG;
    } else {
        if (y_dtype != W4A8_F16 && y_dtype != W4A8_F32) return W4A8_ERR_DTYPE;
    }
    if (M == 0) return W4A8_OK;
    if (!q_x || !s_a || !w_packed || !y || (path == w4a8::gemm::kIntScale ? !S : !s_g)) return W4A8_ERR_INVALID_ARG;
    if (zp && (!z_a || !zc)) return W4A8_ERR_INVALID_ARG;
    if (zp && ((reinterpret_cast<uintptr_t>(z_a) | reinterpret_cast<uintptr_t>(zc)) & 3u) != 0) return W4A8_ERR_ALIGN;
    if (!aligned16(q_x) || !aligned16(w_packed) || !aligned16(y) || !aligned16(s_a) ||
        !aligned16(path == w4a8::gemm::kIntScale ? static_cast<const void*>(S) : static_cast<const void*>(s_g)))
        return W4A8_ERR_ALIGN;

    DeviceInfo dev;
    if ((st = current_device(dev)) != W4A8_OK) return st;
    if (gemv_path(M, N, K, w8, zp)) {
        // decode-shaped: the CUDA-core kernel, no workspace
        w4a8::gemv::GemvParams g{};
        g.x = q_x;
        g.s_a = s_a;
        g.w = w_packed;
        g.S = S;
        g.s_g = s_g;
        g.y = y;
        g.y_dtype = y_dtype == W4A8_F16 ? w4a8::gemm::kOutF16
                                        : (y_dtype == W4A8_I32 ? w4a8::gemm::kOutI32 : w4a8::gemm::kOutF32);
        g.M = int32_t(M);
        g.N = int32_t(N);
        g.K = int32_t(K);
        g.G = int32_t(K / group);
        g.group = group;
        g.inv_alpha = path == w4a8::gemm::kIntScale ? std::ldexp(1.0f, -int(std::log2(double(alpha)))) : 1.0f;
        g.status = dev.status;
        g.wait_limit = g_wait_limit.load();
        if (zp) {
            g.z_a = z_a;
            g.zc = zc;
        }
        CUtensorMap tm;
        if (!gemv_weight_map(&tm, w_packed, N, K, M, w8)) return W4A8_ERR_CUDA;
        if (w8)
            W4A8_CUDA_TRY(w4a8::gemv::launch_w8(tm, g, dev.sms, static_cast<cudaStream_t>(stream)));
        else
            W4A8_CUDA_TRY(
                w4a8::gemv::launch(tm, g, path, w4a8::gemv::kXCodes, dev.sms, static_cast<cudaStream_t>(stream)));
        return W4A8_OK;
    }
    const w4a8::gemm::Plan pl = w4a8::gemm::make_plan(M, N, K, group, dev.sms, w8);
    if (pl.W >= (int64_t(1) << 31)) return W4A8_ERR_SHAPE;  // the kernel indexes (tile, group) steps in 32 bits
    int32_t* ws_count = nullptr;
    int32_t* ws_part = nullptr;
    if (plan_splits_tiles(pl)) {
        if (!workspace || workspace_bytes < pl.ws_bytes) return W4A8_ERR_WORKSPACE;
        if (!aligned16(workspace)) return W4A8_ERR_ALIGN;
        ws_count = static_cast<int32_t*>(workspace);
        ws_part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + pl.count_bytes);
    }

    CUtensorMap tm_w, tm_x, tm_y;
    // packed weights: one box = 128 columns x 128 bytes (two 128-wide K blocks), 128-byte swizzle;
    // int8 weights: one box = 128 columns x 128 bytes (one K block)
    if (!make_map_u8(&tm_w, w_packed, uint64_t(w8 ? K : K / 2), uint64_t(N), uint64_t(w8 ? K : K / 2),
                     uint32_t(w4a8::gemm::weight_box_bytes()), 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    if (!make_map_u8(&tm_x, q_x, uint64_t(K), uint64_t(M), uint64_t(K), 128, uint32_t(pl.BT),
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    // output: one box = 128 columns x BT rows, stored from the CTA's staging tile
    {
        const bool f16 = (y_dtype == W4A8_F16);
        const CUtensorMapDataType t = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                          : (y_dtype == W4A8_I32 ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
        if (!make_map_2d(&tm_y, t, y, uint64_t(N), uint64_t(M), uint64_t(N) * (f16 ? 2u : 4u), 128,
                         uint32_t(pl.BT), CU_TENSOR_MAP_SWIZZLE_NONE))
            return W4A8_ERR_CUDA;
    }

    w4a8::gemm::Params p{};
    p.s_a = s_a;
    p.S = S;
    p.wq = w8 ? nullptr : w_packed;
    p.s_g = s_g;
    p.y = y;
    p.ws_part = ws_part;
    p.ws_count = ws_count;
    p.status = dev.status;
    p.M = M;
    p.N = N;
    p.G = pl.G;
    p.kb_per_group = group / 128;
    p.m_tiles = pl.m_tiles;
    p.W = pl.W;
    p.grid = pl.grid;
    p.w_q = uint32_t(pl.W / pl.grid);
    p.w_r = uint32_t(pl.W % pl.grid);
    p.inv_alpha = path == w4a8::gemm::kIntScale ? std::ldexp(1.0f, -int(std::log2(double(alpha)))) : 1.0f;
    p.y_dtype = y_dtype == W4A8_F16 ? w4a8::gemm::kOutF16
                                    : (y_dtype == W4A8_I32 ? w4a8::gemm::kOutI32 : w4a8::gemm::kOutF32);
    p.wait_limit = g_wait_limit.load();
    if (zp) {
        w4a8::gemm::ParamsZp pz{};
        static_cast<w4a8::gemm::Params&>(pz) = p;
        pz.z_a = z_a;
        pz.zc = zc;
        W4A8_CUDA_TRY(w4a8::gemm::launch_zp(tm_w, tm_x, tm_y, pz, pl.BT, static_cast<cudaStream_t>(stream)));
        return W4A8_OK;
    }
    W4A8_CUDA_TRY(w4a8::gemm::launch(tm_w, tm_x, tm_y, p, pl.BT, path, static_cast<cudaStream_t>(stream), w8));
    return W4A8_OK;
}

int64_t align256(int64_t v) { return (v + 255) & ~int64_t(255); }

// Layout of the grouped (mixture-of-experts) workspace: [arrival counters and
// split-tile partials of the tiles] [E weight tensor maps]
// [schedule: W, W / grid, W % grid, status, m_tiles[E+1], first tile[E+1],
// first row[E+1]], every part 256-byte aligned.
struct GroupedLayout {
    int64_t grid = 0, gemm_bytes = 0, maps_off = 0, sched_off = 0, total = 0;
};

GroupedLayout grouped_layout(int32_t E, const DeviceInfo& dev) {
    GroupedLayout L;
    L.grid = dev.sms;
    L.gemm_bytes = 4096 + L.grid * 128 * 128 * 4;  // counters, then one 128 x 128 int32 partial per CTA
    L.maps_off = align256(L.gemm_bytes);
    L.sched_off = L.maps_off + align256(int64_t(E) * 128);
    L.total = L.sched_off + align256((4 + 3 * (int64_t(E) + 1)) * 4);
    return L;
}

}  // namespace

extern "C" {

const char* w4a8_status_string(int32_t status) {
    switch (status) {
        case W4A8_OK: return "ok";
        case W4A8_ERR_INVALID_ARG: return "invalid argument";
        case W4A8_ERR_SHAPE: return "unsupported shape";
        case W4A8_ERR_ALIGN: return "misaligned pointer or leading dimension";
        case W4A8_ERR_DTYPE: return "unsupported dtype";
        case W4A8_ERR_OVERFLOW_BOUND: return "worst-case int32 accumulator bound exceeded";
        case W4A8_ERR_SCALE_RANGE: return "integer scale or amplifier out of range";
        case W4A8_ERR_CUDA: return "CUDA runtime error";
        case W4A8_ERR_TIMEOUT: return "kernel wait timed out";
        case W4A8_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

w4a8_status quantize_act_per_token(const void* x, int32_t x_dtype, int64_t M, int64_t K, int64_t ldx,
                                   int8_t* q_x, float* s_a, void* stream) {
    if (x_dtype != W4A8_F32 && x_dtype != W4A8_BF16) return W4A8_ERR_DTYPE;
    if (M < 0 || K <= 0 || K % 16 != 0 || ldx < K) return W4A8_ERR_SHAPE;
    if (M == 0) return W4A8_OK;
    if (!x || !q_x || !s_a) return W4A8_ERR_INVALID_ARG;
    const int64_t esz = x_dtype == W4A8_BF16 ? 2 : 4;
    if (!aligned16(x) || !aligned16(q_x) || (ldx * esz) % 16 != 0) return W4A8_ERR_ALIGN;
    if (!aligned4(s_a)) return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    W4A8_CUDA_TRY(w4a8::quant::launch(x, x_dtype == W4A8_BF16, M, K, ldx, q_x, s_a, dev.status,
                                      static_cast<cudaStream_t>(stream), dev.sms));
    return W4A8_OK;
}

w4a8_status quantize_act_routed(const void* x, int32_t x_dtype, int64_t T, int64_t K, int64_t ldx,
                                const int32_t* row_index, int64_t R, int8_t* q_r, float* s_r, void* stream) {
    if (x_dtype != W4A8_F32 && x_dtype != W4A8_BF16) return W4A8_ERR_DTYPE;
    if (R < 0 || T < 0 || K <= 0 || K % 16 != 0 || ldx < K) return W4A8_ERR_SHAPE;
    if (R == 0) return W4A8_OK;
    if (T < 1) return W4A8_ERR_SHAPE;
    if (!x || !row_index || !q_r || !s_r) return W4A8_ERR_INVALID_ARG;
    const int64_t esz = x_dtype == W4A8_BF16 ? 2 : 4;
    if (!aligned16(x) || !aligned16(q_r) || (ldx * esz) % 16 != 0) return W4A8_ERR_ALIGN;
    if (!aligned4(s_r) || !aligned4(row_index)) return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    W4A8_CUDA_TRY(w4a8::quant::launch(x, x_dtype == W4A8_BF16, R, K, ldx, q_r, s_r, dev.status,
                                      static_cast<cudaStream_t>(stream), dev.sms, row_index, T));
    return W4A8_OK;
}

w4a8_status quantize_act_per_token_asym(const void* x, int32_t x_dtype, int64_t M, int64_t K, int64_t ldx,
                                        int8_t* q_x, float* s_a, int32_t* z_a, void* stream) {
    if (x_dtype != W4A8_F32 && x_dtype != W4A8_BF16) return W4A8_ERR_DTYPE;
    if (M < 0 || K <= 0 || K % 16 != 0 || ldx < K) return W4A8_ERR_SHAPE;
    if (M == 0) return W4A8_OK;
    if (!x || !q_x || !s_a || !z_a) return W4A8_ERR_INVALID_ARG;
    const int64_t esz = x_dtype == W4A8_BF16 ? 2 : 4;
    if (!aligned16(x) || !aligned16(q_x) || (ldx * esz) % 16 != 0) return W4A8_ERR_ALIGN;
    if (!aligned4(s_a) || !aligned4(z_a)) return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    W4A8_CUDA_TRY(w4a8::quant::launch_asym(x, x_dtype == W4A8_BF16, M, K, ldx, q_x, s_a, z_a,
                                           static_cast<cudaStream_t>(stream), dev.sms));
    return W4A8_OK;
}

w4a8_status w4_zero_point_term(const uint8_t* w_packed, const int16_t* S, int64_t K, int64_t N, int32_t group,
                               int32_t qmin, int64_t colsum_max, int32_t* zc, void* stream) {
    if (K <= 0 || N <= 0 || group <= 0 || group % 32 != 0 || K % group != 0) return W4A8_ERR_SHAPE;
    if (K > INT32_MAX || N > INT32_MAX) return W4A8_ERR_SHAPE;
    if (qmin != -7 && qmin != -8) return W4A8_ERR_INVALID_ARG;
    if (colsum_max < 0) return W4A8_ERR_INVALID_ARG;
    // asymmetric token codes span 255 values: the accumulator of the
    // asymmetric GEMM stays exact only while 255 * |qmin| * group * colsum < 2^31
    if (255.0 * double(-qmin) * double(group) * double(colsum_max) >= 2147483648.0) return W4A8_ERR_OVERFLOW_BOUND;
    if (!w_packed || !S || !zc) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(w_packed) || (reinterpret_cast<uintptr_t>(S) & 1u) != 0 || !aligned4(zc)) return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    W4A8_CUDA_TRY(w4a8::pack::zero_point_term(w_packed, S, K, N, group, zc, static_cast<cudaStream_t>(stream),
                                              dev.sms));
    return W4A8_OK;
}

w4a8_status w4a8_amplifier_search(const float* scales, int64_t count, void* workspace, int32_t* alpha_host,
                                  void* stream) {
    if (!scales || !workspace || !alpha_host) return W4A8_ERR_INVALID_ARG;
    if (count <= 0) return W4A8_ERR_SHAPE;
    if (!aligned16(workspace)) return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    W4A8_CUDA_TRY(w4a8::pack::amplifier(scales, count, 0, workspace, s, dev.sms));
    w4a8::pack::Results r;
    W4A8_CUDA_TRY(cudaMemcpyAsync(&r, workspace, sizeof(r), cudaMemcpyDeviceToHost, s));
    W4A8_CUDA_TRY(cudaStreamSynchronize(s));
    if (r.error) return W4A8_ERR_SCALE_RANGE;
    *alpha_host = r.alpha;
    return W4A8_OK;
}

w4a8_status pack_w4_groupwise_range(const float* w, int64_t K, int64_t N, int32_t group, int32_t alpha_in,
                                    int32_t qmin, uint8_t* w_packed, float* s_g, int16_t* S, int32_t* alpha_out_host,
                                    int64_t* colsum_max_host, void* workspace, void* stream) {
    if (qmin != -7 && qmin != -8) return W4A8_ERR_INVALID_ARG;
    if (K <= 0 || N <= 0 || group <= 0 || group % 32 != 0 || K % group != 0 || N % 8 != 0) return W4A8_ERR_SHAPE;
    if (K > INT32_MAX || N > INT32_MAX || K / group > 65535 || K / 32 > 65535) return W4A8_ERR_SHAPE;
    if (!w || !s_g) return W4A8_ERR_INVALID_ARG;
    const bool scales_only = (w_packed == nullptr && S == nullptr);
    if (!scales_only && (!w_packed || !S || !alpha_out_host || !workspace)) return W4A8_ERR_INVALID_ARG;
    if (alpha_in < 0 || (alpha_in > 0 && (!is_pow2(alpha_in) || alpha_in > (1 << 30)))) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(s_g) || (w_packed && !aligned16(w_packed)) || (S && !aligned16(S)) ||
        (workspace && !aligned16(workspace)))
        return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    W4A8_CUDA_TRY(w4a8::pack::group_scales(w, K, N, group, qmin, s_g, s));
    if (scales_only) {
        W4A8_CUDA_TRY(cudaStreamSynchronize(s));
        return W4A8_OK;
    }

    const int64_t G = K / group;
    W4A8_CUDA_TRY(w4a8::pack::amplifier(s_g, G * N, alpha_in, workspace, s, dev.sms));
    w4a8::pack::Results r;
    W4A8_CUDA_TRY(cudaMemcpyAsync(&r, workspace, sizeof(r), cudaMemcpyDeviceToHost, s));
    W4A8_CUDA_TRY(cudaStreamSynchronize(s));
    if (r.error) return W4A8_ERR_SCALE_RANGE;
    // the largest integer scale is round(s_max * alpha)
    if (std::nearbyint(double(r.s_max) * double(r.alpha)) > 32767.0) {
        *alpha_out_host = r.alpha;
        return W4A8_ERR_SCALE_RANGE;
    }
    W4A8_CUDA_TRY(w4a8::pack::quantize_pack(w, s_g, r.alpha, K, N, group, qmin, w_packed, S, workspace, s));
    W4A8_CUDA_TRY(cudaMemcpyAsync(&r, workspace, sizeof(r), cudaMemcpyDeviceToHost, s));
    W4A8_CUDA_TRY(cudaStreamSynchronize(s));
    *alpha_out_host = r.alpha;
    if (colsum_max_host) *colsum_max_host = int64_t(r.colsum_max);
    const double bound = 127.0 * double(-qmin) * double(group) * double(r.colsum_max);
    if (bound >= 2147483648.0) return W4A8_ERR_OVERFLOW_BOUND;
    return W4A8_OK;
}

w4a8_status pack_w8_groupwise(const float* w, int64_t K, int64_t N, int32_t group, int32_t alpha_in, int8_t* w8,
                              float* s_g, int16_t* S, int32_t* alpha_out_host, int64_t* colsum_max_host,
                              void* workspace, void* stream) {
    if (K <= 0 || N <= 0 || group <= 0 || group % 32 != 0 || K % group != 0 || N % 8 != 0) return W4A8_ERR_SHAPE;
    if (K > INT32_MAX || N > INT32_MAX || K / group > 65535 || K / 32 > 65535) return W4A8_ERR_SHAPE;
    if (!w || !s_g || !w8 || !S || !alpha_out_host || !workspace) return W4A8_ERR_INVALID_ARG;
    if (alpha_in < 0 || (alpha_in > 0 && (!is_pow2(alpha_in) || alpha_in > (1 << 30)))) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(s_g) || !aligned16(w8) || !aligned16(S) || !aligned16(workspace))
        return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    W4A8_CUDA_TRY(w4a8::pack::group_scales_div(w, K, N, group, 127.0f, s_g, s));
    const int64_t G = K / group;
    W4A8_CUDA_TRY(w4a8::pack::amplifier(s_g, G * N, alpha_in, workspace, s, dev.sms));
    w4a8::pack::Results r;
    W4A8_CUDA_TRY(cudaMemcpyAsync(&r, workspace, sizeof(r), cudaMemcpyDeviceToHost, s));
    W4A8_CUDA_TRY(cudaStreamSynchronize(s));
    if (r.error) return W4A8_ERR_SCALE_RANGE;
    if (std::nearbyint(double(r.s_max) * double(r.alpha)) > 32767.0) {
        *alpha_out_host = r.alpha;
        return W4A8_ERR_SCALE_RANGE;
    }
    W4A8_CUDA_TRY(w4a8::pack::quantize_w8(w, s_g, r.alpha, K, N, group, w8, S, workspace, s));
    W4A8_CUDA_TRY(cudaMemcpyAsync(&r, workspace, sizeof(r), cudaMemcpyDeviceToHost, s));
    W4A8_CUDA_TRY(cudaStreamSynchronize(s));
    *alpha_out_host = r.alpha;
    if (colsum_max_host) *colsum_max_host = int64_t(r.colsum_max);
    const double bound = 127.0 * 127.0 * double(group) * double(r.colsum_max);
    if (bound >= 2147483648.0) return W4A8_ERR_OVERFLOW_BOUND;
    return W4A8_OK;
}

w4a8_status pack_w4_groupwise(const float* w, int64_t K, int64_t N, int32_t group, int32_t alpha_in,
                              uint8_t* w_packed, float* s_g, int16_t* S, int32_t* alpha_out_host,
                              int64_t* colsum_max_host, void* workspace, void* stream) {
    return pack_w4_groupwise_range(w, K, N, group, alpha_in, -7, w_packed, s_g, S, alpha_out_host, colsum_max_host,
                                   workspace, stream);
}

int64_t w4a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group, int32_t path) {
    if (check_gemm_shape(M, N, K, group) != W4A8_OK || M == 0) return 0;
    DeviceInfo dev;
    if (current_device(dev) != W4A8_OK) return -1;
    const w4a8::gemm::Plan pl = w4a8::gemm::make_plan(M, N, K, group, dev.sms, path == 2);
    // the decode kernel takes no workspace; the asymmetric-token GEMM (path 0
    // too) always runs the tiles, so path 0 returns their size
    if (gemv_path(M, N, K, path == 2, false) && path != 0) return 0;
    return plan_splits_tiles(pl) ? pl.ws_bytes : 0;
}

w4a8_status w4a8_gemm_intscale(const int8_t* q_x, const float* s_a, const uint8_t* w_packed, const int16_t* S,
                               int32_t alpha, int64_t M, int64_t N, int64_t K, int32_t group, void* y,
                               int32_t y_dtype, void* workspace, int64_t workspace_bytes, void* stream) {
    return run_gemm(w4a8::gemm::kIntScale, q_x, s_a, w_packed, S, nullptr, alpha, M, N, K, group, y, y_dtype,
                    workspace, workspace_bytes, stream);
}

w4a8_status w4a8_gemm_intscale_asym(const int8_t* q_x, const float* s_a, const int32_t* z_a,
                                    const uint8_t* w_packed, const int16_t* S, const int32_t* zc, int32_t alpha,
                                    int64_t M, int64_t N, int64_t K, int32_t group, void* y, int32_t y_dtype,
                                    void* workspace, int64_t workspace_bytes, void* stream) {
    return run_gemm(w4a8::gemm::kIntScale, q_x, s_a, w_packed, S, nullptr, alpha, M, N, K, group, y, y_dtype,
                    workspace, workspace_bytes, stream, false, z_a, zc, true);
}

w4a8_status w8a8_gemm_intscale(const int8_t* q_x, const float* s_a, const int8_t* w8, const int16_t* S, int32_t alpha,
                               int64_t M, int64_t N, int64_t K, int32_t group, void* y, int32_t y_dtype,
                               void* workspace, int64_t workspace_bytes, void* stream) {
    return run_gemm(w4a8::gemm::kIntScale, q_x, s_a, reinterpret_cast<const uint8_t*>(w8), S, nullptr, alpha, M, N,
                    K, group, y, y_dtype, workspace, workspace_bytes, stream, true);
}

w4a8_status w4a8_gemm_intscale_static_ws(const int8_t* q_x, const float* s_a, const uint8_t* w_packed,
                                         const int16_t* S, int32_t alpha, int64_t M, int64_t N, int64_t K,
                                         int32_t group, void* y, int32_t y_dtype, void* stream) {
    const w4a8_status st = check_gemm_shape(M, N, K, group);
    if (st != W4A8_OK) return st;
    const int64_t need = w4a8_gemm_workspace_size(M, N, K, group, 0);
    if (need < 0) return W4A8_ERR_CUDA;
    if (need > int64_t(W4A8_STATIC_WORKSPACE_BYTES)) return W4A8_ERR_WORKSPACE;
    void* ws = nullptr;
    const w4a8_status sw = static_workspace(&ws);
    if (sw != W4A8_OK) return sw;
    return run_gemm(w4a8::gemm::kIntScale, q_x, s_a, w_packed, S, nullptr, alpha, M, N, K, group, y, y_dtype, ws,
                    int64_t(W4A8_STATIC_WORKSPACE_BYTES), stream);
}

w4a8_status w4a8_linear_intscale(const void* x, int32_t x_dtype, int64_t M, int64_t K, int64_t ldx,
                                 const uint8_t* w_packed, const int16_t* S, int32_t alpha, int64_t N, int32_t group,
                                 void* y, int32_t y_dtype, int8_t* q_x, float* s_a, void* workspace,
                                 int64_t workspace_bytes, void* stream) {
    if (x_dtype != W4A8_F32 && x_dtype != W4A8_BF16) return W4A8_ERR_DTYPE;
    w4a8_status st = check_gemm_shape(M, N, K, group);
    if (st != W4A8_OK) return st;
    if (ldx < K) return W4A8_ERR_SHAPE;
    if (y_dtype != W4A8_F16 && y_dtype != W4A8_F32 && y_dtype != W4A8_I32) return W4A8_ERR_DTYPE;
    if (!is_pow2(alpha) || alpha > (1 << 30)) return W4A8_ERR_INVALID_ARG;
    if (M == 0) return W4A8_OK;
    if (!x || !w_packed || !S || !y) return W4A8_ERR_INVALID_ARG;
    const int64_t esz = x_dtype == W4A8_BF16 ? 2 : 4;
    if (!aligned16(x) || (ldx * esz) % 16 != 0 || !aligned16(w_packed) || !aligned16(S) || !aligned16(y))
        return W4A8_ERR_ALIGN;
    if ((q_x && !aligned16(q_x)) || (s_a && !aligned4(s_a))) return W4A8_ERR_ALIGN;
    // One kernel for a single token on the decode path, and for up to four
    // when the caller gave no buffers; otherwise quantize into the caller's
    // buffers, then the GEMM (measured faster from two tokens up: the
    // quantizer overlaps the decode kernel's weight prefetch, while the one
    // kernel quantizes every row again in each CTA).
    const bool fused = gemv_fits(M, K, false, false) && (!(q_x && s_a) || (M == 1 && gemv_path(M, N, K, false, false)));
    if (!fused) {
        if (!q_x || !s_a) return W4A8_ERR_INVALID_ARG;
        if (!aligned16(s_a)) return W4A8_ERR_ALIGN;
        st = quantize_act_per_token(x, x_dtype, M, K, ldx, q_x, s_a, stream);
        if (st != W4A8_OK) return st;
        return w4a8_gemm_intscale(q_x, s_a, w_packed, S, alpha, M, N, K, group, y, y_dtype, workspace,
                                  workspace_bytes, stream);
    }
    DeviceInfo dev;
    if ((st = current_device(dev)) != W4A8_OK) return st;
    w4a8::gemv::GemvParams g{};
    g.x = x;
    g.ldx = ldx;
    g.w = w_packed;
    g.S = S;
    g.y = y;
    g.y_dtype = y_dtype == W4A8_F16 ? w4a8::gemm::kOutF16
                                    : (y_dtype == W4A8_I32 ? w4a8::gemm::kOutI32 : w4a8::gemm::kOutF32);
    g.M = int32_t(M);
    g.N = int32_t(N);
    g.K = int32_t(K);
    g.G = int32_t(K / group);
    g.group = group;
    g.inv_alpha = std::ldexp(1.0f, -int(std::log2(double(alpha))));
    g.q_out = q_x;
    g.s_out = s_a;
    g.status = dev.status;
    g.wait_limit = g_wait_limit.load();
    CUtensorMap tm;
    if (!gemv_weight_map(&tm, w_packed, N, K, M)) return W4A8_ERR_CUDA;
    W4A8_CUDA_TRY(w4a8::gemv::launch(tm, g, w4a8::gemm::kIntScale,
                                     x_dtype == W4A8_BF16 ? w4a8::gemv::kXBf16 : w4a8::gemv::kXF32, dev.sms,
                                     static_cast<cudaStream_t>(stream)));
    return W4A8_OK;
}

int64_t w4a8_grouped_workspace_size(int32_t E, int64_t N, int64_t K, int32_t group) {
    if (E < 1 || E > 256 || check_gemm_shape(1, N, K, group) != W4A8_OK) return -1;
    DeviceInfo dev;
    if (current_device(dev) != W4A8_OK) return -1;
    return grouped_layout(E, dev).total;
}

w4a8_status w4a8_gemm_intscale_grouped(const int8_t* q_x, const float* s_a, int64_t T, const int32_t* row_index,
                                       const int64_t* expert_offsets, const int32_t* out_row,
                                       const uint8_t* const* w_packed, const int16_t* const* S, int32_t alpha,
                                       int32_t E, int64_t R, int64_t N, int64_t K, int32_t group, void* y,
                                       int32_t y_dtype, int64_t y_rows, void* workspace, int64_t workspace_bytes,
                                       void* stream) {
    w4a8_status st = check_gemm_shape(1, N, K, group);
    if (st != W4A8_OK) return st;
    if (E < 1 || E > 256) return W4A8_ERR_INVALID_ARG;
    if (R < 0 || R > INT32_MAX || T < 0 || T > INT32_MAX || y_rows < 0) return W4A8_ERR_SHAPE;
    if (y_dtype != W4A8_F16 && y_dtype != W4A8_F32 && y_dtype != W4A8_I32) return W4A8_ERR_DTYPE;
    if (!is_pow2(alpha) || alpha > (1 << 30)) return W4A8_ERR_INVALID_ARG;
    if (R == 0) return W4A8_OK;
    if (T == 0 || !out_row && y_rows < R) return W4A8_ERR_SHAPE;
    if (!row_index && T < R) return W4A8_ERR_SHAPE;  // the routed rows themselves
    if (!q_x || !s_a || !expert_offsets || !w_packed || !S || !y) return W4A8_ERR_INVALID_ARG;
    if (!aligned16(q_x) || !aligned16(y) || !aligned4(s_a) || (row_index && !aligned4(row_index)) ||
        (out_row && !aligned4(out_row)) ||
        (reinterpret_cast<uintptr_t>(expert_offsets) & 7u) != 0 || (reinterpret_cast<uintptr_t>(w_packed) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(S) & 7u) != 0)
        return W4A8_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = current_device(dev)) != W4A8_OK) return st;
    const GroupedLayout L = grouped_layout(E, dev);
    if (!workspace || workspace_bytes < L.total) return W4A8_ERR_WORKSPACE;
    if (!aligned16(workspace)) return W4A8_ERR_ALIGN;
    uint8_t* ws = static_cast<uint8_t*>(workspace);

    const float inv_alpha = std::ldexp(1.0f, -int(std::log2(double(alpha))));
    const int32_t y_kind = y_dtype == W4A8_F16 ? w4a8::gemm::kOutF16
                                               : (y_dtype == W4A8_I32 ? w4a8::gemm::kOutI32 : w4a8::gemm::kOutF32);
    // The tiles of w4a8_gemm_intscale (token tile 128) in grouped mode.
    // Tensor maps: a template for the experts' packed weights (its address is
    // replaced per expert on the device), and the codes [T][K]: boxes of 128
    // rows for routed-order codes, one row high for rows gathered by index
    // (four rows per copy).
    CUtensorMap tm_w, tm_x;
    if (!make_map_u8(&tm_w, workspace, uint64_t(K / 2), uint64_t(N), uint64_t(K / 2),
                     uint32_t(w4a8::gemm::weight_box_bytes()), 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    if (!make_map_u8(&tm_x, q_x, uint64_t(K), uint64_t(T), uint64_t(K), 128, row_index ? 1u : 128u,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A8_ERR_CUDA;
    w4a8::gemm::ParamsGr g{};
    g.s_a = s_a;
    g.y = y;
    g.ws_count = reinterpret_cast<int32_t*>(ws);
    g.ws_part = reinterpret_cast<int32_t*>(ws + 4096);
    g.status = dev.status;
    g.M = 0;
    g.N = N;
    g.G = K / group;
    g.kb_per_group = group / 128;
    g.grid = L.grid;
    g.inv_alpha = inv_alpha;
    g.y_dtype = y_kind;
    g.wait_limit = g_wait_limit.load();
    g.grp_sched = reinterpret_cast<const int32_t*>(ws + L.sched_off);
    g.grp_maps = reinterpret_cast<const CUtensorMap*>(ws + L.maps_off);
    g.grp_scales = reinterpret_cast<const void* const*>(S);
    g.out_row = out_row;
    g.row_index = row_index;
    g.y_rows = out_row ? y_rows : R;
    g.E = E;
    g.n_tiles = int32_t((N + 127) / 128);
    g.T = int32_t(T);
    W4A8_CUDA_TRY(w4a8::gemm::launch_grouped(tm_w, tm_x, expert_offsets,
                                             reinterpret_cast<const void* const*>(w_packed), R, g,
                                             reinterpret_cast<int32_t*>(ws + L.sched_off),
                                             reinterpret_cast<CUtensorMap*>(ws + L.maps_off),
                                             static_cast<cudaStream_t>(stream)));
    return W4A8_OK;
}

w4a8_status w4a8_gemm_floatscale(const int8_t* q_x, const float* s_a, const uint8_t* w_packed, const float* s_g,
                                 int64_t M, int64_t N, int64_t K, int32_t group, void* y, int32_t y_dtype,
                                 void* workspace, int64_t workspace_bytes, void* stream) {
    return run_gemm(w4a8::gemm::kFloatScale, q_x, s_a, w_packed, nullptr, s_g, 1, M, N, K, group, y, y_dtype,
                    workspace, workspace_bytes, stream);
}

w4a8_status w4a8_tensor_i8_peak_probe(int64_t iters, int32_t n, int32_t a_in_tmem, int32_t* grid_host,
                                      double* ops_host, void* stream) {
    if (iters < 1 || iters > (int64_t(1) << 30) || n < 16 || n > 256 || n % 16 != 0) return W4A8_ERR_SHAPE;
    if (!grid_host || !ops_host) return W4A8_ERR_INVALID_ARG;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    W4A8_CUDA_TRY(w4a8::peak::launch(iters, n, a_in_tmem != 0, dev.sms, dev.status, static_cast<cudaStream_t>(stream)));
    *grid_host = dev.sms;
    *ops_host = 2.0 * 128.0 * double(n) * 128.0 * double(iters) * double(dev.sms);
    return W4A8_OK;
}

int64_t w4a8_set_wait_limit(int64_t cycles) {
    const long long v = cycles > 0 ? (long long)cycles : kDefaultWaitLimit;
    return int64_t(g_wait_limit.exchange(v));
}

int32_t w4a8_last_cuda_error(int32_t clear) {
    const int32_t e = int32_t(t_last_cuda_error);
    if (clear) t_last_cuda_error = cudaSuccess;
    return e;
}

const char* w4a8_cuda_error_string(int32_t code) { return cudaGetErrorString(cudaError_t(code)); }

w4a8_status w4a8_device_status(int32_t* code_host, int32_t clear) {
    if (!code_host) return W4A8_ERR_INVALID_ARG;
    DeviceInfo dev;
    w4a8_status st = current_device(dev);
    if (st != W4A8_OK) return st;
    int v = 0;
    W4A8_CUDA_TRY(cudaMemcpy(&v, dev.status, sizeof(int), cudaMemcpyDeviceToHost));
    *code_host = v;
    if (clear) {
        const int zero = 0;
        W4A8_CUDA_TRY(cudaMemcpy(dev.status, &zero, sizeof(int), cudaMemcpyHostToDevice));
        // Any device-side error may have cut a GEMM short (the word keeps only
        // the last error, so a timeout can hide behind a later code): the
        // split-tile arrival counts of the library's own workspace may be
        // stale, so zero them whenever a nonzero status is cleared.
        if (v != 0) {
            const w4a8_status r = w4a8_static_workspace_reset();
            if (r != W4A8_OK) return r;
        }
    }
    return W4A8_OK;
}

w4a8_status w4a8_static_workspace_reset(void) {
    int d = 0;
    W4A8_CUDA_TRY(cudaGetDevice(&d));
    void* ws = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_static_ws_mutex);
        if (d >= 0 && d < kMaxDevices && g_static_ws[d].ready) ws = g_static_ws[d].ptr;
    }
    if (ws) {  // the arrival counters: the first 4096 bytes of the array
        W4A8_CUDA_TRY(cudaMemset(ws, 0, 4096));
        W4A8_CUDA_TRY(cudaDeviceSynchronize());
    }
    return W4A8_OK;
}

}  // extern "C"
