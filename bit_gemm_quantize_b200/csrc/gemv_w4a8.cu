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
// Layout: a CTA owns 32 consecutive output columns (lane = column) and splits
// K over its warps.  Each warp streams its share of the 32 columns with TMA:
// one box of 32 rows x 128 bytes (two 128-wide K blocks of every column) per
// stage into a ring of shared-memory slots (128-byte swizzle, so the lanes'
// 16-byte reads of their own rows are conflict-free); the rings fill the
// SMs' shared memory, which is what keeps enough bytes in flight.
// A lane unpacks its column's int4 codes to 16 * q in int8 lanes (three
// integer ops per 8 weights) and dp4a multiplies them with the token codes,
// kept in shared memory and read by all lanes at once (broadcast).  Per
// 128-wide K block and token:
//   P = (sum of dp4a) >> 4              (exact: every product is 16 q x)
// and per group, after its last block:
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

#ifndef W4A8_GEMV_WARPS_PER_SM
#define W4A8_GEMV_WARPS_PER_SM 24  // target warps per SM of the launch shape
#endif
#ifndef W4A8_GEMV_INTERLEAVE
#define W4A8_GEMV_INTERLEAVE 1
#endif

constexpr int kCols = 32;              // output columns per CTA (one per lane)
// A stage is SUB 128-wide K blocks of the CTA's 32 columns: one box of 32 rows
// x 64 SUB bytes, 64 SUB * 32 bytes of shared memory.
constexpr int stage_bytes(int sub) { return kCols * 64 * sub; }
constexpr int kMaxStages = 16;
constexpr int kSmemCap = 225 * 1024;  // dynamic shared memory a CTA may take (the rest: static, alignment)

// Shared memory of a CTA with ks warps and rings of `stages` slots: the token
// codes [mt][K], the rings [ks][stages][2 KB], one mbarrier per slot, the
// partial sums [ks][mt][32], the tokens' output scales.
int smem_bytes(int mt, int K, int ks, int stages, int sub) {
    return ((mt * K + 1023) / 1024) * 1024 + ks * stages * stage_bytes(sub) + ks * stages * 8 + ks * mt * kCols * 4 +
           16;
}

// W8: 8-bit weight codes [N][K] (the W8A8 variant): a 128-byte box is one
// 128-wide K block, used as it lands (no unpack, no shift of P).
template <int MT, int PATH, typename XT, int kSub, bool W8 = false>
__global__ void __launch_bounds__(512) gemv_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvParams p) {
    constexpr int kStage = stage_bytes(kSub);
    constexpr int kBoxBytes = 64 * kSub;
    constexpr int kKB = W8 ? kSub / 2 : kSub;  // 128-wide K blocks per stage
    static_assert(!W8 || (kSub == 2 && PATH == gemm::kIntScale && std::is_same<XT, int8_t>::value), "W8 form");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int K = p.K, N = p.N;
    const int ks = blockDim.x >> 5;
    const int nst = p.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int8_t* codes = reinterpret_cast<int8_t*>(smem);                                      // [MT][K]
    uint8_t* rings = smem + ((MT * K + 1023) / 1024) * 1024;                              // [ks][nst][kStage]
    uint64_t* bars = reinterpret_cast<uint64_t*>(rings + ks * nst * kStage);              // [ks][nst]
    int32_t* red = reinterpret_cast<int32_t*>(bars + ks * nst);                           // [ks][MT][32]
    float* redf = reinterpret_cast<float*>(red);
    float* scl = reinterpret_cast<float*>(red + ks * MT * kCols);                         // [MT]
    __shared__ float wmax[16 * MT];
    __shared__ int abort_s;
    if (threadIdx.x == 0) {
        for (int i = 0; i < ks * nst; ++i) mbar_init(&bars[i], 1);
        abort_s = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_w);
        griddep_launch_dependents();
    }
    __syncthreads();  // barriers initialized

    // this warp's stages (kSub K blocks of the CTA's 32 columns each); the
    // first stages' boxes go out before anything else (packed weights are never
    // written by a kernel that lets its successor start early)
    const int n0 = blockIdx.x * kCols;
    const int kbpg = p.group >> 7;  // 128-wide K blocks per group
    const int nkbt = K >> 7;
    const int nstt = (nkbt + kKB - 1) / kKB;  // stages of the whole K
#if W4A8_GEMV_INTERLEAVE
    // warp w takes stages w, w + ks, w + 2 ks, ...: at any time the CTA's
    // warps read neighbouring pieces of each column
    const int s0 = warp, sstep = ks, nkb = (nstt - warp + ks - 1) / ks;
#else
    // warp w takes a contiguous run of stages
    const int s0 = (warp * nstt) / ks, sstep = 1, nkb = ((warp + 1) * nstt) / ks - s0;
#endif
    uint8_t* ring = rings + warp * nst * kStage;
    uint64_t* wbar = bars + warp * nst;
    int issued = 0;
    auto issue = [&](int j, int slot) {  // this warp's stage j (stage s0 + j sstep), into ring slot `slot`
        issued = j + 1;
        mbar_arrive_expect_tx_one(&wbar[slot], uint32_t(kStage));
        tma_load_2d_one(ring + slot * kStage, &tm_w, (s0 + j * sstep) * kBoxBytes, n0, &wbar[slot]);
    };
    for (int j = 0; j < nst && j < nkb; ++j) issue(j, j);
    griddep_wait();  // the tokens may be the previous kernel's output, y its input

    // ---- the token codes of rows 0..MT-1 (rows past M: zero codes, scale 0)
    constexpr bool kFused = !std::is_same<XT, int8_t>::value;
    const int nthreads = blockDim.x;
    if constexpr (kFused) {
        // every row's absolute maximum at once (all rows' loads in flight),
        // one block-wide exchange, then every row's codes
        float a[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            a[m] = 0.0f;
            if (m < p.M) {
                const XT* row = reinterpret_cast<const XT*>(p.x) + int64_t(m) * p.ldx;
                for (int c = threadIdx.x; c < K / 16; c += nthreads) {
                    float v[16];
                    quant::load16<XT>(row + c * 16, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) a[m] = fmaxf(a[m], fabsf(v[i]));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a[m] = fmaxf(a[m], __shfl_xor_sync(0xffffffffu, a[m], o));
            if (lane == 0) wmax[warp * MT + m] = a[m];
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const bool live = m < p.M;
            const XT* row = reinterpret_cast<const XT*>(p.x) + int64_t(m) * p.ldx;
            float amax = 0.0f;
            for (int w = 0; w < ks; ++w) amax = fmaxf(amax, wmax[w * MT + m]);
            const float s = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, 127.0f);
            const bool zero = (s == 0.0f);
            const bool exact_only = s < 1e-30f;
            const float rcp = zero ? 0.0f : __frcp_rn(s);
            for (int c = threadIdx.x; c < K / 16; c += nthreads) {
                uint32_t packed[4] = {0u, 0u, 0u, 0u};
                if (live && !zero) {
                    float v[16];
                    quant::load16<XT>(row + c * 16, v);
                    uint32_t cb[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) cb[i] = quant::code_i8_byte(v[i], s, rcp, exact_only);
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        packed[w] = quant::pack4_low_bytes(cb[4 * w], cb[4 * w + 1], cb[4 * w + 2], cb[4 * w + 3]);
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
            const float s = int(threadIdx.x) < p.M ? p.s_a[threadIdx.x] : 0.0f;
            scl[threadIdx.x] = PATH == gemm::kIntScale ? __fmul_rn(s, p.inv_alpha) : s;
        }
    }
    __syncthreads();

    // ---- the stages: lane = column n0 + lane, its row of the box
    const int n = n0 + lane;
    const bool nvalid = n < N;
    const int n_ld = nvalid ? n : 0;  // a column past N: its row of the box reads as zero, its scale as column 0's
    // 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3) (64-byte
    // swizzle of 64-byte rows) or c ^ (r & 7) (128-byte swizzle)
    const int sw = kSub == 1 ? (lane >> 1) & 3 : lane & 7;
    int32_t acc[MT], pg[MT];
    float accf[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        acc[m] = 0;
        pg[m] = 0;
        accf[m] = 0.0f;
    }
    // the scales of stage jj's K blocks, loaded two stages ahead (0 past the
    // last block)
    auto ld_scales = [&](int jj, uint32_t (&sc)[kKB]) {
#pragma unroll
        for (int u = 0; u < kKB; ++u) {
            const int kb = (s0 + jj * sstep) * kKB + u;
            sc[u] = 0u;
            if (jj < nkb && kb < nkbt) {
                const int64_t si = int64_t(kb / kbpg) * N + n_ld;
                if constexpr (PATH == gemm::kIntScale)
                    sc[u] = uint32_t(int32_t(__ldg(p.S + si)));
                else
                    sc[u] = __float_as_uint(__ldg(p.s_g + si));
            }
        }
    };
    uint32_t sc0[kKB], sc1[kKB], sc2[kKB];
    ld_scales(0, sc0);
    ld_scales(1, sc1);
    bool ok = true;
    int j = 0, slot = 0;
    uint32_t phase = 0;
    for (; j < nkb; ++j) {
        if (!mbar_wait_warp(&wbar[slot], phase, &abort_s, p.status, p.wait_limit)) {
            ok = false;
            break;
        }
        ld_scales(j + 2, sc2);
        const uint8_t* row = ring + slot * kStage + lane * kBoxBytes;
        const int kbs = (s0 + j * sstep) * kKB;
#pragma unroll
        for (int u = 0; u < kKB; ++u) {
            const int kb = kbs + u;
            if (kKB > 1 && kb >= nkbt) break;  // the last stage of a K that is not a whole number of stages
            // the block's 128 weights of this column in int8 lanes (as 16 q,
            // unpacked once for all tokens, or the 8-bit codes as they are)
            uint32_t wq[32];
            if constexpr (W8) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ sw) << 4));
                    wq[4 * c] = v.x;
                    wq[4 * c + 1] = v.y;
                    wq[4 * c + 2] = v.z;
                    wq[4 * c + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(row + (((4 * u + c) ^ sw) << 4));
                    const uint32_t pk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint2 e = gemm::unpack_int4x8_x16(pk[h]);
                        wq[8 * c + 2 * h] = e.x;
                        wq[8 * c + 2 * h + 1] = e.y;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint4* xr = reinterpret_cast<const uint4*>(codes + m * K + kb * 128);
                int32_t t0 = 0, t1 = 0, t2 = 0, t3 = 0;
#pragma unroll
                for (int c = 0; c < 8; ++c) {  // 16 weights against 16 token codes (one broadcast load)
                    const uint4 x = xr[c];
                    t0 = __dp4a(int(wq[4 * c]), int(x.x), t0);
                    t1 = __dp4a(int(wq[4 * c + 1]), int(x.y), t1);
                    t2 = __dp4a(int(wq[4 * c + 2]), int(x.z), t2);
                    t3 = __dp4a(int(wq[4 * c + 3]), int(x.w), t3);
                }
                pg[m] += (t0 + t1) + (t2 + t3);
            }
            // the group ends, or this warp's run of it: apply the group's
            // scale to the part summed so far (S times a partial sum is still
            // exact)
            if ((kb + 1) % kbpg == 0 || u == kKB - 1 || kb + 1 == nkbt) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const int32_t P = W8 ? pg[m] : pg[m] >> 4;  // exact: every 4-bit product is 16 q x
                    if constexpr (PATH == gemm::kIntScale)
                        acc[m] += int32_t(sc0[u]) * P;
                    else
                        accf[m] = __fmaf_rn(__uint_as_float(sc0[u]), __int2float_rn(P), accf[m]);
                    pg[m] = 0;
                }
            }
        }
        __syncwarp();  // every lane has used its row of the slot: refill it
        if (j + nst < nkb) issue(j + nst, slot);
        if (++slot == nst) {
            slot = 0;
            phase ^= 1u;
        }
#pragma unroll
        for (int u = 0; u < kKB; ++u) {
            sc0[u] = sc1[u];
            sc1[u] = sc2[u];
        }
    }
    if (!ok && lane == 0) {  // after a timeout, let the boxes in flight (stages j..issued-1) land
        for (int jj = j; jj < issued; ++jj) gemm::drain_wait(&wbar[jj % nst], uint32_t((jj / nst) & 1));
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
    for (int m = warp; m < MT && m < p.M && nvalid; m += ks) {
        int32_t a = 0;
        float af = 0.0f;
        for (int w = 0; w < ks; ++w) {
            if constexpr (PATH == gemm::kIntScale)
                a += red[(w * MT + m) * kCols + lane];
            else
                af = __fadd_rn(af, redf[(w * MT + m) * kCols + lane]);
        }
        if constexpr (PATH == gemm::kIntScale) {
            // asymmetric token codes: acc - z[m] * zc[n] in two's-complement
            // arithmetic (the terms may wrap; the difference fits in 32 bits)
            if (p.zc != nullptr) a = int32_t(uint32_t(a) - uint32_t(p.z_a[m]) * uint32_t(p.zc[n]));
        }
        const float v = __fmul_rn(PATH == gemm::kIntScale ? __int2float_rn(a) : af, scl[m]);
        const int64_t o = int64_t(m) * N + n;
        if (p.y_dtype == gemm::kOutI32)
            reinterpret_cast<int32_t*>(p.y)[o] = a;
        else if (p.y_dtype == gemm::kOutF16)
            reinterpret_cast<__half*>(p.y)[o] = __float2half_rn(v);
        else
            reinterpret_cast<float*>(p.y)[o] = v;
    }
}

// The launch shape: enough CTAs per SM that the grid is one wave, the most
// warps per CTA (the K split: at most 16, at most one per stage, about 24
// warps per SM) and rings as deep as the shared memory left to each
// CTA allows.
template <auto kern>
static int regs_of() {  // registers a thread of `kern` uses (read once)
    static const int regs = [] {
        cudaFuncAttributes a{};
        return cudaFuncGetAttributes(&a, kern) == cudaSuccess ? a.numRegs : 255;
    }();
    return regs;
}

// CTAs of `threads` threads and `smem` bytes one SM holds at once (SM limits:
// 2048 threads, 32 CTAs, 64 K registers allocated per warp in units of 256,
// 228 KB of shared memory with 1 KB reserved per CTA).
static int resident(int regs, int threads, int smem) {
    const int warps = threads / 32;
    const int warp_regs = ((regs * 32 + 255) / 256) * 256;
    int occ = 2048 / threads;
    occ = occ < 32 ? occ : 32;
    const int by_regs = 65536 / (warp_regs * warps);
    const int by_smem = (228 * 1024) / (smem + 1024);
    occ = occ < by_regs ? occ : by_regs;
    return occ < by_smem ? occ : by_smem;
}

template <auto kern>
static void shape(const GemvParams& p, int mt, int sub, int kb_per_stage, int num_sms, int& ks, int& stages,
                  int& smem) {
    const int64_t blocks = (p.N + kCols - 1) / kCols;
    const int nkb_total = (p.K / 128 + kb_per_stage - 1) / kb_per_stage;  // stages of the whole K
    // CTAs each SM holds: the whole grid at once if the shared memory allows,
    // else fewer (more waves)
    for (int per_sm = int((blocks + num_sms - 1) / num_sms);; --per_sm) {
        ks = W4A8_GEMV_WARPS_PER_SM / per_sm;
        ks = ks > 16 ? 16 : (ks < 1 ? 1 : ks);
        ks = ks > nkb_total ? nkb_total : ks;
        for (; ks >= 1; --ks) {
            const int fixed = smem_bytes(mt, p.K, ks, 0, sub) + 1024;  // + alignment slack
            int cap = (228 * 1024) / per_sm - 2048;               // 1 KB reserved per CTA, 1 KB static
            cap = cap < kSmemCap ? cap : kSmemCap;
            const int nkb = (nkb_total + ks - 1) / ks;
            stages = (cap - fixed) / (ks * (stage_bytes(sub) + 8));
            stages = stages > kMaxStages ? kMaxStages : stages;
            stages = stages > nkb ? nkb : stages;
            if (stages < 2 && stages < nkb) continue;  // a ring needs two slots to overlap
            smem = smem_bytes(mt, p.K, ks, stages, sub) + 1024;
            if (resident(regs_of<kern>(), 32 * ks, smem) >= per_sm) return;
        }
        if (per_sm == 1) break;
    }
    // one warp, one slot (always fits: the token codes take at most 64 KB)
    ks = 1;
    stages = 1;
    smem = smem_bytes(mt, p.K, 1, 1, sub) + 1024;
}

template <int MT, int PATH, typename XT, bool W8 = false>
static cudaError_t launch_t(const CUtensorMap& tm_w, const GemvParams& p, int num_sms, cudaStream_t stream) {
    constexpr int sub = box_bytes(MT, W8) / 64;
    constexpr auto kern = gemv_kernel<MT, PATH, XT, sub, W8>;
    cudaError_t e = configure_once<kern>(512, kSmemCap);
    if (e != cudaSuccess) return e;
    int ks = 1, stages = 1, smem = 0;
    shape<kern>(p, MT, sub, W8 ? sub / 2 : sub, num_sms, ks, stages, smem);
    GemvParams q = p;
    q.stages = stages;
    const unsigned grid = unsigned((p.N + kCols - 1) / kCols);
    const LaunchPdl lc(grid, unsigned(32 * ks), size_t(smem), stream);
    return cudaLaunchKernelEx(&lc.cfg, kern, tm_w, q);
}

template <int PATH, typename XT, bool W8 = false>
static cudaError_t launch_path(const CUtensorMap& tm_w, const GemvParams& p, int num_sms, cudaStream_t stream) {
    switch (p.M) {
        case 1: return launch_t<1, PATH, XT, W8>(tm_w, p, num_sms, stream);
        case 2: return launch_t<2, PATH, XT, W8>(tm_w, p, num_sms, stream);
        default: return launch_t<4, PATH, XT, W8>(tm_w, p, num_sms, stream);
    }
}

cudaError_t launch_w8(const CUtensorMap& tm_w, const GemvParams& p, int num_sms, cudaStream_t stream) {
    return launch_path<gemm::kIntScale, int8_t, true>(tm_w, p, num_sms, stream);
}

cudaError_t launch(const CUtensorMap& tm_w, const GemvParams& p, int path, int x_kind, int num_sms,
                   cudaStream_t stream) {
    if (path == gemm::kIntScale) {
        if (x_kind == kXCodes) return launch_path<gemm::kIntScale, int8_t>(tm_w, p, num_sms, stream);
        if (x_kind == kXBf16) return launch_path<gemm::kIntScale, __nv_bfloat16>(tm_w, p, num_sms, stream);
        return launch_path<gemm::kIntScale, float>(tm_w, p, num_sms, stream);
    }
    if (x_kind == kXCodes) return launch_path<gemm::kFloatScale, int8_t>(tm_w, p, num_sms, stream);
    if (x_kind == kXBf16) return launch_path<gemm::kFloatScale, __nv_bfloat16>(tm_w, p, num_sms, stream);
    return launch_path<gemm::kFloatScale, float>(tm_w, p, num_sms, stream);
}

}  // namespace gemv
}  // namespace w4a8
