// W4A8 GEMM for sm_100a: int8 tokens x int4 group-quantized weights on the
// tcgen05 tensor cores, with either integer group scales (the Integer-Scale
// scheme: one IMAD per output per group, one rescale at the end) or float
// group scales (the comparison path: one I32->F32 conversion and FMA per
// output per group).
//
// Integer Scale: A Free Lunch for Faster Fine-grained Quantization of LLMs
// (summary), Fig. 3(b)/(c) and §4; "Quantization" notes, 矩阵乘法中的量化计算.
//
// Layout of the computation ("swap AB"): the MMA's 128-row side is a tile of
// 128 weight columns n, the MMA's N side is a tile of BT tokens m.  A TMEM
// lane therefore owns one output column n, so the group scale S[g,n] is a
// per-thread scalar in the per-group drain.
//
//   HBM --TMA--> packed int4 tile [128 n][64 B]  --unpack warps-->
//   int8 tile [128 n][128 k] (128-byte swizzle, K-major) = MMA operand A
//   HBM --TMA--> token codes [BT m][128 k] (128-byte swizzle) = MMA operand B
//   tcgen05.mma.kind::i8 x4 (K = 32 each) -> TMEM int32 P_g [128 lanes][BT cols]
//   epilogue warps: tcgen05.ld P_g, acc += S[g,n] * P_g (or accf += s_g * float(P_g))
//   after the last group: y = acc * s_a[m] / alpha  (or accf * s_a[m])
//
// Work partition: the (tile, group) steps of the whole problem are split into
// one contiguous range per CTA of a persistent grid (stream-K).  A tile whose
// groups fall into several CTAs' ranges is combined through a workspace: each
// contributor stores its partial, the last one to arrive (per-tile counter)
// sums the partials in CTA order and writes y.  Integer partials are exact;
// float partials are summed in a fixed order, so results are deterministic.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm_w4a8.h"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace gemm {

constexpr int kTileN = 128;   // weight columns per tile (MMA M)
constexpr int kBlockK = 128;  // K per pipeline stage
constexpr int kUnpackWarps = 4;
constexpr int kEpiWarps = 8;
constexpr int kNumWarps = 2 + kUnpackWarps + kEpiWarps;
constexpr int kThreads = kNumWarps * 32;

template <int BT>
struct Cfg {
    static constexpr int kA = kTileN * kBlockK;       // unpacked weights, bytes
    static constexpr int kB = BT * kBlockK;           // token codes, bytes
    static constexpr int kWp = kTileN * kBlockK / 2;  // packed weights, bytes
    static constexpr int kStageBytes = kA + kB + kWp;
    static constexpr int kStages = (200 * 1024) / kStageBytes > 8 ? 8 : (200 * 1024) / kStageBytes;
    static constexpr int offA = 0;
    static constexpr int offB = offA + kStages * kA;
    static constexpr int offWp = offB + kStages * kB;
    static constexpr int offBar = offWp + kStages * kWp;
    static constexpr int kBars = 3 * kStages + 5;  // full, wready, empty, tfull x2, tempty x2, mma_done
    static constexpr int offMisc = offBar + kBars * 8;
    static constexpr int kSmemBytes = offMisc + 64 + 1024;  // + slack to align the base to 1024
    static constexpr uint32_t kTmemCols = (2 * BT) < 32 ? 32u : uint32_t(2 * BT);
    static_assert(kB % 1024 == 0, "token tile must hold whole 8-row swizzle atoms");
    static_assert(kStages >= 2, "pipeline too shallow");
};

// One contiguous run of groups [g0, g1) of one tile inside a CTA's range.
struct Segment {
    int64_t tile;
    int g0, g1;
    int64_t first;  // flattened index of the segment's first step
};

__device__ __forceinline__ int64_t range_start(int64_t b, int64_t W, int64_t grid) { return b * W / grid; }

// CTA whose range holds flattened step i.
__device__ __forceinline__ int64_t range_owner(int64_t i, int64_t W, int64_t grid) {
    return ((i + 1) * grid - 1) / W;
}

// Iterates the segments of CTA `b`.
struct SegmentIter {
    int64_t i, end, G;
    __device__ SegmentIter(const Params& p, int64_t b) {
        G = p.G;
        i = range_start(b, p.W, p.grid);
        end = range_start(b + 1, p.W, p.grid);
    }
    __device__ bool next(Segment& s) {
        if (i >= end) return false;
        s.tile = i / G;
        s.g0 = int(i - s.tile * G);
        int64_t stop = (s.tile + 1) * G < end ? (s.tile + 1) * G : end;
        s.g1 = int(stop - s.tile * G);
        s.first = i;
        i = stop;
        return true;
    }
};

// int4 two's-complement nibbles -> int8, 8 values per 32-bit word.  Input byte
// j holds k = 2j (low nibble) and k = 2j+1 (high nibble); output words hold
// k = 0..3 and k = 4..7 in byte order.  Per byte: ((v ^ 8) + 0x78) ^ 0x80
// maps nibble v to its sign-extended byte without carries between bytes.
__device__ __forceinline__ uint2 unpack_int4x8(uint32_t w) {
    uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
    uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
    lo = (lo + 0x78787878u) ^ 0x80808080u;
    hi = (hi + 0x78787878u) ^ 0x80808080u;
    return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

__device__ __forceinline__ void epi_bar_sync() {
    asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 8) {
        tmem_ld8(taddr, r);
    } else if constexpr (N == 16) {
        tmem_ld16(taddr, r);
    } else {
        static_assert(N == 32, "columns per load");
        tmem_ld32(taddr, r);
    }
}

// Bounded wait without the abort short-cut, for draining copies in flight.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > 1000000000ull) break;
    }
}

template <int PATH>
__device__ __forceinline__ void store_output(const Params& p, int64_t m, int64_t n, float vf, int32_t vi) {
    const int64_t idx = m * p.N + n;
    if (PATH == kIntScale) {
        if (p.y_dtype == kOutI32) {
            static_cast<int32_t*>(p.y)[idx] = vi;
            return;
        }
        const float scale = __fmul_rn(p.s_a[m], p.inv_alpha);  // exact: inv_alpha is a power of two
        vf = __fmul_rn(__int2float_rn(vi), scale);
    } else {
        vf = __fmul_rn(vf, p.s_a[m]);
    }
    if (p.y_dtype == kOutF16)
        static_cast<__half*>(p.y)[idx] = __float2half_rn(vf);
    else
        static_cast<float*>(p.y)[idx] = vf;
}

template <int BT, int PATH>
__global__ void __launch_bounds__(kThreads, 1)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                     const Params p) {
    using C = Cfg<BT>;
    constexpr int S = C::kStages;
    constexpr int HC = BT / 2;  // columns per epilogue thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::offBar);
    uint64_t* full = bars;
    uint64_t* wready = bars + S;
    uint64_t* empty = bars + 2 * S;
    uint64_t* tfull = bars + 3 * S;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::offMisc);  // [0] tmem base [1] abort [2] last
    volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&wready[s], kUnpackWarps);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        mbar_init(mma_done, 1);
        misc[1] = 0;
        misc[2] = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
    }
    if (warp == 1) tmem_alloc(&misc[0], C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const int64_t b = blockIdx.x;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued_parity[S];
            for (int s = 0; s < S; ++s) issued_parity[s] = -1;
            SegmentIter it(p, b);
            Segment sg;
            bool ok = true;
            while (ok && it.next(sg)) {
                const int32_t n0 = int32_t((sg.tile / p.m_tiles) * kTileN);
                const int32_t m0 = int32_t((sg.tile % p.m_tiles) * BT);
                for (int g = sg.g0; ok && g < sg.g1; ++g) {
                    for (int kb = 0; kb < p.kb_per_group; ++kb) {
                        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        const int32_t kblk = g * p.kb_per_group + kb;
                        mbar_arrive_expect_tx(&full[stage], C::kWp + C::kB);
                        tma_load_2d(smem + C::offWp + stage * C::kWp, &tm_w, kblk * (kBlockK / 2), n0, &full[stage]);
                        tma_load_2d(smem + C::offB + stage * C::kB, &tm_x, kblk * kBlockK, m0, &full[stage]);
                        issued_parity[stage] = int(phase);
                        if (++stage == S) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            if (!ok) {  // let copies in flight land before the CTA leaves
                for (int s = 0; s < S; ++s)
                    if (issued_parity[s] >= 0) drain_wait(&full[s], uint32_t(issued_parity[s]));
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kTileN, BT);
            int stage = 0;
            uint32_t phase = 0;
            int ab = 0;
            uint32_t aphase = 0;
            SegmentIter it(p, b);
            Segment sg;
            bool ok = true;
            while (ok && it.next(sg)) {
                for (int g = sg.g0; ok && g < sg.g1; ++g) {
                    if (!mbar_wait(&tempty[ab], aphase ^ 1u, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem_base + uint32_t(ab * BT);
                    for (int kb = 0; kb < p.kb_per_group; ++kb) {
                        if (!mbar_wait(&wready[stage], phase, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + C::offA + stage * C::kA);
                        const uint32_t b_addr = smem_u32(smem + C::offB + stage * C::kB);
#pragma unroll
                        for (int k = 0; k < kBlockK / 32; ++k)
                            mma_i8(d, smem_desc_sw128(a_addr + k * 32), smem_desc_sw128(b_addr + k * 32), idesc,
                                   uint32_t(kb | k));
                        mma_commit(&empty[stage]);
                        if (++stage == S) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    mma_commit(&tfull[ab]);
                    ab ^= 1;
                    if (ab == 0) aphase ^= 1u;
                }
            }
            // every MMA this thread issued has finished before TMEM is released
            mma_commit(mma_done);
            drain_wait(mma_done, 0);
        }
    } else if (warp < 2 + kUnpackWarps) {
        // ---------------------------------------------------------- int4 -> int8 unpack
        const int uw = warp - 2;
        int stage = 0;
        uint32_t phase = 0;
        SegmentIter it(p, b);
        Segment sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            const int steps = (sg.g1 - sg.g0) * p.kb_per_group;
            for (int st = 0; st < steps; ++st) {
                if (!mbar_wait(&full[stage], phase, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                const uint8_t* wp = smem + C::offWp + stage * C::kWp;
                uint8_t* a = smem + C::offA + stage * C::kA;
#pragma unroll
                for (int itr = 0; itr < kTileN / (8 * kUnpackWarps); ++itr) {
                    const int r = uw * (kTileN / kUnpackWarps) + itr * 8 + (lane >> 2);
                    const int c = lane & 3;
                    const uint4 v = *reinterpret_cast<const uint4*>(wp + r * (kBlockK / 2) + c * 16);
                    const uint2 o0 = unpack_int4x8(v.x), o1 = unpack_int4x8(v.y);
                    const uint2 o2 = unpack_int4x8(v.z), o3 = unpack_int4x8(v.w);
                    uint8_t* row = a + r * kBlockK;
                    const int sw = r & 7;
                    *reinterpret_cast<uint4*>(row + (((2 * c) ^ sw) << 4)) = make_uint4(o0.x, o0.y, o1.x, o1.y);
                    *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ sw) << 4)) = make_uint4(o2.x, o2.y, o3.x, o3.y);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&wready[stage]);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int ew = warp - (2 + kUnpackWarps);
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int half = ew >> 2;      // which half of the BT columns
        const int r = quarter * 32 + lane;
        int ab = 0;
        uint32_t aphase = 0;
        SegmentIter it(p, b);
        Segment sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            const int64_t n0 = (sg.tile / p.m_tiles) * kTileN;
            const int64_t m0 = (sg.tile % p.m_tiles) * BT + half * HC;
            const int64_t n = n0 + r;
            const bool nvalid = n < p.N;
            int32_t acc[HC];
            float accf[HC];
#pragma unroll
            for (int j = 0; j < HC; ++j) {
                acc[j] = 0;
                accf[j] = 0.0f;
            }
            int32_t s_next = 0;
            float f_next = 0.0f;
            if (nvalid) {
                if (PATH == kIntScale)
                    s_next = p.S[int64_t(sg.g0) * p.N + n];
                else
                    f_next = p.s_g[int64_t(sg.g0) * p.N + n];
            }
            for (int g = sg.g0; g < sg.g1; ++g) {
                const int32_t s_cur = s_next;
                const float f_cur = f_next;
                if (nvalid && g + 1 < sg.g1) {
                    if (PATH == kIntScale)
                        s_next = p.S[int64_t(g + 1) * p.N + n];
                    else
                        f_next = p.s_g[int64_t(g + 1) * p.N + n];
                }
                if (!mbar_wait(&tfull[ab], aphase, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(ab * BT + half * HC);
                constexpr int CH = HC < 32 ? HC : 32;
#pragma unroll
                for (int c0 = 0; c0 < HC; c0 += CH) {
                    uint32_t v[CH];
                    tmem_load<CH>(taddr + uint32_t(c0), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < CH; ++j) {
                        if (PATH == kIntScale)
                            acc[c0 + j] += s_cur * int32_t(v[j]);
                        else
                            accf[c0 + j] = __fmaf_rn(f_cur, __int2float_rn(int32_t(v[j])), accf[c0 + j]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[ab]);
                ab ^= 1;
                if (ab == 0) aphase ^= 1u;
            }
            if (!ok) break;

            const bool whole = (sg.g0 == 0 && sg.g1 == p.G);
            if (whole) {
                if (nvalid) {
#pragma unroll
                    for (int j = 0; j < HC; ++j)
                        if (m0 + j < p.M) store_output<PATH>(p, m0 + j, n, accf[j], acc[j]);
                }
                continue;
            }
            // ---- split tile: store this CTA's partial, the last contributor combines
            const int slot = (sg.first == range_start(b, p.W, p.grid)) ? 0 : 1;
            const int64_t slot_elems = int64_t(kTileN) * BT;
            int32_t* part = p.ws_part + (b * 2 + slot) * slot_elems;
#pragma unroll
            for (int j = 0; j < HC; ++j) {
                const int64_t e = int64_t(half * HC + j) * kTileN + r;
                if (PATH == kIntScale)
                    part[e] = acc[j];
                else
                    part[e] = __float_as_int(accf[j]);
            }
            __threadfence();
            epi_bar_sync();
            const int64_t t0 = sg.tile * p.G;
            const int64_t b_first = range_owner(t0, p.W, p.grid);
            const int64_t b_last = range_owner(t0 + p.G - 1, p.W, p.grid);
            if (ew == 0 && lane == 0) {
                const int old = atomicAdd(&p.ws_count[sg.tile], 1);
                misc[2] = (old == int(b_last - b_first)) ? 1u : 0u;
            }
            epi_bar_sync();
            if (misc[2]) {
                __threadfence();
#pragma unroll
                for (int j = 0; j < HC; ++j) {
                    acc[j] = 0;
                    accf[j] = 0.0f;
                }
                for (int64_t c = b_first; c <= b_last; ++c) {
                    const int cslot = (range_start(c, p.W, p.grid) >= t0) ? 0 : 1;
                    const int32_t* cp = p.ws_part + (c * 2 + cslot) * slot_elems;
#pragma unroll
                    for (int j = 0; j < HC; ++j) {
                        const int32_t v = __ldcg(cp + int64_t(half * HC + j) * kTileN + r);
                        if (PATH == kIntScale)
                            acc[j] += v;
                        else
                            accf[j] = __fadd_rn(accf[j], __int_as_float(v));
                    }
                }
                if (nvalid) {
#pragma unroll
                    for (int j = 0; j < HC; ++j)
                        if (m0 + j < p.M) store_output<PATH>(p, m0 + j, n, accf[j], acc[j]);
                }
                if (ew == 0 && lane == 0) p.ws_count[sg.tile] = 0;
            }
            epi_bar_sync();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

static int token_tile_for(int64_t M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    return 128;
}

Plan make_plan(int64_t M, int64_t N, int64_t K, int32_t group, int num_sms) {
    Plan pl{};
    pl.BT = token_tile_for(M);
    pl.n_tiles = (N + kTileN - 1) / kTileN;
    pl.m_tiles = (M + pl.BT - 1) / pl.BT;
    pl.G = K / group;
    pl.tiles = pl.n_tiles * pl.m_tiles;
    pl.W = pl.tiles * pl.G;
    pl.grid = pl.W < num_sms ? pl.W : num_sms;
    const int64_t slot_bytes = int64_t(kTileN) * pl.BT * 4;
    pl.count_bytes = ((pl.tiles * 4 + 255) / 256) * 256;
    pl.ws_bytes = pl.count_bytes + pl.grid * 2 * slot_bytes;
    return pl;
}

template <int BT, int PATH>
static cudaError_t launch_bt(const CUtensorMap& tw, const CUtensorMap& tx, const Params& p, cudaStream_t stream) {
    auto kern = w4a8_gemm_kernel<BT, PATH>;
    const int smem = Cfg<BT>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(unsigned(p.grid)), dim3(kThreads), smem, stream>>>(tw, tx, p);
    return cudaGetLastError();
}

cudaError_t launch(const CUtensorMap& tw, const CUtensorMap& tx, const Params& p, int BT, int path,
                   cudaStream_t stream) {
    if (path == kIntScale) {
        switch (BT) {
            case 16: return launch_bt<16, kIntScale>(tw, tx, p, stream);
            case 32: return launch_bt<32, kIntScale>(tw, tx, p, stream);
            case 64: return launch_bt<64, kIntScale>(tw, tx, p, stream);
            default: return launch_bt<128, kIntScale>(tw, tx, p, stream);
        }
    }
    switch (BT) {
        case 16: return launch_bt<16, kFloatScale>(tw, tx, p, stream);
        case 32: return launch_bt<32, kFloatScale>(tw, tx, p, stream);
        case 64: return launch_bt<64, kFloatScale>(tw, tx, p, stream);
        default: return launch_bt<128, kFloatScale>(tw, tx, p, stream);
    }
}

int token_tile_rows() { return kTileN; }

}  // namespace gemm
}  // namespace w4a8
