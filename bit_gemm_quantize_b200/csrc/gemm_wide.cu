// Wide-tile W4A8 GEMM for sm_100a (token tiles of 256), the large-M path:
// int8 tokens x int4 group-quantized weights on the tcgen05 tensor cores with
// integer group scales (one IMAD per output per group, one rescale at the
// end) or float group scales (one I32->F32 conversion and FMA per output per
// group).
//
// Integer Scale: A Free Lunch for Faster Fine-grained Quantization of LLMs
// (summary), Fig. 3(b)/(c) and §4; "Quantization" notes, 矩阵乘法中的量化计算.
//
// Layout ("swap AB", as in the narrow-tile kernel): the MMA's 128-row side is
// a tile of 128 weight columns n, its N side a tile of 256 tokens, so a TMEM
// lane owns one output column and its group scale is a per-thread scalar.
//
// Why 256-token tiles with both operands in shared memory: back-to-back
// 128 x 256 x 32 int8 MMAs from shared memory run at 88% of the int8 rate,
// while 128 x 128 x 32 MMAs reach 66% (shared-memory operand bandwidth) and
// 128 x 128 x 32 MMAs with the weight operand in TMEM 46% (measured with the
// library's tensor-pipe probe).  Two 256-column accumulator buffers fill the
// 512 TMEM columns, so the unpacked weights live in shared memory, written by
// the worker threads in the MMA's 128-byte-swizzled K-major layout.
//
// Data flow per pipeline stage (one 128-wide K block):
//   HBM --TMA--> packed int4 box [128 n][64 B]                   (W ring, 4 slots)
//   L2  --TMA--> token codes [256 m][128 B] (128-byte swizzle)   (X ring, 3 slots)
//   16 worker warps: packed int4 -> int8, stored with the swizzle (A ring, 2 slots)
//   tcgen05.mma.kind::i8 (A and B from shared memory) x 4, accumulating the
//   group's P_g in one of two TMEM buffers [128 lanes][256 columns]
//   the same worker warps, per group: tcgen05.ld P_g (32 lanes x 64 columns
//   each), acc += S[g,n] * P_g (or accf += s_g * float(P_g)); after the tile's
//   last group y = acc * s_a[m] / alpha staged in shared memory and stored by
//   TMA (a dense layer) or by one bulk copy per output row (routed rows of a
//   mixture-of-experts layer).
// The worker warps keep the unpack one stage ahead of the drain, so the MMAs
// of the next group run while they drain the current one.
//
// Work partition: stream-K over (tile, group) steps as in the narrow-tile
// kernel, with the same split-tile combine through the workspace.  A
// mixture-of-experts call (MOE) orders tiles expert by expert; its per-expert
// tile counts, weight tensor maps and range sizes are computed on the device
// by moe_setup_kernel from the routing offsets, so no host sync is needed.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm_common.cuh"
#include "gemm_w4a8.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace gemm {
namespace wide {

#ifndef W4A8_WIDE_BT
#define W4A8_WIDE_BT 192
#endif
constexpr int kTileN = 128;                       // weight columns per tile (MMA M)
constexpr int kBT = W4A8_WIDE_BT;                 // tokens per tile (MMA N): 192 or 256
#ifndef W4A8_WIDE_WORKERS
#define W4A8_WIDE_WORKERS 12
#endif
constexpr int kWorkers = W4A8_WIDE_WORKERS;       // warps 2.., each 32 lanes x kHC token columns
constexpr int kWorkerThreads = 32 * kWorkers;
constexpr int kThreads = 32 * (2 + kWorkers);
constexpr int kHC = kBT / (kWorkers / 4);         // accumulator columns per worker thread
#ifndef W4A8_WIDE_DRAIN_COLS
#define W4A8_WIDE_DRAIN_COLS 16
#endif
constexpr int kDrainCols = W4A8_WIDE_DRAIN_COLS;  // TMEM columns per drain load
constexpr int SW = 4, SA = 2, SX = (kBT == 256 ? 3 : 4), SD = 8, kAcc = 2;
constexpr int kWBytes = kTileN * 64;              // packed weights of one K block
constexpr int kABytes = kTileN * 128;             // unpacked operand of one K block
constexpr int kXBytes = kBT * 128;                // token codes of one K block
constexpr int kYBytes = kBT * kTileN * 2;         // output staging: all rows as fp16, or kHC rows of 4-byte words
constexpr int offW = 0;
constexpr int offA = offW + SW * kWBytes;
constexpr int offX = offA + SA * kABytes;
constexpr int offY = offX + SX * kXBytes;
constexpr int offSA = offY + kYBytes;             // the tile's output scales (one per token row)
constexpr int offOK = offSA + kBT * 4;            // MOE: whether each row's token index is in range
constexpr int offBar = offOK + kBT * 4;
constexpr int kBars = 2 * SW + SA + SX + SD + 2 * kAcc + 1;
constexpr int offMisc = offBar + kBars * 8;
constexpr int kSmemBytes = offMisc + 64 + 1024;  // + slack to align the base to 1024
static_assert(offA % 1024 == 0 && offX % 1024 == 0 && offY % 1024 == 0, "swizzle atoms and TMA sources");
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kHC % 16 == 0 && kBT % kHC == 0 && kTileN * kHC * 4 <= kYBytes, "output staging");
static_assert(2 * kBT <= 512 && kWorkers % 4 == 0, "TMEM: two accumulator buffers of kBT columns");

// Step range of CTA b from the (W, w_q, w_r) of the call: [start(b),
// start(b + 1)).  CTAs at or past `grid` (a grouped call launches one per SM
// and may have fewer steps than that) get the empty range [W, W).
struct Range {
    uint32_t W, w_q, w_r, grid;
    __device__ uint32_t start(uint32_t b) const {
        const uint32_t c = b < grid ? b : grid;
        return c * w_q + (c * w_r) / grid;
    }
    __device__ uint32_t owner(uint32_t i) const {
        uint32_t o = uint32_t((double(i) + 1.0) * double(grid) / double(W));
        if (o >= grid) o = grid - 1;
        while (o > 0 && start(o) > i) --o;
        while (o + 1 < grid && start(o + 1) <= i) ++o;
        return o;
    }
};

// Per-expert schedule of a mixture-of-experts call, in global memory (written
// by moe_setup_kernel after W, W / g, W % g and the CTAs g that take ranges):
// m_tiles[e], the first tile tstart[e] and the first routed row rstart[e] of
// every expert, with one entry past the last.
struct Sched {
    const int32_t* mt;
    const int32_t* tstart;
    const int32_t* rstart;
    int32_t E;
};

__device__ __forceinline__ Sched sched_of(const WideParams& p) {
    const int32_t* base = p.moe_sched + 4;
    return Sched{base, base + (p.E + 1), base + 2 * (p.E + 1), p.E};
}

template <bool MOE>
__device__ __forceinline__ Range range_of(const WideParams& p) {
    if constexpr (MOE)
        return Range{uint32_t(p.moe_sched[0]), uint32_t(p.moe_sched[1]), uint32_t(p.moe_sched[2]),
                     uint32_t(p.moe_sched[3])};
    else
        return Range{p.W, p.w_q, p.w_r, uint32_t(p.grid)};
}

struct WSeg {
    uint32_t tile;  // global tile index (expert-major for MOE)
    int32_t e, n_tile, m_tile, g0, g1;
};

// Segments of CTA b in order: tiles expert by expert, then by weight-column
// tile, then by token tile; each segment a run of groups of one tile.
template <bool MOE>
struct WIter {
    uint32_t i, end, tile;
    int32_t G, g, e, n_tile, m_tile, mt, n_tiles;
    Sched sc;
    __device__ WIter(const WideParams& p, const Range& r, uint32_t b) {
        G = p.G;
        n_tiles = p.n_tiles;
        i = r.start(b);
        end = r.start(b + 1);
        tile = i / uint32_t(G);
        g = int32_t(i - tile * uint32_t(G));
        uint32_t local = tile;
        e = 0;
        if constexpr (MOE) {
            sc = sched_of(p);
            if (i < end) {
                while (e + 1 < sc.E && uint32_t(sc.tstart[e + 1]) <= tile) ++e;
                local = tile - uint32_t(sc.tstart[e]);
                mt = sc.mt[e];
            } else {
                mt = 1;
            }
        } else {
            mt = p.m_tiles;
        }
        n_tile = int32_t(local / uint32_t(mt));
        m_tile = int32_t(local - uint32_t(n_tile) * uint32_t(mt));
    }
    __device__ bool next(WSeg& s) {
        if (i >= end) return false;
        s.tile = tile;
        s.e = e;
        s.n_tile = n_tile;
        s.m_tile = m_tile;
        s.g0 = g;
        const uint32_t left = end - i;
        s.g1 = (left >= uint32_t(G - g)) ? G : g + int32_t(left);
        i += s.g1 - s.g0;
        if (s.g1 == G) {
            g = 0;
            ++tile;
            if (++m_tile == mt) {
                m_tile = 0;
                if (++n_tile == n_tiles) {
                    n_tile = 0;
                    if constexpr (MOE) {
                        if (i < end) {  // the next expert with rows
                            do {
                                ++e;
                            } while (e + 1 < sc.E && sc.mt[e] == 0);
                            mt = sc.mt[e];
                        }
                    }
                }
            }
        } else {
            g = s.g1;
        }
        return true;
    }
};

// Pipeline stages (one K block each) in the order every role walks them.
struct WStage {
    int32_t e, n_tile, m_tile, kb;
    bool first_of_seg;
};

template <bool MOE>
struct WStageIter {
    WIter<MOE> seg;
    int32_t kbpg, e = 0, n_tile = 0, m_tile = 0, kb = 0, kb_end = 0;
    __device__ WStageIter(const WideParams& p, const Range& r, uint32_t b) : seg(p, r, b), kbpg(p.kb_per_group) {}
    __device__ bool next(WStage& st) {
        st.first_of_seg = false;
        if (kb >= kb_end) {
            WSeg s;
            if (!seg.next(s)) return false;
            e = s.e;
            n_tile = s.n_tile;
            m_tile = s.m_tile;
            kb = s.g0 * kbpg;
            kb_end = s.g1 * kbpg;
            st.first_of_seg = true;
        }
        st.e = e;
        st.n_tile = n_tile;
        st.m_tile = m_tile;
        st.kb = kb++;
        return true;
    }
};

template <int PATH, bool MOE>
__global__ void __launch_bounds__(kThreads, 1)
    w4a8_gemm_wide_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_y, const WideParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + offBar);
    uint64_t* full_w = bars;             // packed box landed (transaction count)
    uint64_t* empty_w = full_w + SW;     // every worker warp has read the packed box
    uint64_t* full_a = empty_w + SW;     // every worker warp has written its part of the unpacked operand
    uint64_t* full_x = full_a + SA;      // token codes landed
    uint64_t* sdone = full_x + SX;       // all MMAs of a stage complete
    uint64_t* tempty = sdone + SD;       // every worker warp has read an accumulator buffer
    uint64_t* afull = tempty + kAcc;     // a group's MMAs into an accumulator buffer are complete
    uint64_t* mma_done = afull + kAcc;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + offMisc);  // [0] tmem base [1] abort [2] combine ok
    volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);
    float* sa_tile = reinterpret_cast<float*>(smem + offSA);
    int32_t* ok_tile = reinterpret_cast<int32_t*>(smem + offOK);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SW; ++s) {
            mbar_init(&full_w[s], 1);
            mbar_init(&empty_w[s], kWorkers);
        }
        for (int s = 0; s < SA; ++s) mbar_init(&full_a[s], kWorkers);
        for (int s = 0; s < SX; ++s) mbar_init(&full_x[s], 1);
        for (int s = 0; s < SD; ++s) mbar_init(&sdone[s], 1);
        for (int s = 0; s < kAcc; ++s) {
            mbar_init(&tempty[s], kWorkers);
            mbar_init(&afull[s], 1);
        }
        mbar_init(&mma_done[0], 1);
        misc[1] = 0;
        misc[2] = 0;
        fence_mbar_init();
        if constexpr (!MOE) prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
        if constexpr (!MOE) prefetch_tensormap(&tm_y);
    }
    if (warp == 1) tmem_alloc(&misc[0], 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const uint32_t b = blockIdx.x;
    if (threadIdx.x == 0) griddep_launch_dependents();
    // A mixture-of-experts call reads its schedule and tensor maps, written by
    // the setup kernel launched just before it: every role waits for it first.
    if constexpr (MOE) griddep_wait();
    const Range range = range_of<MOE>(p);

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        Ring rw, rx, rxd;
        int32_t pst = 0;
        uint32_t w_issued = 0u, w_par = 0u, x_issued = 0u, x_par = 0u;
        int32_t prefetched = 0;
        const CUtensorMap* wmap = &tm_w;
        int32_t wmap_e = -1;
        auto issue_w = [&](const WStage& st, const Ring& slot) {
            mbar_arrive_expect_tx_one(&full_w[slot.idx], uint32_t(kWBytes));
            tma_load_2d_one(smem + offW + slot.idx * kWBytes, wmap, st.kb * 64, st.n_tile * kTileN, &full_w[slot.idx]);
            w_issued |= 1u << slot.idx;
            w_par = (w_par & ~(1u << slot.idx)) | (slot.phase << slot.idx);
        };
        if constexpr (!MOE) {
            // the first stages' packed weights before waiting for the previous
            // kernel (packed weights are never written by a kernel that lets its
            // successor start early)
            WStageIter<MOE> it(p, range, b);
            WStage st;
            while (prefetched < 2 && it.next(st)) {
                issue_w(st, rw);
                rw.advance(SW);
                ++prefetched;
            }
            rw = Ring{};
            griddep_wait();  // the token codes may be the previous kernel's output
        }
        // token rows of the current tile (MOE: gathered by routed row)
        int32_t trow[8];
        WStageIter<MOE> it(p, range, b);
        WStage st;
        bool ok = true;
        while (ok && it.next(st)) {
            if constexpr (MOE) {
                if (st.e != wmap_e) {  // this expert's weight tensor map
                    wmap = p.moe_maps + st.e;
                    wmap_e = st.e;
                    tensormap_acquire(wmap);
                }
                if (st.first_of_seg) {
                    const Sched sc = sched_of(p);
                    const int32_t r0 = sc.rstart[st.e] + st.m_tile * kBT;
                    const int32_t r1 = sc.rstart[st.e + 1];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        // lane l gathers rows 4l..4l+3 and 128+4l..128+4l+3 (those
                        // below kBT); rows past the expert's last take token 0
                        // (never stored)
                        const int32_t rt = (q >> 2) * 128 + 4 * lane + (q & 3);
                        const int32_t r = r0 + rt;
                        const int32_t tk = (rt < kBT && r < r1) ? p.row_index[r] : 0;
                        trow[q] = (tk >= 0 && tk < p.moe_T) ? tk : 0;  // out of range: checked by the workers
                    }
                }
            }
            if (pst >= prefetched) {
                if (!mbar_wait_warp(&empty_w[rw.idx], rw.phase ^ 1u, abort_flag, p.status, p.wait_limit)) {
                    ok = false;
                    break;
                }
                issue_w(st, rw);
            }
            rw.advance(SW);
            if (pst >= SX) {  // the MMAs of stage pst - SX have read this token slot
                if (!mbar_wait_warp(&sdone[rxd.idx], rxd.phase, abort_flag, p.status, p.wait_limit)) {
                    ok = false;
                    break;
                }
                rxd.advance(SD);
            }
            uint8_t* xdst = smem + offX + rx.idx * kXBytes;
            mbar_arrive_expect_tx_one(&full_x[rx.idx], uint32_t(kXBytes));
            if constexpr (MOE) {
                __syncwarp();
                tma_gather4(xdst + 4 * lane * 128, &tm_x, st.kb * 128, trow[0], trow[1], trow[2], trow[3],
                            &full_x[rx.idx]);
                if (128 + 4 * lane < kBT)
                    tma_gather4(xdst + (128 + 4 * lane) * 128, &tm_x, st.kb * 128, trow[4], trow[5], trow[6],
                                trow[7], &full_x[rx.idx]);
            } else {
                tma_load_2d_one(xdst, &tm_x, st.kb * 128, st.m_tile * kBT, &full_x[rx.idx]);
            }
            x_issued |= 1u << rx.idx;
            x_par = (x_par & ~(1u << rx.idx)) | (rx.phase << rx.idx);
            rx.advance(SX);
            ++pst;
        }
        if (!ok && lane == 0) {  // let copies in flight land before the CTA leaves
            for (int s = 0; s < SW; ++s)
                if (w_issued & (1u << s)) drain_wait(&full_w[s], (w_par >> s) & 1u);
            for (int s = 0; s < SX; ++s)
                if (x_issued & (1u << s)) drain_wait(&full_x[s], (x_par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = idesc_i8(kTileN, kBT);
        Ring ra, rx, rt, rd;
        WStageIter<MOE> it(p, range, b);
        WStage st;
        bool ok = true;
        int32_t kin = 0;  // position of the next K block inside its group
        const uint32_t a_lo0 = smem_desc_sw128_lo(smem_u32(smem + offA));
        const uint32_t x_lo0 = smem_desc_sw128_lo(smem_u32(smem + offX));
        while (ok && it.next(st)) {
            if (!mbar_wait_warp(&full_a[ra.idx], ra.phase, abort_flag, p.status, p.wait_limit) ||
                !mbar_wait_warp(&full_x[rx.idx], rx.phase, abort_flag, p.status, p.wait_limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool first = (kin == 0);
            const bool last = (kin == p.kb_per_group - 1);
            kin = last ? 0 : kin + 1;
            if (first) {
                if (!mbar_wait_warp(&tempty[rt.idx], rt.phase ^ 1u, abort_flag, p.status, p.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            const uint32_t d = tmem_base + uint32_t(rt.idx * kBT);
            const uint32_t a_lo = a_lo0 + uint32_t(ra.idx) * uint32_t(kABytes >> 4);
            const uint32_t x_lo = x_lo0 + uint32_t(rx.idx) * uint32_t(kXBytes >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)  // 32 K per MMA: 2 descriptor units of A and of B
                mma_i8_ss_one(d, smem_desc_from_lo(a_lo + 2u * k), smem_desc_from_lo(x_lo + 2u * k), idesc,
                              (first && k == 0) ? 0u : 1u);
            if (last) {
                mma_commit_one(&afull[rt.idx]);
                rt.advance(kAcc);
            }
            mma_commit_one(&sdone[rd.idx]);
            ra.advance(SA);
            rx.advance(SX);
            rd.advance(SD);
        }
        mma_commit_one(&mma_done[0]);  // every MMA issued has finished before TMEM is released
        if (lane == 0) drain_wait(&mma_done[0], 0);
        __syncwarp();
    } else {
        // ---------------------------------------------------------- workers: unpack, drain, tail
        if constexpr (!MOE) griddep_wait();  // s_a, y and the workspace may be in use by the previous kernel
        const int wi = warp - 2;             // 0..15
        const int quarter = warp & 3;        // TMEM lanes this warp may access
        const int h = wi >> 2;               // which 64 of the 256 token columns
        const int r = quarter * 32 + lane;   // TMEM lane = weight row of the tile
        const int t = wi * 32 + lane;        // 0..511
        constexpr bool kX16 = (PATH == kFloatScale);  // float path: 16 q, the 1/16 folded into s_g
        const int32_t N = p.N;
        const Sched sc = MOE ? sched_of(p) : Sched{nullptr, nullptr, nullptr, 0};

        // ---- unpack, one stage ahead of the drain
        WStageIter<MOE> uit(p, range, b);
        WStage ust;
        bool u_more = uit.next(ust);
        Ring uw, ua, uad;
        int32_t n_unpacked = 0;
        // A K block's packed weights are 512 chunks of 16 bytes (128 rows x 4);
        // worker thread t unpacks chunks t, t + kWorkerThreads, ...
        constexpr int kChunks = kTileN * 4;
        constexpr int kChunkIters = (kChunks + kWorkerThreads - 1) / kWorkerThreads;
        bool ok = true;
        auto unpack_next = [&]() -> bool {
            if (!u_more) return true;
            if (!mbar_wait_warp(&full_w[uw.idx], uw.phase, abort_flag, p.status, p.wait_limit)) return false;
            uint4 pk[kChunkIters];
#pragma unroll
            for (int ci = 0; ci < kChunkIters; ++ci) {
                const int ch = t + ci * kWorkerThreads;
                if (ch < kChunks) pk[ci] = *reinterpret_cast<const uint4*>(smem + offW + uw.idx * kWBytes + ch * 16);
            }
            __syncwarp();
            mbar_arrive_one(&empty_w[uw.idx]);
            uw.advance(SW);
            if (n_unpacked >= SA) {  // the MMAs of stage n - SA have read this operand slot
                if (!mbar_wait_warp(&sdone[uad.idx], uad.phase, abort_flag, p.status, p.wait_limit)) return false;
                uad.advance(SD);
            }
#pragma unroll
            for (int ci = 0; ci < kChunkIters; ++ci) {
                const int ch = t + ci * kWorkerThreads;
                if (ch < kChunks) {
                    // packed row ur, chunk uc (32 K values) -> bytes [32 uc, 32 uc + 32) of
                    // the operand's row ur: 16-byte chunks 2 uc and 2 uc + 1, swizzled
                    const int ur = ch >> 2, uc = ch & 3;
                    uint8_t* arow = smem + offA + ua.idx * kABytes + (ur >> 3) * 1024 + (ur & 7) * 128;
                    const uint2 o0 = unpack8<kX16>(pk[ci].x), o1 = unpack8<kX16>(pk[ci].y);
                    const uint2 o2 = unpack8<kX16>(pk[ci].z), o3 = unpack8<kX16>(pk[ci].w);
                    *reinterpret_cast<uint4*>(arow + (((2 * uc) ^ (ur & 7)) << 4)) = make_uint4(o0.x, o0.y, o1.x, o1.y);
                    *reinterpret_cast<uint4*>(arow + (((2 * uc + 1) ^ (ur & 7)) << 4)) =
                        make_uint4(o2.x, o2.y, o3.x, o3.y);
                }
            }
            fence_proxy_async_smem();  // the operand, visible to the tensor core
            __syncwarp();
            mbar_arrive_one(&full_a[ua.idx]);
            ua.advance(SA);
            ++n_unpacked;
            u_more = uit.next(ust);
            return true;
        };
        ok = unpack_next();

        // ---- per-group drain and per-tile tail
        Ring rt;
        WIter<MOE> it(p, range, b);
        WSeg sg;
        const int32_t kbpg = p.kb_per_group;
        const int32_t G = p.G;
        const uint32_t lane_cols = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(h * kHC);
        while (ok && it.next(sg)) {
            const int32_t n0 = sg.n_tile * kTileN;
            const int32_t n = n0 + r;
            const bool nvalid = n < N;
            // rows of this tile: dense tokens m0.., or routed rows rbase.. of expert e
            int32_t rows_valid, rbase = 0;
            const int16_t* S = p.S;
            if constexpr (MOE) {
                rbase = sc.rstart[sg.e] + sg.m_tile * kBT;
                rows_valid = sc.rstart[sg.e + 1] - rbase;
                S = reinterpret_cast<const int16_t*>(p.moe_scales[sg.e]);
            } else {
                rows_valid = p.M - sg.m_tile * kBT;
            }
            if (rows_valid > kBT) rows_valid = kBT;
            // output scale of token (tile start + t) for t < 256, handed to the tail through shared memory
            float sa_pref = 0.0f;
            int32_t ok_pref = 1;
            if (t < kBT && t < rows_valid) {
                int32_t tok;
                bool tok_ok = true;
                if constexpr (MOE) {
                    tok = p.row_index[rbase + t];
                    tok_ok = tok >= 0 && tok < p.moe_T;
                    if (!tok_ok) atomicExch(p.status, 1);  // W4A8_ERR_INVALID_ARG: the row's outputs are zero
                } else {
                    tok = sg.m_tile * kBT + t;
                }
                const float sa = tok_ok ? p.s_a[tok] : 0.0f;
                sa_pref = PATH == kIntScale ? __fmul_rn(sa, p.inv_alpha) : sa;
                ok_pref = tok_ok ? 1 : 0;
            }
            int32_t acc[kHC];
            float accf[kHC];
#pragma unroll
            for (int j = 0; j < kHC; ++j) {
                acc[j] = 0;
                accf[j] = 0.0f;
            }
            // this column's scales, read two groups ahead (a column past N reads
            // column 0's: its outputs are never stored)
            const int32_t n_ld = nvalid ? n : 0;
            int32_t sidx = sg.g0 * N + n_ld;
            auto ld_scale = [&](int32_t i) -> uint32_t {
                if constexpr (PATH == kIntScale)
                    return uint32_t(int32_t(__ldg(S + i)));
                else
                    return __float_as_uint(__ldg(p.s_g + i));
            };
            uint32_t s1 = ld_scale(sidx);
            sidx += N;
            uint32_t s2 = (sg.g0 + 1 < sg.g1) ? ld_scale(sidx) : 0u;
            sidx += N;
            for (int32_t g = sg.g0; g < sg.g1; ++g) {
                for (int32_t k = 0; k < kbpg; ++k) {
                    if (!unpack_next()) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                const uint32_t sraw = s1;
                s1 = s2;
                if (g + 2 < sg.g1) s2 = ld_scale(sidx);
                sidx += N;
                if (!mbar_wait_warp(&afull[rt.idx], rt.phase, abort_flag, p.status, p.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < kHC / kDrainCols; ++hh) {
                    uint32_t v[kDrainCols];
                    tmem_load<kDrainCols>(lane_cols + uint32_t(rt.idx * kBT + hh * kDrainCols), v);
                    tmem_wait_ld();
                    if constexpr (PATH == kIntScale) {
                        const int32_t s_cur = int32_t(sraw);
#pragma unroll
                        for (int q = 0; q < kDrainCols; ++q) acc[hh * kDrainCols + q] += s_cur * int32_t(v[q]);
                    } else {
                        const float f_cur = __fmul_rn(__uint_as_float(sraw), 0.0625f);  // P_g was 16 P_g
#pragma unroll
                        for (int q = 0; q < kDrainCols; ++q)
                            accf[hh * kDrainCols + q] =
                                __fmaf_rn(f_cur, __int2float_rn(int32_t(v[q])), accf[hh * kDrainCols + q]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                mbar_arrive_one(&tempty[rt.idx]);
                rt.advance(kAcc);
            }
            if (!ok) break;

            // valid token columns of this thread's share (split-tile partials)
            const int nv = rows_valid - h * kHC >= kHC ? kHC : (rows_valid - h * kHC > 0 ? rows_valid - h * kHC : 0);
            const bool whole = (sg.g0 == 0 && sg.g1 == G);
            const int64_t slot_elems = int64_t(kTileN) * kBT;
            if (!whole) {
                // split tile: the tile's first contributor combines (as in the
                // narrow-tile kernel); the others store their partial and signal
                const uint32_t t0 = sg.tile * uint32_t(G);
                const uint32_t b_first = range.owner(t0);
                const uint32_t b_last = range.owner(t0 + uint32_t(G) - 1u);
                if (b != b_first) {
                    int32_t* part = p.ws_part + int64_t(b) * slot_elems + int64_t(h * kHC) * kTileN + r;
#pragma unroll
                    for (int j = 0; j < kHC; ++j)
                        if (j < nv) part[j * kTileN] = PATH == kIntScale ? acc[j] : __float_as_int(accf[j]);
                    epi_bar_sync(kWorkerThreads);  // the CTA's partial stores, before the arrival
                    if (t == 0) red_release_gpu_add(&p.ws_count[b_first], 1);
                    continue;
                }
                if (t == 0) {
                    const int expect = int(b_last - b_first);
                    const long long w0 = clock64();
                    int ok_wait = 1;
                    while (ld_acquire_gpu(&p.ws_count[b_first]) < expect) {
                        if (*abort_flag || clock64() - w0 > p.wait_limit) {
                            *abort_flag = 1;
                            atomicExch(p.status, kStatusTimeout);
                            ok_wait = 0;
                            break;
                        }
                        __nanosleep(64);
                    }
                    misc[2] = uint32_t(ok_wait);
                }
                epi_bar_sync(kWorkerThreads);
                if (!misc[2]) {
                    ok = false;
                    break;
                }
                for (uint32_t c = b_first + 1; c <= b_last; ++c) {
                    const int32_t* cp = p.ws_part + int64_t(c) * slot_elems + int64_t(h * kHC) * kTileN + r;
#pragma unroll
                    for (int j = 0; j < kHC; ++j) {
                        if (j < nv) {
                            const int32_t v = __ldcg(cp + j * kTileN);
                            if (PATH == kIntScale)
                                acc[j] += v;
                            else
                                accf[j] = __fadd_rn(accf[j], __int_as_float(v));
                        }
                    }
                }
                epi_bar_sync(kWorkerThreads);  // every thread has read the partials before the counter is reused
                if (t == 0) p.ws_count[b_first] = 0;
            }

            // ---- the tile's outputs, converted and staged in shared memory as
            // [tokens][128 columns]: fp16 in one pass of 256 rows, 4-byte
            // outputs in two passes of 128 rows; stored by TMA (dense) or by
            // one bulk copy per routed row (MOE)
            const bool leader_warp = (wi == 0);
            if (leader_warp) bulk_wait_read_all();  // the previous tile's stores have read the staging buffer
            epi_bar_sync(kWorkerThreads);
            if (t < kBT) {
                sa_tile[t] = sa_pref;
                ok_tile[t] = ok_pref;
            }
            epi_bar_sync(kWorkerThreads);
            const int esz = p.y_dtype == kOutF16 ? 2 : 4;
            const int rows = esz == 2 ? kBT : kHC;  // rows per pass: all, or one worker group's kHC
            const int passes = kBT / rows;
            for (int pass = 0; pass < passes; ++pass) {
                const int tok0 = pass * rows;  // first token of this pass
                if (h * kHC >= tok0 && h * kHC < tok0 + rows) {
                    const float* sa = sa_tile + h * kHC;
                    const int base = (h * kHC - tok0) * kTileN + r;
                    if (p.y_dtype == kOutI32) {
                        int32_t* yo = reinterpret_cast<int32_t*>(smem + offY) + base;
                        const int32_t* okr = ok_tile + h * kHC;
#pragma unroll
                        for (int j = 0; j < kHC; ++j) yo[j * kTileN] = (!MOE || okr[j]) ? acc[j] : 0;
                    } else if (p.y_dtype == kOutF16) {
                        __half* yo = reinterpret_cast<__half*>(smem + offY) + base;
#pragma unroll
                        for (int j = 0; j < kHC; ++j)
                            yo[j * kTileN] = __float2half_rn(
                                __fmul_rn(PATH == kIntScale ? __int2float_rn(acc[j]) : accf[j], sa[j]));
                    } else {
                        float* yo = reinterpret_cast<float*>(smem + offY) + base;
#pragma unroll
                        for (int j = 0; j < kHC; ++j)
                            yo[j * kTileN] = __fmul_rn(PATH == kIntScale ? __int2float_rn(acc[j]) : accf[j], sa[j]);
                    }
                }
                fence_proxy_async_smem();  // the staged outputs, visible to the bulk copies
                epi_bar_sync(kWorkerThreads);
                if constexpr (MOE) {
                    if (leader_warp) {
                        const int ncols = N - n0 < kTileN ? N - n0 : kTileN;
                        const uint32_t bytes = uint32_t(ncols * esz);
                        for (int q = lane; q < rows; q += 32) {
                            const int tok = tok0 + q;
                            if (tok < rows_valid) {
                                const int32_t rr = rbase + tok;
                                const int64_t orow = p.out_row ? int64_t(p.out_row[rr]) : int64_t(rr);
                                if (orow >= 0 && orow < p.y_rows) {
                                    uint8_t* dst = static_cast<uint8_t*>(p.y) + (orow * N + n0) * esz;
                                    bulk_store(dst, smem + offY + q * kTileN * esz, bytes);
                                } else {
                                    atomicExch(p.status, 1);  // W4A8_ERR_INVALID_ARG: output row out of range
                                }
                            }
                        }
                        bulk_commit_group();
                    }
                } else {
                    if (t == 0) {
                        tma_store_2d(&tm_y, smem + offY, n0, sg.m_tile * kBT + tok0);
                        bulk_commit_group();
                    }
                }
                if (pass + 1 < passes) {  // the next pass reuses the staging buffer
                    if (leader_warp) bulk_wait_read_all();
                    epi_bar_sync(kWorkerThreads);
                }
            }
        }
        if (wi == 0) bulk_wait_read_all();  // shared memory stays until the stores have read it
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace wide
}  // namespace gemm
}  // namespace w4a8

// ------------------------------------------------------------------ mixture-of-experts setup

namespace w4a8 {
namespace gemm {
namespace wide {

// One CTA: validates the routing offsets, writes the per-expert schedule
// (m_tiles, first tile, first row) and the call's step range (W, W / grid,
// W % grid) into `sched`, and builds every expert's weight tensor map from
// the template by replacing its global address.  Offsets that are not
// non-decreasing from 0 to R, or a step count beyond 2^31, make the GEMM do
// nothing (W = 0) and set W4A8_ERR_INVALID_ARG in the device status word.
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

template <int PATH, bool MOE>
static cudaError_t launch_t(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty, const WideParams& p,
                            cudaStream_t stream) {
    constexpr auto kern = w4a8_gemm_wide_kernel<PATH, MOE>;
    const cudaError_t e = configure_once<kern>(kThreads, kSmemBytes);
    if (e != cudaSuccess) return e;
    const LaunchPdl lc(unsigned(p.grid), kThreads, size_t(kSmemBytes), stream);
    return cudaLaunchKernelEx(&lc.cfg, kern, tw, tx, ty, p);
}

}  // namespace wide

cudaError_t launch_wide(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const CUtensorMap& tm_y, const WideParams& p,
                        int path, cudaStream_t stream) {
    return path == kIntScale ? wide::launch_t<kIntScale, false>(tm_w, tm_x, tm_y, p, stream)
                             : wide::launch_t<kFloatScale, false>(tm_w, tm_x, tm_y, p, stream);
}

cudaError_t launch_grouped_setup(const CUtensorMap& tm_w_template, const int64_t* offsets, const void* const* w_ptrs,
                                 const void* const* s_ptrs, int32_t E, int64_t R, int32_t bt, int32_t n_tiles,
                                 int32_t G, int32_t grid, int32_t* sched, CUtensorMap* maps, int* status,
                                 cudaStream_t stream) {
    const LaunchPdl lc(1u, 256, 0, stream);
    return cudaLaunchKernelEx(&lc.cfg, wide::moe_setup_kernel, tm_w_template, offsets, w_ptrs, s_ptrs, E, R, bt,
                              n_tiles, G, grid, sched, maps, status);
}

cudaError_t launch_wide_moe(const CUtensorMap& tm_w_template, const CUtensorMap& tm_x, const int64_t* offsets,
                            const void* const* w_ptrs, int64_t R, const WideParams& p, int32_t* sched,
                            CUtensorMap* maps, cudaStream_t stream) {
    const cudaError_t e = launch_grouped_setup(tm_w_template, offsets, w_ptrs, p.moe_scales, p.E, R, wide::kBT,
                                               p.n_tiles, p.G, p.grid, sched, maps, p.status, stream);
    if (e != cudaSuccess) return e;
    return wide::launch_t<kIntScale, true>(tm_w_template, tm_x, tm_w_template, p, stream);
}

int wide_token_tile() { return wide::kBT; }

int wide_tail_rows() { return wide::kHC; }

}  // namespace gemm
}  // namespace w4a8
