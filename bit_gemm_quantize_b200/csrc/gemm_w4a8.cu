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
// Data flow per pipeline stage (256 consecutive K):
//   HBM --TMA--> packed int4 box [128 n][128 B] (128-byte swizzle)      (W ring, smem)
//   HBM --TMA--> token codes [BT m][128 k] x2 (128-byte swizzle)        (X ring, smem)
//   unpack warps (one thread per weight row = TMEM lane): packed int4 ->
//   int8, written with tcgen05.st as the MMA's A operand, 64 TMEM columns
//   of 4 K values each                                                  (A ring, TMEM)
//   tcgen05.mma.kind::i8, A from TMEM, B = token codes from smem, K = 32
//   each, accumulating one group's P_g in a TMEM buffer [128][BT]       (acc ring, TMEM)
//   epilogue warps per group: this column's S[g,n] (or s_g), loaded from
//   global memory two stages ahead; tcgen05.ld P_g, acc += S[g,n] * P_g (or
//   accf += s_g * float(P_g)); after the tile's last group y = acc * s_a[m]
//   / alpha (or accf * s_a[m]), staged in shared memory and written by one
//   TMA tensor store.
// Folded integer scales (128-token tiles, when every scale the CTA meets is
// small enough for S * q to stay in int8): the unpack writes S[g,n] * q
// instead of q (the stage's scale rows travel with the packed box), the MMAs
// sum the whole segment in one TMEM buffer, and the epilogue reads it once:
// the same integer acc with no per-group drain.
// Keeping the unpacked operand in TMEM instead of shared memory saves two of
// its passes through the shared-memory port (the unpack's store and the MMA's
// read, 64 KB per stage), which bound small-token-tile MMAs at about 40
// cycles each; read from TMEM they take 16 (N = 16) to 64 (N = 128, the full
// int8 rate) cycles.
// The W ring is released by the unpack warps as soon as they have read a
// stage, so the HBM stream only waits on the unpack; the X ring and the A
// ring are released by one tcgen05.commit per stage, after its MMAs.
//
// Work partition: the (tile, group) steps of the whole problem are split into
// one contiguous range per CTA of a persistent grid (stream-K).  A tile whose
// groups fall into several CTAs' ranges is combined through a workspace: its
// first contributor covers the tile's first groups at the end of its own
// range, so it finishes its share last; every other contributor stores its
// partial and signals an arrival counter (indexed by the first contributor,
// which is the first contributor of no other split tile); the first
// contributor waits for them, adds the partials to its own in CTA order and
// writes y.  Integer partials are exact; float partials are summed in a fixed
// order, so results are deterministic.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "gemm_common.cuh"
#include "gemm_w4a8.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace w4a8 {
namespace gemm {

constexpr int kTileN = 128;   // weight columns per tile (MMA M)
constexpr int kBlockK = 128;  // K per MMA block (one 128-byte swizzle row of int8 token codes)
constexpr int kStageK = 256;  // K per pipeline stage (one 128-byte row of packed int4)
constexpr int kStageCols = kStageK / 4;  // TMEM columns of one stage's A operand (4 int8 per column)
constexpr int64_t kCounterBytes = 4096;  // one int32 arrival counter per CTA, fixed region
constexpr int64_t kMaxGrid = kCounterBytes / 4;

// Epilogue warps (multiples of 4) and TMEM columns per drain load.  Token
// tiles of 64 and 128 use two warpgroups (32 or 64 running sums a thread):
// fewer warps repeat the per-group waits and barrier traffic (measured 2-5%
// faster at 128 than four warpgroups).
#ifndef W4A8_EPI_WARPS
#define W4A8_EPI_WARPS(BT) ((BT) <= 32 ? 4 : 8)
#endif
#ifndef W4A8_DRAIN_CH
#define W4A8_DRAIN_CH 16
#endif
// Token tiles up to which the integer-scale path unpacks to 16*q.
#ifndef W4A8_X16_IS_MAX_BT
#define W4A8_X16_IS_MAX_BT 64
#endif

// Leading stages whose packed weights are requested before waiting on the
// previous kernel (at most the weight ring depth).  Two: the first stage's
// token codes then go out right behind them instead of queueing behind a
// whole ring of weight boxes (measured: 1.4 us less per decode call).  With
// two CTAs per SM (4-stage rings each), three (measured: 0.7 us less).
#ifndef W4A8_PREFETCH
#define W4A8_PREFETCH(CTAS) ((CTAS) == 2 ? 3 : 2)
#endif

#ifndef W4A8_GROUP_COMMIT_MIN_BT
#define W4A8_GROUP_COMMIT_MIN_BT 64
#endif

// CTAs per SM: decode-shaped calls (16-token tiles) run two CTAs per SM,
// each with half of the TMEM and shared memory, so that the two pipelines'
// chains of dependent waits and copies overlap.
#ifndef W4A8_CTAS_PER_SM
#define W4A8_CTAS_PER_SM(BT) ((BT) == 16 ? 2 : 1)
#endif

// Ring depths (stages) of the packed weights and the token codes (per CTA).
#ifndef W4A8_SW
#define W4A8_SW(BT) (W4A8_CTAS_PER_SM(BT) == 2 ? 4 : ((BT) <= 32 ? 8 : ((BT) == 64 ? 6 : 4)))
#endif
#ifndef W4A8_SX
#define W4A8_SX(BT) (W4A8_CTAS_PER_SM(BT) == 2 ? 3 : ((BT) <= 32 ? 6 : ((BT) == 64 ? 4 : 3)))
#endif

// W8: 8-bit weight codes w8 [N, K] (the W8A8 variant).  The weight box then
// is the MMA's A operand as it stands (read from shared memory through a
// descriptor, like the token codes): no unpack, no TMEM operand slots, and
// the weight slot is released by the stage's MMA commit.
// ZP: asymmetric token codes with a zero point z[m] per token (integer-scale
// path only).  The tile's tail subtracts z[m] * c[n] from the accumulator
// before the rescale, c[n] = sum_g S[g,n] * sum_{k in g} q[k,n] precomputed
// per weight column; nothing else changes.
template <int BT, int PATH, bool W8 = false, bool ZP = false>
struct Cfg {
    // warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2-5 unpack
    // (four consecutive warps cover the four TMEM lane quarters), then the
    // epilogue: each warpgroup covers the 128 lanes for its share of the BT
    // columns (1, 2 or 4 warpgroups: wide tiles split the per-group drain so
    // that each thread keeps fewer running sums and more drains overlap)
    static constexpr int kUnpackWarps = 4;
    static constexpr int kFirstUnpackWarp = 2;
    static constexpr int kFirstEpiWarp = kFirstUnpackWarp + kUnpackWarps;
    static constexpr int kEpiWarps = W4A8_EPI_WARPS(BT);
    static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
    // TMEM (512 columns): kSA unpacked-operand slots of 64 columns, then kAcc
    // accumulator buffers of BT columns.  The MMA may run kAcc - 1 groups
    // ahead of the per-group drain.
    static constexpr bool kW8 = W8;
    static constexpr int kCtasPerSm = W8 ? 1 : W4A8_CTAS_PER_SM(BT);
    static constexpr uint32_t kTmemCols = 512u / uint32_t(kCtasPerSm);  // TMEM columns of this CTA
    static constexpr int kAcc = W8 ? (BT == 128 ? 4 : 8) : (BT == 128 ? 3 : (BT == 64 ? 4 : 8));
    static constexpr int kSA = W8 ? 0
                                  : ((int(kTmemCols) - kAcc * BT) / kStageCols > 6 ? 6
                                                                                    : (int(kTmemCols) - kAcc * BT) / kStageCols);
    static constexpr uint32_t kAccCol0 = uint32_t(kSA * kStageCols);
    static_assert((W8 || kSA >= 2) && kSA * kStageCols + kAcc * BT <= int(kTmemCols), "TMEM budget");
    // Unpack to 16*q (nibble into the high half of each byte, 3 integer ops per
    // 8 weights) instead of q (7 ops).  The float-scale path folds the 1/16 into
    // s_g for free; the integer-scale path pays one shift per output per group
    // (P_g is 16 times the group product exactly).  With 128-token tiles the
    // drain's shifts (32 per 8 weights unpacked) outweigh the cheaper unpack,
    // so the integer path unpacks q exactly there.
    static constexpr bool kX16 = !W8 && ((PATH == kFloatScale) || BT <= W4A8_X16_IS_MAX_BT);
    static constexpr int kWBytes = kTileN * kStageK / (W8 ? 1 : 2);  // weights per stage: 16 KB packed, 32 KB int8
    static constexpr int kXBytes = BT * kStageK;          // token codes per stage
    // Wide token tiles commit every group to its accumulator buffer, so the
    // epilogue drains a group while the MMAs of the next one run; narrow tiles
    // commit once per stage (their drains are short, the extra commits are not).
    static constexpr bool kGroupCommit = BT >= W4A8_GROUP_COMMIT_MIN_BT;
    // Narrow tiles read a split tile's single other partial when their
    // segment starts (registers to spare for it).
    static constexpr bool kEarlyCombine = BT <= 32;
    static constexpr int kSW = W8 ? (BT == 128 ? 2 : (BT == 16 ? 6 : 4)) : W4A8_SW(BT);
    static constexpr int kSX = W8 ? (BT <= 32 ? 6 : (BT == 64 ? 4 : 3)) : W4A8_SX(BT);
    // stage-done ring: one tcgen05.commit per stage, read by every role that
    // recycles a resource of that stage
    static constexpr int kSD = 16;
    static_assert(kSD >= kSX && kSD >= kSA, "stage-done ring shallower than a ring it releases");
    // output staging tile [BT tokens][128 columns] (elements of at most 4
    // bytes) and the tile's output scales, for the TMA store of the tail
    static constexpr int kYBytes = BT * kTileN * 4;
    static constexpr int offW = 0;
    static constexpr int offX = offW + kSW * kWBytes;
    static constexpr int offY = offX + kSX * kXBytes;
    static constexpr int offSA = offY + kYBytes;
    static constexpr int offZ = offSA + BT * 4;                     // the tile's zero points (ZP)
    // integer scales of each weight slot's two K blocks (int16 [2][128]),
    // copied with the packed box, for folding them into the operand: 128-token
    // tiles only (narrow tiles accumulate a segment faster in several buffers,
    // measured), and not on the asymmetric-token path (no room beside its zero
    // points)
    static constexpr bool kScaleRing = PATH == kIntScale && !W8 && !ZP && BT == 128;
    static constexpr int kSSlotBytes = 2 * kTileN * 2;
    static constexpr int offS = offZ + (ZP ? BT * 4 : 0);
    static constexpr int offBar = offS + (kScaleRing ? kSW * kSSlotBytes : 0);
    static_assert(!ZP || PATH == kIntScale, "zero points are applied on the integer-scale path");
    static constexpr int kBars = 2 * kSW + kSX + kSA + 2 * kSD + 2 * kAcc + 2;
    static constexpr int offMisc = offBar + kBars * 8;
    // + up to 1024 bytes of slack to align the base to 1024 (the base of
    // dynamic shared memory is 1024-aligned when nothing precedes it; the
    // kernel checks that the slack it has covers the misalignment it sees)
    static constexpr int kSmemBytes = offMisc + 64 + 1024 <= 227 * 1024 ? offMisc + 64 + 1024 : 227 * 1024;
    static constexpr int kSlack = kSmemBytes - (offMisc + 64);
    static_assert(kXBytes % 2048 == 0, "token stage must hold whole 8-row swizzle atoms per k-block");
    static_assert(offY % 128 == 0, "TMA store source alignment");
    static_assert(kSlack >= 0, "shared memory");
    static_assert(kCtasPerSm == 1 || kSmemBytes * kCtasPerSm <= 227 * 1024, "shared memory for two CTAs per SM");
};

// One contiguous run of groups [g0, g1) of one tile inside a CTA's range.
// Step counts stay below 2^31 (checked on the host), so all index arithmetic
// is 32-bit: a 64-bit division is a long software sequence on the GPU.
struct Segment {
    uint32_t tile;
    int32_t e;  // expert (grouped calls)
    int32_t n_tile, m_tile;
    int32_t g0, g1;
    uint32_t first;  // flattened index of the segment's first step
};

// The stream-K partition of a call's (tile, group) steps over its CTAs:
// W steps, W / grid and W % grid, and the CTAs that take ranges (a grouped
// call reads all four from its schedule, written on the device).
struct Part {
    uint32_t W, w_q, w_r, grid;
};

template <bool GR, typename P>
__device__ __forceinline__ Part part_of(const P& p) {
    if constexpr (GR)
        return Part{uint32_t(p.grp_sched[0]), uint32_t(p.grp_sched[1]), uint32_t(p.grp_sched[2]),
                    uint32_t(p.grp_sched[3])};
    else
        return Part{uint32_t(p.W), p.w_q, p.w_r, uint32_t(p.grid)};
}

// First step of CTA b's range: floor(b * W / grid) = b * (W / grid) + floor(b * (W % grid) / grid).
// CTAs at or past `grid` (a grouped call launches one per SM and may have
// fewer steps than that) get the empty range [W, W).
__device__ __forceinline__ uint32_t range_start(uint32_t b, const Part& pt) {
    const uint32_t c = b < pt.grid ? b : pt.grid;
    return c * pt.w_q + (c * pt.w_r) / pt.grid;
}

// CTA whose range holds step i: the largest b with range_start(b) <= i, from
// a floating-point estimate corrected with exact starts.
__device__ __forceinline__ uint32_t range_owner(uint32_t i, const Part& pt) {
    const uint32_t grid = pt.grid;
    uint32_t o = uint32_t((double(i) + 1.0) * double(grid) / double(pt.W));
    if (o >= grid) o = grid - 1;
    while (o > 0 && range_start(o, pt) > i) --o;
    while (o + 1 < grid && range_start(o + 1, pt) <= i) ++o;
    return o;
}

// Per-expert schedule of a grouped call, after the partition in its
// workspace: m_tiles[E+1], first tile[E+1] and first routed row[E+1].
struct GrSched {
    const int32_t* mt;
    const int32_t* tstart;
    const int32_t* rstart;
};

template <typename P>
__device__ __forceinline__ GrSched grsched_of(const P& p) {
    const int32_t* base = p.grp_sched + 4;
    return GrSched{base, base + (p.E + 1), base + 2 * (p.E + 1)};
}

// Iterates the segments of CTA `b`.  The divisions happen once, at the start
// of the range; afterwards the tile coordinates advance incrementally.  A
// grouped call orders its tiles expert by expert (then by weight-column tile,
// then by token tile), each expert with its own count of token tiles.
template <bool GR>
struct SegmentIter {
    uint32_t i, end, tile;
    int32_t G, g, n_tile, m_tile, m_tiles;
    int32_t e, n_tiles, E;  // grouped calls
    GrSched sc;
    template <typename P>
    __device__ SegmentIter(const P& p, const Part& pt, uint32_t b) {
        G = int32_t(p.G);
        i = range_start(b, pt);
        end = range_start(b + 1, pt);
        tile = i / uint32_t(G);
        g = int32_t(i - tile * uint32_t(G));
        e = 0;
        uint32_t local = tile;
        if constexpr (GR) {
            sc = grsched_of(p);
            E = p.E;
            n_tiles = p.n_tiles;
            m_tiles = 1;
            if (i < end) {
                while (e + 1 < E && uint32_t(sc.tstart[e + 1]) <= tile) ++e;
                local = tile - uint32_t(sc.tstart[e]);
                m_tiles = sc.mt[e];
            }
        } else {
            m_tiles = int32_t(p.m_tiles);
        }
        n_tile = int32_t(local / uint32_t(m_tiles));
        m_tile = int32_t(local - uint32_t(n_tile) * uint32_t(m_tiles));
    }
    __device__ bool next(Segment& s) {
        if (i >= end) return false;
        s.tile = tile;
        s.e = e;
        s.n_tile = n_tile;
        s.m_tile = m_tile;
        s.g0 = g;
        const uint32_t left = end - i;
        s.g1 = (left >= uint32_t(G - g)) ? G : g + int32_t(left);
        s.first = i;
        i += s.g1 - s.g0;
        if (s.g1 == G) {
            g = 0;
            ++tile;
            if (++m_tile == m_tiles) {
                m_tile = 0;
                if constexpr (GR) {
                    if (++n_tile == n_tiles) {
                        n_tile = 0;
                        if (i < end) {  // the next expert with rows
                            do {
                                ++e;
                            } while (e + 1 < E && sc.mt[e] == 0);
                            m_tiles = sc.mt[e];
                        }
                    }
                } else {
                    ++n_tile;
                }
            }
        } else {
            g = s.g1;
        }
        return true;
    }
};

// One pipeline stage: up to two consecutive 128-wide K blocks of one segment.
struct Stage {
    int32_t e;    // expert (grouped calls)
    int32_t n_tile, m_tile;
    int32_t kb;   // first K block (global index along K)
    int32_t nkb;  // 1 or 2
    bool seg_first, seg_last;  // the stage opens / closes its segment
};

template <bool GR>
struct StageIter {
    SegmentIter<GR> seg;
    int32_t kbpg;
    int32_t e = 0, n_tile = 0, m_tile = 0;
    int32_t kb = 0, kb_end = 0;
    template <typename P>
    __device__ StageIter(const P& p, const Part& pt, uint32_t b) : seg(p, pt, b), kbpg(p.kb_per_group) {}
    __device__ bool next(Stage& st) {
        st.seg_first = false;
        while (kb >= kb_end) {
            Segment s;
            if (!seg.next(s)) return false;
            e = s.e;
            n_tile = s.n_tile;
            m_tile = s.m_tile;
            kb = s.g0 * kbpg;
            kb_end = s.g1 * kbpg;
            st.seg_first = true;
        }
        st.e = e;
        st.n_tile = n_tile;
        st.m_tile = m_tile;
        st.kb = kb;
        st.nkb = (kb_end - kb) >= 2 ? 2 : 1;
        kb += st.nkb;
        st.seg_last = kb >= kb_end;
        return true;
    }
};

// Folded integer scales.  When every integer scale S[g,n] a CTA meets lies in
// [0, 16], S * q fits in int8 for every 4-bit code q in [-8, 7] (-8 * 16 =
// -128, 7 * 16 = 112), so the unpack can write the operand S[g,n] * q[k,n]
// instead of q: the MMAs then sum S * q * x over the whole segment in the
// TMEM accumulator, which is the same integer as sum_g S[g,n] * P_g, and the
// per-group drain disappears (one accumulator read per tile instead of one
// per group).  This needs the scales to be integers: a float scale cannot be
// folded into an int8 operand exactly.
// Scales above kFoldMaxS (or negative) keep a CTA on the per-group drain:
// S * q fits in int8 for every 4-bit code q in [-8, 7] up to S = 16, and up
// to S = kFoldMaxS7 for a group whose codes avoid -8 (codes in [-7, 7], the
// default packing).
constexpr int kFoldMaxS = 16;
constexpr int kFoldMaxS7 = 18;

// Whether any of 8 packed codes is -8 (nibble 1000): bit 3 set and bits 0-2
// clear (adding 7 to the low three bits sets bit 3 unless they are zero; no
// carry leaves a nibble).
__device__ __forceinline__ bool has_code_minus8(uint32_t w) {
    const uint32_t low_nonzero = ((w & 0x77777777u) + 0x77777777u) & 0x88888888u;
    return (w & 0x88888888u & ~low_nonzero) != 0u;
}

// The largest of 8 int16 scales read as unsigned 16-bit values.
__device__ __forceinline__ uint32_t scales_max_u16(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0xFFFFu, w[i] >> 16));
    return m;
}

// The CTA's choice, read by every role once the epilogue warps' scan of its
// scales is complete (misc[4]: some scale out of range).
__device__ __forceinline__ bool fold_decision(const uint32_t* misc) {
    return *reinterpret_cast<const volatile uint32_t*>(&misc[4]) == 0u;
}

// S * q for 8 packed codes (low nibbles: K 0-3, high nibbles: K 4-7), as int8
// bytes.  With the offset code u = q + 8 in [0, 15] in each byte, the 32-bit
// word * S + (128 - 8 S) * 0x01010101 equals sum_i (S * q_i + 128) * 256^i
// exactly (mod 2^32, k1 wrapping for S > 16): when every S * q_i lies in
// [-128, 127] each coefficient is a byte in [0, 255], so the result's bytes
// are S * q_i + 128 (any carries of the intermediate product cancel), and
// XOR 0x80 turns each byte from excess-128 into two's complement.
__device__ __forceinline__ uint2 unpack8_folded(uint32_t w, uint32_t s, uint32_t k1) {
    const uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
    const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
    return make_uint2((lo * s + k1) ^ 0x80808080u, (hi * s + k1) ^ 0x80808080u);
}

// Output scale of token m: s_a[m] / alpha (exact: 1/alpha is a power of two)
// for the integer-scale path, s_a[m] for the float-scale path.
template <int PATH>
__device__ __forceinline__ float output_scale(const Params& p, int64_t m) {
    return PATH == kIntScale ? __fmul_rn(p.s_a[m], p.inv_alpha) : p.s_a[m];
}


// G1: the group is one 128-wide K block (group = 128, the method's group
// size), so every K block ends a group; wide token tiles then drain each group
// in a loop with no per-stage bookkeeping.
// GR: a grouped (mixture-of-experts) call: tiles expert by expert from a
// schedule in the workspace, each expert's weights through its own tensor
// map, outputs one row at a time; token rows as blocks of routed-order codes,
// or (GATHER) gathered from q_x by a row index.
template <int BT, int PATH, bool W8, bool ZP, bool G1, bool GR = false, bool GATHER = false>
__global__ void __launch_bounds__(Cfg<BT, PATH, W8, ZP>::kThreads, Cfg<BT, PATH, W8, ZP>::kCtasPerSm)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_y,
                     const std::conditional_t<ZP, ParamsZp, std::conditional_t<GR, ParamsGr, Params>> p) {
    using C = Cfg<BT, PATH, W8, ZP>;
    constexpr bool kLean = G1 && C::kGroupCommit;  // the per-group drain loop below
    constexpr int kAcc = C::kAcc;
    constexpr int kU = C::kUnpackWarps;
    constexpr int SW = C::kSW, SX = C::kSX, SA = C::kSA, SD = C::kSD;
    constexpr int kEpiWarps = C::kEpiWarps;
    constexpr int HC = BT / (kEpiWarps / 4);  // columns per epilogue thread
    // integer scales on 4-bit weights may be folded into the unpacked operand
    constexpr bool kFoldable = C::kScaleRing;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u) > uint32_t(C::kSlack)) {
        // the layout would not fit behind the aligned base: refuse (no
        // barrier, TMEM or copy has been touched yet)
        if (threadIdx.x == 0) atomicExch(p.status, kStatusAlign);
        return;
    }
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::offBar);
    uint64_t* full_w = bars;              // W box landed (TMA transaction count)
    uint64_t* empty_w = full_w + SW;      // unpack warps have read the W box
    uint64_t* full_x = empty_w + SW;      // token codes landed
    uint64_t* full_a = full_x + SX;       // unpacked operand written to its TMEM slot
    uint64_t* sdone = full_a + SA;        // all MMAs of a stage complete (one commit per stage)
    uint64_t* sseen = sdone + SD;         // per-stage commits: the epilogue has seen a stage-done phase
    uint64_t* tempty = sseen + SD;        // epilogue has read a TMEM accumulator buffer
    uint64_t* afull = tempty + kAcc;      // a group's MMAs into an accumulator buffer are complete
    uint64_t* mma_done = afull + kAcc;
    uint64_t* fold_ready = mma_done + 1;  // the epilogue warps have checked the CTA's scales (misc[4])
    // [0] tmem base [1] abort [2] last [3] early combine [4] nonzero: some
    // scale of the CTA's steps cannot be folded
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::offMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(&misc[1]);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SW; ++s) {
            mbar_init(&full_w[s], 1);
            mbar_init(&empty_w[s], kU);
        }
        for (int s = 0; s < SX; ++s) mbar_init(&full_x[s], 1);
        for (int s = 0; s < SA; ++s) mbar_init(&full_a[s], kU);
        for (int s = 0; s < SD; ++s) {
            mbar_init(&sdone[s], 1);
            mbar_init(&sseen[s], kEpiWarps);
        }
        for (int s = 0; s < kAcc; ++s) {
            mbar_init(&tempty[s], kEpiWarps);
            mbar_init(&afull[s], 1);
        }
        mbar_init(&mma_done[0], 1);
        mbar_init(fold_ready, kEpiWarps);
        misc[1] = 0;
        misc[2] = 0;
        misc[4] = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_y);
    }
    if (warp == 1) tmem_alloc(&misc[0], C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const uint32_t b = blockIdx.x;
    // The next kernel in the stream may be scheduled now; it cannot share an
    // SM with this CTA (shared memory), so its CTAs start where ours finish.
    if (threadIdx.x == 0) griddep_launch_dependents();
    // a grouped call's schedule and weight maps come from the setup kernel
    if constexpr (GR) griddep_wait();
    const Part pt = part_of<GR>(p);

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        // The whole warp walks the loop; one elected lane issues the copies.
        // The packed weights of the first stages are requested before
        // waiting for the previous kernel in the stream (this kernel may start
        // early under programmatic dependent launch; packed weights are never
        // written by a kernel that lets its successor start early), so the
        // weight stream is under way by the time the token codes, which that
        // kernel may still be writing, can be read.
        Ring rw, rx;
        Ring rxd;          // stage-done slot of the stage whose token slot is reused (SX stages back)
        Ring rwd;          // int8 weights: stage-done slot of the stage whose weight slot is reused (SW back)
        int32_t pst = 0;   // stages issued so far
        uint32_t w_issued = 0u, w_par = 0u, x_issued = 0u, x_par = 0u;  // per slot: copy issued / its parity
        // the weights' tensor map: one per expert in a grouped call (fetched
        // to the tensor-map proxy when the expert changes)
        const CUtensorMap* wmap = &tm_w;
        int32_t wmap_e = -1;
        auto issue_w = [&](const Stage& st, const Ring& slot) {
            if constexpr (GR) {
                if (st.e != wmap_e) {
                    wmap = p.grp_maps + st.e;
                    wmap_e = st.e;
                    tensormap_acquire(wmap);
                }
            }
            if constexpr (C::kW8) {
                // int8 weights: one 128-row x 128 B box per K block
                uint8_t* dst = smem + C::offW + slot.idx * C::kWBytes;
                mbar_arrive_expect_tx_one(&full_w[slot.idx], uint32_t(st.nkb * kTileN * kBlockK));
                tma_load_2d_one(dst, wmap, st.kb * kBlockK, st.n_tile * kTileN, &full_w[slot.idx]);
                if (st.nkb == 2)
                    tma_load_2d_one(dst + kTileN * kBlockK, wmap, (st.kb + 1) * kBlockK, st.n_tile * kTileN,
                                    &full_w[slot.idx]);
            } else {
                // one 128 x 128 B box = two K blocks (a lone last block over-reads 64 B per row: harmless)
                // and, for folding, the K blocks' rows of integer scales of the
                // tile's columns (columns < N; a 16-byte aligned array only:
                // otherwise the scales are not folded and not read here)
                uint32_t s_bytes = 0u;
                const int16_t* Sx = nullptr;
                if constexpr (C::kScaleRing) {
                    Sx = p.S;
                    if constexpr (GR) Sx = static_cast<const int16_t*>(p.grp_scales[st.e]);
                    const int64_t n0 = int64_t(st.n_tile) * kTileN;
                    const int64_t cols = p.N - n0 < kTileN ? p.N - n0 : kTileN;
                    if ((reinterpret_cast<uintptr_t>(Sx) & 15u) == 0) s_bytes = uint32_t(cols * 2);
                }
                mbar_arrive_expect_tx_one(&full_w[slot.idx], C::kWBytes + uint32_t(st.nkb) * s_bytes);
                tma_load_2d_one(smem + C::offW + slot.idx * C::kWBytes, wmap, st.kb * (kBlockK / 2),
                                st.n_tile * kTileN, &full_w[slot.idx]);
                if constexpr (C::kScaleRing) {
                    if (s_bytes != 0u && lane == 0) {
                        const int32_t kbpg = p.kb_per_group;
                        for (int j = 0; j < st.nkb; ++j) {
                            const int32_t g = kbpg == 1 ? st.kb + j : (st.kb + j) / kbpg;
                            bulk_load(smem + C::offS + slot.idx * C::kSSlotBytes + j * (kTileN * 2),
                                      Sx + int64_t(g) * p.N + int64_t(st.n_tile) * kTileN, s_bytes,
                                      &full_w[slot.idx]);
                        }
                    }
                    __syncwarp();
                }
            }
            w_issued |= 1u << slot.idx;
            w_par = (w_par & ~(1u << slot.idx)) | (slot.phase << slot.idx);
        };
        int32_t prefetched = 0;  // leading stages whose weights were requested before the wait
        {
            StageIter<GR> it(p, pt, b);
            Stage st;
            while (prefetched < (W4A8_PREFETCH(C::kCtasPerSm) < SW ? W4A8_PREFETCH(C::kCtasPerSm) : SW) &&
                   it.next(st)) {
                issue_w(st, rw);  // fresh ring: every slot is free
                rw.advance(SW);
                ++prefetched;
            }
        }
        rw = Ring{};
        wmap_e = -1;
        if constexpr (!GR) griddep_wait();  // the token codes may be the previous kernel's output
        StageIter<GR> it(p, pt, b);
        Stage st;
        bool ok = true;
        // a grouped call with a row index: the tokens of the tile's routed rows
        // 4 lane .. 4 lane + 3, gathered four rows per copy (rows past the
        // expert's last, and indices outside [0, T), read token 0: their
        // outputs are not stored or are zeroed)
        int32_t trow[4] = {0, 0, 0, 0};
        int32_t t_e = -1, t_n = -1, t_m = -1;
        while (ok && it.next(st)) {
            // first token row of the tile (a grouped call: of the expert's routed rows)
            int32_t m0 = st.m_tile * BT;
            if constexpr (GR) {
                const GrSched gs = grsched_of(p);
                m0 += gs.rstart[st.e];
                if (GATHER && (st.e != t_e || st.n_tile != t_n || st.m_tile != t_m)) {
                    t_e = st.e;
                    t_n = st.n_tile;
                    t_m = st.m_tile;
                    const int32_t rend = gs.rstart[st.e + 1];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int32_t r = m0 + 4 * lane + q;
                        const int32_t tk = r < rend ? p.row_index[r] : 0;
                        trow[q] = (tk >= 0 && tk < p.T) ? tk : 0;
                    }
                }
            }
            if (pst >= prefetched) {
                bool free_slot;
                if constexpr (C::kW8) {
                    // the MMAs of stage pst - SW have read this weight slot
                    free_slot = pst < SW || mbar_wait_warp(&sdone[rwd.idx], rwd.phase, abort_flag, p.status, p.wait_limit);
                    if (pst >= SW) rwd.advance(SD);
                } else {
                    free_slot = mbar_wait_warp(&empty_w[rw.idx], rw.phase ^ 1u, abort_flag, p.status, p.wait_limit);
                }
                if (!free_slot) {
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
            mbar_arrive_expect_tx_one(&full_x[rx.idx], uint32_t(st.nkb * BT * kBlockK));
            if constexpr (GATHER) {
                // every lane gathers its four rows of each K block (box one row high)
                __syncwarp();
                uint8_t* xdst = smem + C::offX + rx.idx * C::kXBytes + 4 * lane * kBlockK;
                tma_gather4(xdst, &tm_x, st.kb * kBlockK, trow[0], trow[1], trow[2], trow[3], &full_x[rx.idx]);
                if (st.nkb == 2)
                    tma_gather4(xdst + BT * kBlockK, &tm_x, (st.kb + 1) * kBlockK, trow[0], trow[1], trow[2],
                                trow[3], &full_x[rx.idx]);
            } else {
                tma_load_2d_one(smem + C::offX + rx.idx * C::kXBytes, &tm_x, st.kb * kBlockK, m0, &full_x[rx.idx]);
                if (st.nkb == 2)
                    tma_load_2d_one(smem + C::offX + rx.idx * C::kXBytes + BT * kBlockK, &tm_x,
                                    (st.kb + 1) * kBlockK, m0, &full_x[rx.idx]);
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
        // One converged warp; each MMA and commit is issued by one elected
        // lane.  Per stage: wait for the unpacked operand (TMEM slot) and the
        // token codes, issue up to 8 MMAs (4 per K block) into the accumulator
        // buffer of the current group, commit each group that ends to its
        // buffer's full barrier (the epilogue drains it as soon as its MMAs
        // are done, while the next group's run), and commit the stage to the
        // stage-done ring, which frees the operand slot and the token slot.
        constexpr uint32_t idesc = idesc_i8(kTileN, BT);
        Ring rx, ra, rt, rd;
        Ring rw;  // int8 weights: the weight slot (the MMA's A operand in shared memory)
        StageIter<GR> it(p, pt, b);
        Stage st;
        bool ok = true;
        int32_t kin = 0;  // position of the next K block inside its group (segments start on group boundaries)
        const uint32_t x_lo0 = smem_desc_sw128_lo(smem_u32(smem + C::offX));
        const uint32_t w_lo0 = smem_desc_sw128_lo(smem_u32(smem + C::offW));
        // folded scales: one accumulator buffer per segment (its first MMA
        // overwrites, its last K block commits), no per-group commits
        bool fold = false;
        if constexpr (kFoldable) {
            ok = mbar_wait_warp(fold_ready, 0u, abort_flag, p.status, p.wait_limit);
            fold = fold_decision(misc);
        }
        while (ok && it.next(st)) {
            // the A operand: the unpacked slot in TMEM, or the int8 weight box itself
            const bool a_ready = C::kW8 ? mbar_wait_warp(&full_w[rw.idx], rw.phase, abort_flag, p.status, p.wait_limit)
                                        : mbar_wait_warp(&full_a[ra.idx], ra.phase, abort_flag, p.status, p.wait_limit);
            if (!a_ready || !mbar_wait_warp(&full_x[rx.idx], rx.phase, abort_flag, p.status, p.wait_limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_col = tmem_base + uint32_t(ra.idx * kStageCols);
            const uint32_t w_lo = w_lo0 + uint32_t(rw.idx) * uint32_t(C::kWBytes >> 4);
            const uint32_t x_lo = x_lo0 + uint32_t(rx.idx) * uint32_t(C::kXBytes >> 4);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (j >= st.nkb) break;
                const bool first = fold ? (st.seg_first && j == 0) : (G1 || (kin == 0));
                const bool last = fold ? (st.seg_last && j == st.nkb - 1) : (G1 || (kin == p.kb_per_group - 1));
                if constexpr (!G1) kin = (last || fold) ? 0 : kin + 1;
                if (first) {
                    if (!mbar_wait_warp(&tempty[rt.idx], rt.phase ^ 1u, abort_flag, p.status, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                const uint32_t d = tmem_base + C::kAccCol0 + uint32_t(rt.idx * BT);
                const uint32_t xj = x_lo + uint32_t(j * ((BT * kBlockK) >> 4));
                if constexpr (C::kW8) {
                    const uint32_t wj = w_lo + uint32_t(j * ((kTileN * kBlockK) >> 4));
#pragma unroll
                    for (int k = 0; k < kBlockK / 32; ++k)  // 32 K per MMA: 2 descriptor units of A and of B
                        mma_i8_ss_one(d, smem_desc_from_lo(wj + 2u * k), smem_desc_from_lo(xj + 2u * k), idesc,
                                      (first && k == 0) ? 0u : 1u);
                } else {
                    const uint32_t aj = a_col + uint32_t(j * (kBlockK / 4));
#pragma unroll
                    for (int k = 0; k < kBlockK / 32; ++k)  // 32 K per MMA: 8 TMEM columns of A, 2 descriptor units of B
                        mma_i8_tmem_a_one(d, aj + uint32_t(8 * k), smem_desc_from_lo(xj + 2u * k), idesc,
                                          (first && k == 0) ? 0u : 1u);
                }
                if (last) {
                    if (C::kGroupCommit || fold) mma_commit_one(&afull[rt.idx]);
                    rt.advance(kAcc);
                }
            }
            if (!ok) break;
            if (!C::kGroupCommit && !fold) {
                // the epilogue waits on stage-done phases: it must have seen the
                // previous phase of this slot before it is committed again
                if (!mbar_wait_warp(&sseen[rd.idx], rd.phase ^ 1u, abort_flag, p.status, p.wait_limit)) {
                    ok = false;
                    break;
                }
            }
            mma_commit_one(&sdone[rd.idx]);
            if constexpr (C::kW8)
                rw.advance(SW);
            else
                ra.advance(SA);
            rx.advance(SX);
            rd.advance(SD);
        }
        // every MMA issued has finished before TMEM is released
        mma_commit_one(&mma_done[0]);
        if (lane == 0) drain_wait(&mma_done[0], 0);
        __syncwarp();
    } else if (warp < C::kFirstEpiWarp) {
      if constexpr (!C::kW8) {  // int8 weights need no unpack
        // ---------------------------------------------------------- int4 -> int8 unpack
        // Thread = weight row r of the tile = TMEM lane r.  Per stage it reads
        // its row's 128 packed bytes (eight 16-byte chunks; with the 128-byte
        // swizzle the warp's 32 rows spread each chunk over all banks), turns
        // every chunk into 32 int8 values = 8 TMEM columns, and stores the
        // stage's 64 columns to its lane of the operand slot.
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;
        const int sw = r & 7;
        Ring rw, ra;
        Ring rad;          // stage-done slot of the stage whose operand slot is reused (SA stages back)
        int32_t ust = 0;   // stages unpacked so far
        StageIter<GR> it(p, pt, b);
        Stage st;
        bool ok = true;
        const uint32_t lane_base = tmem_base + (uint32_t(quarter * 32) << 16);
        bool fold = false;
        if constexpr (kFoldable) {
            ok = mbar_wait_warp(fold_ready, 0u, abort_flag, p.status, p.wait_limit);
            fold = fold_decision(misc);
        }
        while (ok && it.next(st)) {
            if (!mbar_wait_warp(&full_w[rw.idx], rw.phase, abort_flag, p.status, p.wait_limit)) {
                ok = false;
                break;
            }
            const uint8_t* wrow = smem + C::offW + rw.idx * C::kWBytes + r * (kStageK / 2);
            uint4 v[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < 4 * st.nkb) v[c] = *reinterpret_cast<const uint4*>(wrow + ((c ^ sw) << 4));
            // folding: this row's integer scales of the stage's K blocks, copied
            // with the box (a column past N: 0, its weights read as zero)
            uint32_t sk0 = 0u, sk1 = 0u;
            if constexpr (C::kScaleRing) {
                if (fold && int64_t(st.n_tile) * kTileN + r < p.N) {
                    const int16_t* srow = reinterpret_cast<const int16_t*>(smem + C::offS + rw.idx * C::kSSlotBytes);
                    sk0 = uint32_t(int32_t(srow[r]));
                    sk1 = uint32_t(int32_t(srow[kTileN + r]));
                }
            }
            // the packed box may be refilled once every warp has read it (the
            // arrive releases this thread's loads above)
            __syncwarp();
            mbar_arrive_one(&empty_w[rw.idx]);
            if (ust >= SA) {  // the MMAs of stage ust - SA have read this operand slot
                if (!mbar_wait_warp(&sdone[rad.idx], rad.phase, abort_flag, p.status, p.wait_limit)) {
                    ok = false;
                    break;
                }
                rad.advance(SD);
                tc_fence_after();
            }
            ++ust;
            const uint32_t slot = lane_base + uint32_t(ra.idx * kStageCols);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (j < st.nkb) {
                    uint32_t o[32];
                    const uint32_t fs = j == 0 ? sk0 : sk1;
                    const uint32_t k1 = (128u - 8u * fs) * 0x01010101u;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 w = v[4 * j + c];
                        uint2 o0, o1, o2, o3;
                        if (fold) {
                            o0 = unpack8_folded(w.x, fs, k1);
                            o1 = unpack8_folded(w.y, fs, k1);
                            o2 = unpack8_folded(w.z, fs, k1);
                            o3 = unpack8_folded(w.w, fs, k1);
                        } else {
                            o0 = unpack8<C::kX16>(w.x);
                            o1 = unpack8<C::kX16>(w.y);
                            o2 = unpack8<C::kX16>(w.z);
                            o3 = unpack8<C::kX16>(w.w);
                        }
                        o[8 * c + 0] = o0.x;
                        o[8 * c + 1] = o0.y;
                        o[8 * c + 2] = o1.x;
                        o[8 * c + 3] = o1.y;
                        o[8 * c + 4] = o2.x;
                        o[8 * c + 5] = o2.y;
                        o[8 * c + 6] = o3.x;
                        o[8 * c + 7] = o3.y;
                    }
                    tmem_st32(slot + uint32_t(j * (kBlockK / 4)), o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            mbar_arrive_one(&full_a[ra.idx]);
            rw.advance(SW);
            ra.advance(SA);
        }
      }
    } else {
        // ---------------------------------------------------------- epilogue
        const int ew = warp - C::kFirstEpiWarp;
        bool fold = false;
        bool fold_seen = true;  // false: the wait for the other warps' checks gave up
        if constexpr (kFoldable) {
            // Does this CTA fold its scales?  Every S[g, n] of its steps (the
            // group rows of its segments, 128 columns each) must lie in
            // [0, kFoldMaxS], or in [0, kFoldMaxS7] with no code -8 in the
            // group (read from the packed codes of those few columns; a
            // grouped call does not pass them and folds only up to 16).
            // Scales are written by the weight packing, never
            // by a kernel that lets its successor start early, so this runs
            // before waiting for the previous kernel, like the first weight
            // copies.  A scale array that is not 16-byte aligned (grouped calls
            // take any even address) is not folded.
            const int nthr = kEpiWarps * 32;
            const int t = ew * 32 + lane;
            SegmentIter<GR> si(p, pt, b);
            Segment s2;
            bool bad = false;
            int32_t base = 0;  // steps of the earlier segments, modulo nthr
            const int64_t N = p.N;
            while (si.next(s2)) {
                const int16_t* Sx = p.S;
                if constexpr (GR) Sx = static_cast<const int16_t*>(p.grp_scales[s2.e]);
                if ((reinterpret_cast<uintptr_t>(Sx) & 15u) != 0) bad = true;
                const int64_t n0 = int64_t(s2.n_tile) * kTileN;
                const int32_t steps = s2.g1 - s2.g0;
                int32_t c = t - base;
                if (c < 0) c += nthr;
                if (!bad) {
                    for (; c < steps; c += nthr) {
                        const int32_t g = s2.g0 + c;
                        const int16_t* row = Sx + int64_t(g) * N + n0;
                        uint4 sv[kTileN / 8];
                        uint32_t mx = 0u;
#pragma unroll
                        for (int q = 0; q < kTileN / 8; ++q) {
                            sv[q] = make_uint4(0u, 0u, 0u, 0u);
                            if (n0 + 8 * q < N) sv[q] = __ldg(reinterpret_cast<const uint4*>(row + 8 * q));
                        }
#pragma unroll
                        for (int q = 0; q < kTileN / 8; ++q)
                            mx = max(mx, scales_max_u16(sv[q]));  // a negative scale reads as >= 2^15
                        if (mx > uint32_t(kFoldMaxS7) || (mx > uint32_t(kFoldMaxS) && (GR || p.wq == nullptr))) {
                            bad = true;
                        } else if (mx > uint32_t(kFoldMaxS)) {
                            // scales of 17 or 18: their groups must hold no code -8
                            const int64_t half_k = int64_t(p.G) * p.kb_per_group * (kBlockK / 2);  // K / 2
                            const int32_t gbytes = p.kb_per_group * (kBlockK / 2);                  // group / 2
                            for (int q = 0; q < kTileN / 8 && !bad; ++q) {
                                const uint32_t w4[4] = {sv[q].x, sv[q].y, sv[q].z, sv[q].w};
                                for (int e = 0; e < 8 && !bad; ++e) {
                                    const uint32_t sval = (w4[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                                    if (sval <= uint32_t(kFoldMaxS)) continue;
                                    const uint8_t* cp = p.wq + (n0 + 8 * q + e) * half_k + int64_t(g) * gbytes;
                                    for (int o = 0; o < gbytes; o += 16) {
                                        const uint4 cw = __ldg(reinterpret_cast<const uint4*>(cp + o));
                                        if (has_code_minus8(cw.x) || has_code_minus8(cw.y) || has_code_minus8(cw.z) ||
                                            has_code_minus8(cw.w)) {
                                            bad = true;
                                            break;
                                        }
                                    }
                                }
                            }
                        }
                    }
                }
                base = (base + steps) % nthr;
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&misc[4], 1u);
            __syncwarp();
            mbar_arrive_one(fold_ready);  // lane 0 (the elected lane) made the update above
            fold_seen = mbar_wait_warp(fold_ready, 0u, abort_flag, p.status, p.wait_limit);
            fold = fold_decision(misc);
        }
        griddep_wait();  // s_a, y and the workspace may be in use by the previous kernel
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int half = ew >> 2;      // which part of the BT columns
        const int r = quarter * 32 + lane;
        Ring rt, rd;
        SegmentIter<GR> it(p, pt, b);
        Segment sg;
        bool ok = fold_seen;
        const int32_t kbpg = p.kb_per_group;
        const int32_t G = int32_t(p.G);
        while (ok && it.next(sg)) {
            const int64_t n0 = int64_t(sg.n_tile) * kTileN;
            // the tile's first token row and the end of its rows (a grouped
            // call: the expert's routed rows) and the group scales to use
            int64_t mbase = int64_t(sg.m_tile) * BT;
            int64_t mend = p.M;
            const int16_t* S_g = p.S;
            if constexpr (GR) {
                const GrSched gs = grsched_of(p);
                mbase += gs.rstart[sg.e];
                mend = gs.rstart[sg.e + 1];
                S_g = static_cast<const int16_t*>(p.grp_scales[sg.e]);
            }
            const int64_t m0 = mbase + half * HC;
            const int64_t n = n0 + r;
            const bool nvalid = n < p.N;
            // output scale of token (tile start + this thread's index among the
            // epilogue threads), handed to the tail through shared memory
            float sa_pref = 0.0f;
            int32_t z_pref = 0;   // zero point of the same token (ZP)
            int32_t zc_n = 0;     // zero-point term of this thread's column (ZP)
            {
                const int te = ew * 32 + lane;
                const int64_t mt = mbase + te;
                if constexpr (GATHER) {
                    // rows gathered by index: the scale of the row's token; a
                    // token outside [0, T) marks the row (NaN scale): its
                    // outputs are zeroed
                    if (te < BT && mt < mend) {
                        const int64_t tok = p.row_index[mt];
                        if (tok >= 0 && tok < p.T) {
                            sa_pref = output_scale<PATH>(p, tok);
                        } else {
                            sa_pref = __int_as_float(0x7fc00000);
                            atomicExch(p.status, kStatusInvalidArg);
                        }
                    }
                } else {
                    if (te < BT && mt < mend) sa_pref = output_scale<PATH>(p, mt);
                }
                if constexpr (ZP) {
                    if (te < BT && mt < mend) z_pref = p.z_a[mt];
                    if (nvalid) zc_n = p.zc[n];
                }
            }
            int32_t acc[HC];
            float accf[HC];
#pragma unroll
            for (int j = 0; j < HC; ++j) {
                acc[j] = 0;
                accf[j] = 0.0f;
            }
            // A split tile's first contributor (its segment opens the tile) finishes
            // its share last; the other contributors did theirs at the start of
            // their ranges.  With narrow tiles and one other contributor, that
            // partial is usually complete already: read it now, while this
            // segment's groups are drained, instead of at the end.
            int32_t pacc[C::kEarlyCombine ? HC : 1];
            bool early = false;
            if constexpr (C::kEarlyCombine) {
                if (sg.g0 == 0 && sg.g1 < int32_t(p.G)) {
                    const uint32_t t0 = sg.tile * uint32_t(p.G);
                    const uint32_t b_last = range_owner(t0 + uint32_t(p.G) - 1u, pt);
                    if (ew == 0 && lane == 0)
                        misc[3] = (b_last == b + 1 && ld_acquire_gpu(&p.ws_count[b]) >= 1) ? 1u : 0u;
                    epi_bar_sync(kEpiWarps * 32);
                    early = misc[3] != 0u;  // the same for every epilogue thread
                    if (early) {
                        const int nv = mend - m0 >= HC ? HC : (mend - m0 > 0 ? int(mend - m0) : 0);
                        const int32_t* cp = p.ws_part + int64_t(b + 1) * (int64_t(kTileN) * BT) +
                                            int64_t(half * HC) * kTileN + r;
#pragma unroll
                        for (int j = 0; j < HC; ++j) pacc[j] = j < nv ? __ldcg(cp + j * kTileN) : 0;
                    }
                }
            }
            if (fold) {
                // Folded scales: the segment's MMAs summed S * q * x into one
                // buffer, committed after its last K block: that is the
                // segment's accumulator, read once.
                if (!mbar_wait_warp(&afull[rt.idx], rt.phase, abort_flag, p.status, p.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t lane_cols =
                    tmem_base + (uint32_t(quarter * 32) << 16) + C::kAccCol0 + uint32_t(rt.idx * BT + half * HC);
                constexpr int CH = HC < 32 ? HC : 32;
#pragma unroll
                for (int c0 = 0; c0 < HC; c0 += CH) {
                    uint32_t v[CH];
                    tmem_load<CH>(lane_cols + uint32_t(c0), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < CH; ++q) acc[c0 + q] = int32_t(v[q]);
                }
                tc_fence_before();
                __syncwarp();
                mbar_arrive_one(&tempty[rt.idx]);
                rt.advance(kAcc);
            } else if constexpr (kLean) {
                // One group per K block, each committed to its own accumulator
                // buffer: wait for the group's MMAs, load this thread's HC
                // columns of P_g, hand the buffer back, and add
                // acc += S[g,n] * P_g (or accf += s_g * float(P_g)).  This
                // column's scale is read from global memory two groups ahead
                // (a column past N reads column 0's scales: its outputs are
                // never stored).
                const uint32_t lane_cols =
                    tmem_base + (uint32_t(quarter * 32) << 16) + C::kAccCol0 + uint32_t(half * HC);
                const int32_t n_ld = nvalid ? int32_t(n) : 0;
                const int32_t nstride = int32_t(p.N);
                int32_t sidx = sg.g0 * nstride + n_ld;  // element index of the next scale to load (< 2^31)
                auto ld_scale = [&](int32_t i) -> uint32_t {
                    if constexpr (PATH == kIntScale)
                        return uint32_t(int32_t(__ldg(S_g + i)));
                    else
                        return __float_as_uint(__ldg(p.s_g + i));
                };
                uint32_t s1 = ld_scale(sidx);
                sidx += nstride;
                uint32_t s2 = (sg.g0 + 1 < sg.g1) ? ld_scale(sidx) : 0u;
                sidx += nstride;
                for (int32_t g = sg.g0; g < sg.g1; ++g) {
                    const uint32_t sraw = s1;
                    s1 = s2;
                    if (g + 2 < sg.g1) s2 = ld_scale(sidx);
                    sidx += nstride;
                    if (!mbar_wait_warp(&afull[rt.idx], rt.phase, abort_flag, p.status, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // in parts (load, multiply-add, load, multiply-add, ...):
                    // the two epilogue warps of an SM sub-partition then drift
                    // apart, one loading while the other multiplies (measured
                    // at M = 1024 against one load of all HC columns: two parts
                    // 3% faster on the integer path, four parts 2% on the
                    // float path)
                    constexpr int kParts = PATH == kIntScale ? 2 : 4;
                    constexpr int H = HC / kParts;
#pragma unroll
                    for (int hh = 0; hh < kParts; ++hh) {
                        uint32_t v[H];
                        tmem_load<H>(lane_cols + uint32_t(rt.idx * BT + hh * H), v);
                        tmem_wait_ld();
                        if (hh == kParts - 1) {
                            tc_fence_before();
                            __syncwarp();
                            mbar_arrive_one(&tempty[rt.idx]);
                            rt.advance(kAcc);
                        }
                        if constexpr (PATH == kIntScale) {
                            const int32_t s_cur = int32_t(sraw);
#pragma unroll
                            for (int q = 0; q < H; ++q) {
                                const int32_t pg = C::kX16 ? (int32_t(v[q]) >> 4) : int32_t(v[q]);  // exact
                                acc[hh * H + q] += s_cur * pg;
                            }
                        } else {
                            const float f_cur = C::kX16 ? __fmul_rn(__uint_as_float(sraw), 0.0625f)
                                                        : __uint_as_float(sraw);
#pragma unroll
                            for (int q = 0; q < H; ++q)
                                accf[hh * H + q] = __fmaf_rn(f_cur, __int2float_rn(int32_t(v[q])), accf[hh * H + q]);
                        }
                    }
                }
            } else {
            // This column's scales (raw 32 bits) of group g, read straight from
            // global memory two stages before they are used, so that no wait
            // or shared-memory round trip sits between two drains.  Rows past
            // the last group and columns past N read as zero.
            auto load_scale = [&](int32_t g) -> uint32_t {
                if (g >= G || !nvalid) return 0u;
                const int64_t idx = int64_t(g) * int32_t(p.N) + n;  // N < 2^31 (checked on the host)
                if constexpr (PATH == kIntScale)
                    return uint32_t(int32_t(__ldg(S_g + idx)));
                else
                    return __float_as_uint(__ldg(p.s_g + idx));
            };
            // the groups ending in a stage are the stage's first group and the next one
            auto stage_group = [&](int32_t kb_first) -> int32_t {
                return kbpg == 1 ? kb_first : int32_t(uint32_t(kb_first) / uint32_t(kbpg));
            };
            // Walk the segment's stages in the order the MMA warp issues them and
            // drain every group whose last K block was in that stage, each as
            // soon as its MMAs are complete, handing its accumulator buffer back
            // to the MMA warp.
            int32_t kin = 0;    // position of the next K block inside its group
            int32_t kb = sg.g0 * kbpg;
            const int32_t kb_end = sg.g1 * kbpg;
            uint32_t sc0 = 0u, sc1 = 0u, nx0 = 0u, nx1 = 0u;  // scales of this stage and of the next
            {
                const int32_t g0 = stage_group(kb);
                sc0 = load_scale(g0);
                sc1 = load_scale(g0 + 1);
                if (kb + 2 < kb_end) {
                    const int32_t g1 = stage_group(kb + 2);
                    nx0 = load_scale(g1);
                    nx1 = load_scale(g1 + 1);
                }
            }
            while (kb < kb_end) {
                const int32_t nkb = (kb_end - kb) >= 2 ? 2 : 1;
                const uint32_t s0 = sc0, s1 = sc1;
                sc0 = nx0;
                sc1 = nx1;
                if (kb + 4 < kb_end) {  // the stage after next
                    const int32_t g2 = stage_group(kb + 4);
                    nx0 = load_scale(g2);
                    nx1 = load_scale(g2 + 1);
                }
                kb += nkb;
                if constexpr (!C::kGroupCommit) {
                    // Per-stage commits: wait for the stage, then tell the MMA
                    // warp its phase was seen (it waits for that before it
                    // commits the slot again).
                    if (!mbar_wait_warp(&sdone[rd.idx], rd.phase, abort_flag, p.status, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    __syncwarp();
                    mbar_arrive_one(&sseen[rd.idx]);
                    rd.advance(SD);
                }
                // groups whose last K block is in this stage (at most two)
                int ng = 0;
                uint32_t gb0 = 0u, gb1 = 0u;  // their TMEM buffers
                uint32_t ph0 = 0u, ph1 = 0u;  // and the phases of the buffers' full barriers
                if (kbpg == 1) {  // 128-wide groups: every K block ends one
                    ng = nkb;
                    gb0 = uint32_t(rt.idx);
                    ph0 = rt.phase;
                    rt.advance(kAcc);
                    if (nkb == 2) {
                        gb1 = uint32_t(rt.idx);
                        ph1 = rt.phase;
                        rt.advance(kAcc);
                    }
                } else {
                    for (int j = 0; j < nkb; ++j) {
                        const bool last = (kin == kbpg - 1);
                        kin = last ? 0 : kin + 1;
                        if (last) {
                            if (ng == 0) {
                                gb0 = uint32_t(rt.idx);
                                ph0 = rt.phase;
                            } else {
                                gb1 = uint32_t(rt.idx);
                                ph1 = rt.phase;
                            }
                            ++ng;
                            rt.advance(kAcc);
                        }
                    }
                }
                if (ng == 0) continue;
                const uint32_t lane_cols =
                    tmem_base + (uint32_t(quarter * 32) << 16) + C::kAccCol0 + uint32_t(half * HC);
                auto accumulate = [&](const uint32_t* v, int c0, int cnt, uint32_t sraw) {
                    if constexpr (PATH == kIntScale) {
                        const int32_t s_cur = int32_t(sraw);
#pragma unroll
                        for (int q = 0; q < cnt; ++q) {
                            const int32_t pg = C::kX16 ? (int32_t(v[q]) >> 4) : int32_t(v[q]);  // exact
                            acc[c0 + q] += s_cur * pg;
                        }
                    } else {
                        const float f_cur = C::kX16 ? __fmul_rn(__uint_as_float(sraw), 0.0625f)  // P_g was 16 P_g
                                                    : __uint_as_float(sraw);
#pragma unroll
                        for (int q = 0; q < cnt; ++q)
                            accf[c0 + q] = __fmaf_rn(f_cur, __int2float_rn(int32_t(v[q])), accf[c0 + q]);
                    }
                };
                if constexpr (HC <= 16) {
                    // small tiles: both groups' loads in flight before one wait
                    if constexpr (C::kGroupCommit) {
                        if (!mbar_wait_warp(&afull[gb0], ph0, abort_flag, p.status, p.wait_limit) ||
                            (ng == 2 && !mbar_wait_warp(&afull[gb1], ph1, abort_flag, p.status, p.wait_limit))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    uint32_t v0[HC], v1[HC];
                    tmem_load<HC>(lane_cols + gb0 * uint32_t(BT), v0);
                    if (ng == 2) tmem_load<HC>(lane_cols + gb1 * uint32_t(BT), v1);
                    tmem_wait_ld();
                    accumulate(v0, 0, HC, s0);
                    if (ng == 2) accumulate(v1, 0, HC, s1);
                    tc_fence_before();
                    __syncwarp();
                    mbar_arrive_one(&tempty[gb0]);
                    if (ng == 2) mbar_arrive_one(&tempty[gb1]);
                } else {
                    // wide tiles: each group's buffer goes back to the MMA warp
                    // as soon as it is drained
                    constexpr int CH = W4A8_DRAIN_CH < HC ? W4A8_DRAIN_CH : HC;
                    for (int gi = 0; gi < ng; ++gi) {
                        const uint32_t gb = gi == 0 ? gb0 : gb1;
                        if constexpr (C::kGroupCommit) {
                            if (!mbar_wait_warp(&afull[gb], gi == 0 ? ph0 : ph1, abort_flag, p.status, p.wait_limit)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const uint32_t sraw = gi == 0 ? s0 : s1;
#pragma unroll
                        for (int c0 = 0; c0 < HC; c0 += CH) {
                            uint32_t v[CH];
                            tmem_load<CH>(lane_cols + gb * uint32_t(BT) + uint32_t(c0), v);
                            tmem_wait_ld();
                            accumulate(v, c0, CH, sraw);
                        }
                        tc_fence_before();
                        __syncwarp();
                        mbar_arrive_one(&tempty[gb]);
                    }
                    if (!ok) break;
                }
            }
            }  // kLean
            if (!ok) break;

            // valid token columns of this thread's share (split-tile partials)
            const int nv = mend - m0 >= HC ? HC : (mend - m0 > 0 ? int(mend - m0) : 0);
            const bool whole = (sg.g0 == 0 && sg.g1 == p.G);
            if (!whole) {
                // ---- split tile.  The tile's first contributor b_first covers the
                // tile's first groups at the end of its own range, so it finishes its
                // share last: it combines.  Every other contributor stores its partial
                // (valid columns only, in the slot of its CTA: a CTA contributes a
                // partial to at most one tile, the one whose last groups open its range)
                // and signals an arrival counter indexed by b_first (the first
                // contributor of no other tile).  b_first waits (bounded) for all
                // arrivals, adds the partials to its own, which never leave registers,
                // writes y and re-zeroes the counter.
                const uint32_t t0 = sg.tile * uint32_t(p.G);
                const uint32_t b_first = range_owner(t0, pt);
                const uint32_t b_last = range_owner(t0 + uint32_t(p.G) - 1u, pt);
                const int64_t slot_elems = int64_t(kTileN) * BT;
                if (b != b_first) {
                    int32_t* part = p.ws_part + int64_t(b) * slot_elems + int64_t(half * HC) * kTileN + r;
#pragma unroll
                    for (int j = 0; j < HC; ++j)
                        if (j < nv) part[j * kTileN] = PATH == kIntScale ? acc[j] : __float_as_int(accf[j]);
                    epi_bar_sync(kEpiWarps * 32);  // the CTA's partial stores, before the arrival
                    if (ew == 0 && lane == 0) red_release_gpu_add(&p.ws_count[b_first], 1);
                    continue;
                }
                if (early) {
                    // one other contributor, read at the start of the segment (the
                    // same sum, in the same order, as below)
#pragma unroll
                    for (int j = 0; j < HC; ++j) {
                        if constexpr (C::kEarlyCombine) {
                            if (PATH == kIntScale)
                                acc[j] += pacc[j];
                            else
                                accf[j] = __fadd_rn(accf[j], __int_as_float(pacc[j]));
                        }
                    }
                } else if (ew == 0 && lane == 0) {
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
                if (!early) {
                    epi_bar_sync(kEpiWarps * 32);
                    if (!misc[2]) {
                        ok = false;
                        break;
                    }
                }
                for (uint32_t c = early ? b_last + 1 : b_first + 1; c <= b_last; ++c) {
                    const int32_t* cp = p.ws_part + int64_t(c) * slot_elems + int64_t(half * HC) * kTileN + r;
#pragma unroll
                    for (int j = 0; j < HC; ++j) {
                        if (j < nv) {
                            const int32_t v = __ldcg(cp + j * kTileN);
                            if (PATH == kIntScale)
                                acc[j] += v;
                            else
                                accf[j] = __fadd_rn(accf[j], __int_as_float(v));
                        }
                    }
                }
                epi_bar_sync(kEpiWarps * 32);  // every thread has read the partials before the counter is reused
                if (ew == 0 && lane == 0) p.ws_count[b_first] = 0;
            }
            // ---- the tile's outputs: converted in registers, staged in shared
            // memory as [BT tokens][128 columns], stored by one TMA tensor store
            // (which leaves out rows past M and columns past N).
            const bool leader = (ew == 0 && lane == 0);
            // the previous tile's stores have read the staging buffer (a
            // grouped call's stores come from every lane of the first warp)
            if (GR ? ew == 0 : leader) bulk_wait_read_all();
            epi_bar_sync(kEpiWarps * 32);
            float* sa_tile = reinterpret_cast<float*>(smem + C::offSA);
            if (ew * 32 + lane < BT) sa_tile[ew * 32 + lane] = sa_pref;
            if constexpr (ZP) {
                int32_t* z_tile = reinterpret_cast<int32_t*>(smem + C::offZ);
                if (ew * 32 + lane < BT) z_tile[ew * 32 + lane] = z_pref;
            }
            epi_bar_sync(kEpiWarps * 32);
            if constexpr (ZP) {
                // acc - z[m] * c[n], in two's-complement arithmetic: the terms may
                // wrap, the difference (the true accumulator) fits in 32 bits
                const int32_t* zt = reinterpret_cast<const int32_t*>(smem + C::offZ) + half * HC;
#pragma unroll
                for (int j = 0; j < HC; ++j)
                    acc[j] = int32_t(uint32_t(acc[j]) - uint32_t(zt[j]) * uint32_t(zc_n));
            }
            {
                const int base = half * HC * kTileN + r;  // element index of (token half*HC, column r)
                const float* sa = sa_tile + half * HC;
                if constexpr (GATHER) {
                    // rows marked invalid (NaN scale) are written as zeros
#pragma unroll
                    for (int j = 0; j < HC; ++j) {
                        if (sa[j] != sa[j]) {
                            acc[j] = 0;
                            accf[j] = 0.0f;
                        }
                    }
                }
                if (p.y_dtype == kOutI32) {
                    int32_t* yo = reinterpret_cast<int32_t*>(smem + C::offY) + base;
#pragma unroll
                    for (int j = 0; j < HC; ++j) yo[j * kTileN] = acc[j];
                } else if (p.y_dtype == kOutF16) {
                    __half* yo = reinterpret_cast<__half*>(smem + C::offY) + base;
#pragma unroll
                    for (int j = 0; j < HC; ++j)
                        yo[j * kTileN] = __float2half_rn(
                            __fmul_rn(PATH == kIntScale ? __int2float_rn(acc[j]) : accf[j], GATHER && sa[j] != sa[j] ? 0.0f : sa[j]));
                } else {
                    float* yo = reinterpret_cast<float*>(smem + C::offY) + base;
#pragma unroll
                    for (int j = 0; j < HC; ++j)
                        yo[j * kTileN] = __fmul_rn(PATH == kIntScale ? __int2float_rn(acc[j]) : accf[j],
                                                   GATHER && sa[j] != sa[j] ? 0.0f : sa[j]);
                }
            }
            fence_proxy_async_smem();  // the staged outputs, visible to the TMA unit
            epi_bar_sync(kEpiWarps * 32);
            if constexpr (GR) {
                // one bulk copy per routed row of the tile, to row i or out_row[i]
                // (rows past the expert's last belong to the next expert: not stored)
                if (ew == 0) {
                    const int esz = p.y_dtype == kOutF16 ? 2 : 4;
                    const int64_t cols = p.N - n0 < kTileN ? p.N - n0 : kTileN;
                    const int rows = mend - mbase < BT ? int(mend - mbase) : BT;
                    for (int t = lane; t < rows; t += 32) {
                        int64_t orow = mbase + t;
                        if (p.out_row != nullptr) {
                            orow = p.out_row[orow];
                            if (orow < 0 || orow >= p.y_rows) {
                                atomicExch(p.status, kStatusInvalidArg);
                                continue;
                            }
                        }
                        bulk_store(static_cast<uint8_t*>(p.y) + (orow * p.N + n0) * esz,
                                   smem + C::offY + int64_t(t) * kTileN * esz, uint32_t(cols * esz));
                    }
                    bulk_commit_group();
                }
            } else if (leader) {
                tma_store_2d(&tm_y, smem + C::offY, int32_t(n0), sg.m_tile * BT);
                bulk_commit_group();
            }
        }
        // shared memory stays until the stores have read it
        if (GR ? ew == 0 : (ew == 0 && lane == 0)) bulk_wait_read_all();
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

Plan make_plan(int64_t M, int64_t N, int64_t K, int32_t group, int num_sms, bool w8) {
    Plan pl{};
    pl.BT = token_tile_for(M);
    pl.n_tiles = (N + kTileN - 1) / kTileN;
    pl.m_tiles = (M + pl.BT - 1) / pl.BT;
    pl.G = K / group;
    pl.tiles = pl.n_tiles * pl.m_tiles;
    pl.W = pl.tiles * pl.G;
    const int64_t slots = int64_t(num_sms) * (w8 ? 1 : W4A8_CTAS_PER_SM(pl.BT));  // resident CTAs
    pl.grid = pl.W < slots ? pl.W : slots;
    if (pl.grid > kMaxGrid) pl.grid = kMaxGrid;
    const int64_t slot_bytes = int64_t(kTileN) * pl.BT * 4;
    pl.count_bytes = kCounterBytes;
    pl.ws_bytes = pl.count_bytes + pl.grid * slot_bytes;  // a CTA stores the partial of at most one tile
    return pl;
}

template <auto kern, typename P>
static cudaError_t launch_k(int threads, int smem, const CUtensorMap& tw, const CUtensorMap& tx,
                            const CUtensorMap& ty, const P& p, cudaStream_t stream) {
    const cudaError_t e = configure_once<kern>(threads, smem);
    if (e != cudaSuccess) return e;
    const LaunchPdl lc(unsigned(p.grid), threads, size_t(smem), stream);
    return cudaLaunchKernelEx(&lc.cfg, kern, tw, tx, ty, p);
}

template <int BT, int PATH, bool W8 = false, bool ZP = false>
static cudaError_t launch_bt(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty,
                             const std::conditional_t<ZP, ParamsZp, Params>& p, cudaStream_t stream) {
    using C = Cfg<BT, PATH, W8, ZP>;
    if (p.kb_per_group == 1)
        return launch_k<w4a8_gemm_kernel<BT, PATH, W8, ZP, true>>(C::kThreads, C::kSmemBytes, tw, tx, ty, p, stream);
    return launch_k<w4a8_gemm_kernel<BT, PATH, W8, ZP, false>>(C::kThreads, C::kSmemBytes, tw, tx, ty, p, stream);
}

cudaError_t launch(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty, const Params& p, int BT, int path,
                   cudaStream_t stream, bool w8) {
    if (w8) {  // int8 weights: the integer-scale path
        switch (BT) {
            case 16: return launch_bt<16, kIntScale, true>(tw, tx, ty, p, stream);
            case 32: return launch_bt<32, kIntScale, true>(tw, tx, ty, p, stream);
            case 64: return launch_bt<64, kIntScale, true>(tw, tx, ty, p, stream);
            default: return launch_bt<128, kIntScale, true>(tw, tx, ty, p, stream);
        }
    }
    if (path == kIntScale) {
        switch (BT) {
            case 16: return launch_bt<16, kIntScale>(tw, tx, ty, p, stream);
            case 32: return launch_bt<32, kIntScale>(tw, tx, ty, p, stream);
            case 64: return launch_bt<64, kIntScale>(tw, tx, ty, p, stream);
            default: return launch_bt<128, kIntScale>(tw, tx, ty, p, stream);
        }
    }
    switch (BT) {
        case 16: return launch_bt<16, kFloatScale>(tw, tx, ty, p, stream);
        case 32: return launch_bt<32, kFloatScale>(tw, tx, ty, p, stream);
        case 64: return launch_bt<64, kFloatScale>(tw, tx, ty, p, stream);
        default: return launch_bt<128, kFloatScale>(tw, tx, ty, p, stream);
    }
}

cudaError_t launch_zp(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty, const ParamsZp& p, int BT,
                      cudaStream_t stream) {
    switch (BT) {
        case 16: return launch_bt<16, kIntScale, false, true>(tw, tx, ty, p, stream);
        case 32: return launch_bt<32, kIntScale, false, true>(tw, tx, ty, p, stream);
        case 64: return launch_bt<64, kIntScale, false, true>(tw, tx, ty, p, stream);
        default: return launch_bt<128, kIntScale, false, true>(tw, tx, ty, p, stream);
    }
}

cudaError_t launch_grouped(const CUtensorMap& tm_w_template, const CUtensorMap& tm_x, const int64_t* offsets,
                           const void* const* w_ptrs, int64_t R, const ParamsGr& p, int32_t* sched,
                           CUtensorMap* maps, cudaStream_t stream) {
    cudaError_t e = launch_grouped_setup(tm_w_template, offsets, w_ptrs, p.grp_scales, p.E, R, 128, p.n_tiles,
                                         int32_t(p.G), int32_t(p.grid), sched, maps, p.status, stream);
    if (e != cudaSuccess) return e;
    using C = Cfg<128, kIntScale, false, false>;
    // tm_y is not read by a grouped call (its rows are stored one by one)
    const bool g1 = p.kb_per_group == 1;
    if (p.row_index != nullptr) {
        if (g1)
            return launch_k<w4a8_gemm_kernel<128, kIntScale, false, false, true, true, true>>(
                C::kThreads, C::kSmemBytes, tm_w_template, tm_x, tm_x, p, stream);
        return launch_k<w4a8_gemm_kernel<128, kIntScale, false, false, false, true, true>>(
            C::kThreads, C::kSmemBytes, tm_w_template, tm_x, tm_x, p, stream);
    }
    if (g1)
        return launch_k<w4a8_gemm_kernel<128, kIntScale, false, false, true, true>>(C::kThreads, C::kSmemBytes,
                                                                                    tm_w_template, tm_x, tm_x, p,
                                                                                    stream);
    return launch_k<w4a8_gemm_kernel<128, kIntScale, false, false, false, true>>(C::kThreads, C::kSmemBytes,
                                                                                 tm_w_template, tm_x, tm_x, p, stream);
}

int token_tile_rows() { return kTileN; }

int weight_box_bytes() { return kStageK / 2; }

}  // namespace gemm
}  // namespace w4a8
