// tc_tiles.cuh — pieces shared by the tensor-core GEMMs: INT4 -> E4M3 widening, the
// 128-byte-swizzle address of a K-major tile, the expert-segment tile map and the token-tile
// width choice.
//
// Widening.  The MMA's A operand is the group's weight tile in E4M3 (every INT4 code -8..7 is
// an E4M3 value, so the widening is exact):
//  * signed: byte = E4M3(code) through two byte-permute table lookups (12 integer ops per
//    8 codes); one FMA per element promotes the group.  Used for wide token tiles (prefill).
//  * unsigned: byte = the stored nibble itself (code + 8).  Bytes 0x00..0x0F are the E4M3
//    values 0..15 x 2^-9 (the subnormals and the first normal binade form one equally spaced
//    ladder), so the MMA sees 2^-9 * (code + 8); the GEMM removes the +8 offset (see
//    gemm_ws.cuh).  The even nibbles become bytes 0..3 and the odd ones bytes 4..7 (3 integer
//    ops per 8 codes), i.e. K order 0,2,4,6,1,3,5,7 within each word; the activations of these
//    tiles are stored in the same order (perm8 in common.cuh), and a K-permutation applied to
//    both operands leaves every dot product unchanged.  Used for narrow token tiles (decode).
#pragma once
#include "common.cuh"

namespace moe {

// ---- widening ------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Eight codes of one packed word -> eight E4M3 bytes: signed in K order (lo = codes 0..3);
// unsigned in K order 0,2,4,6 (lo) and 1,3,5,7 (hi).
template <bool kUnsigned>
__device__ __forceinline__ uint2 widen8(uint32_t w) {
    if constexpr (kUnsigned) {
        return make_uint2(w & 0x0F0F0F0Fu,            // nibbles 0, 2, 4, 6
                          (w >> 4) & 0x0F0F0F0Fu);    // nibbles 1, 3, 5, 7
    } else {
        // E4M3 of code = nibble - 8: nibbles 0..7 (negative codes) and 8..15 (0..7)
        constexpr uint32_t kNeg0 = 0xCACCCED0u, kNeg1 = 0xB8C0C4C8u;
        constexpr uint32_t kPos0 = 0x44403800u, kPos1 = 0x4E4C4A48u;
        const uint32_t ws = w << 4;
        const uint32_t sl = w & 0x7777u, sh = (w >> 16) & 0x7777u;
        // byte masks: 0xFF where the nibble's bit 3 is set (sign-replicate mode of prmt)
        const uint32_t ml = prmt(ws, w, 0xD9C8u), mh = prmt(ws, w, 0xFBEAu);
        const uint32_t lo = (prmt(kPos0, kPos1, sl) & ml) | (prmt(kNeg0, kNeg1, sl) & ~ml);
        const uint32_t hi = (prmt(kPos0, kPos1, sh) & mh) | (prmt(kNeg0, kNeg1, sh) & ~mh);
        return make_uint2(lo, hi);
    }
}

// Byte offset of 16-byte chunk j (0..7) of row r in a K-major 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int j) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

// ---- tile map ------------------------------------------------------------------------------

// Slab map of a hybrid layer (hot NVFP4 / cold W4A8 experts): slot_of[e] = i for hot slab i,
// -(j + 1) for cold slab j, kSlotNone for an expert in neither list.
constexpr int32_t kSlotNone = INT32_MIN;
// kSlotShort / kSlotLong select experts by segment length instead (at most kShortRows rows, or
// more): a W4A8 layer of mostly long segments runs its short ones on narrow tiles.
enum SlotWant { kSlotAll = 0, kSlotCold = 1, kSlotHot = 2, kSlotShort = 3, kSlotLong = 4 };
constexpr int kShortRows = 32;

__device__ __forceinline__ bool slot_kept(const int32_t* slot_of, int want, int e) {
    if (!slot_of || want == kSlotAll) return true;
    const int32_t s = slot_of[e];
    return want == kSlotHot ? s >= 0 : (s < 0 && s != kSlotNone);
}

// Weight slab of expert e (e itself for a single-format layer).
__device__ __forceinline__ int weight_slab(const int32_t* slot_of, int e) {
    if (!slot_of) return e;
    const int32_t s = slot_of[e];
    return s >= 0 ? s : -s - 1;
}

// Per-expert prefix of row tiles (ceil(len / BN)) into shared `pre[0..E]` and the segment offsets
// [0..E] into shared `soff`; returns the total.  Every thread loads its share of the offsets at
// once (one global round trip), then one warp scans the tile counts in shared memory.  With
// `slot_of`, experts of the other format get no tiles (`want`: kSlotCold or kSlotHot); with
// kSlotShort / kSlotLong, experts of the other segment-length class get none.
__device__ int row_tile_prefix(const int32_t* __restrict__ offsets, int E, int BN, int* pre, int* soff,
                               const int32_t* slot_of = nullptr, int want = kSlotAll) {
    __shared__ int s_total;
    for (int e = threadIdx.x; e <= E; e += blockDim.x) soff[e] = offsets[e];
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int len = soff[e + 1] - soff[e];
        const bool kept = want >= kSlotShort ? ((len <= kShortRows) == (want == kSlotShort))
                                             : slot_kept(slot_of, want, e);
        pre[e] = kept ? (len + BN - 1) / BN : 0;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int run = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int n = e < E ? pre[e] : 0;
            int inc = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (e < E) pre[e] = run + inc - n;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) {
            pre[E] = run;
            s_total = run;
        }
    }
    __syncthreads();
    return s_total;
}

// Expert owning row tile `rt` (pre[e] <= rt < pre[e+1]).
__device__ __forceinline__ int expert_of_tile(const int* pre, int E, int rt) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= rt) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Launch shape of one kernel instance on one device (set once; later calls only read it).
struct TcLaunchShape {
    int sms = 0, ctas_per_sm = 0;
};

// Token-tile width for the expected rows per expert: 16 / 32 rows at decode (narrow tiles: the
// unsigned widening and the gathered activation rows), else 128 rows.  Wide tiles are as wide
// as TMEM allows whatever the average, because routed segments are skewed: with Zipf routing at
// T = 2048 (48 rows per expert on average) the popular experts' long segments dominate the
// work, and 128-row tiles re-read each of their weight tiles half as often as 64-row ones
// (measured: W4A8 gate/up 1.14 -> 0.94 ms).
constexpr int64_t kWsWideAvg = 160;
inline int tc_tile_rows(int64_t P, int E) {
    const int64_t avg = (P + E - 1) / E;
    return avg <= 8 ? 16 : avg <= 24 ? 32 : 128;
}

// The W4A8 GEMM widens each weight stage once per token tile, so long segments want the widest
// tile whose partial buffers still leave TMEM room for the widened A stages: 192 rows (two
// 192-column partials + four 32-column A stages = 512 columns).
inline int ws_tile_rows(int64_t P, int E) {
    const int bn = tc_tile_rows(P, E);
    return bn == 128 && (P + E - 1) / E >= kWsWideAvg ? 192 : bn;
}

}  // namespace moe
