// gemm_ws.cuh — S4/S6: warp-specialised grouped W4A8 GEMM on tcgen05 with TMA rings.
//
// Roles (persistent CTAs; two per SM on 16-row token tiles, else one):
//   widening warps (8 on narrow token tiles, 4 on wide ones): a thread owns one weight row = one
//              TMEM lane.  Per stage (two K-groups on narrow tiles, one on wide ones) it reads the
//              row's packed INT4 codes from the TMA stage (the 64- or 128-byte TMA swizzle spreads
//              the 32 rows of a warp over distinct banks), widens them to E4M3 and writes them
//              into a TMEM A stage with tcgen05.st; the MMA takes A from TMEM.
//   promotion warps (4 on narrow tiles, 16 on 128- and 192-row tiles, each owning a lane
//              quadrant and a slice of the token columns): per K-group they fold the group's TMEM
//              partial into fp32 register accumulators with the group scale (acc += s[n,g] *
//              partial, two columns per packed FMA), then run the tile's epilogue: SwiGLU, h rows
//              and max|h| per row (gate/up), or Y rows (down).  Requantization and combine are
//              separate passes after the GEMMs.
//   TMA warp:  streams the packed weight tiles into a weight ring and the activation tiles
//              (BN rows x 128 B per group, landing pre-swizzled for the MMA) into an activation
//              ring; narrow gate/up tiles gather their live token rows four at a time.
//   MMA warp:  one lane issues four tcgen05.mma.kind::f8f6f4 per K-group into one of kNT TMEM
//              partial buffers.  Narrow tiles commit once per stage (the partial's barrier; the
//              widening warps free the A stage and the activation slot from that completion);
//              wide tiles also commit the shared A / activation stage.  The warp owns the TMEM.
//
// Widening (see tc_tiles.cuh for the arithmetic):
//   kUnsigned (narrow tiles, decode: gate/up and down): byte = nibble = E4M3 of (code+8)*2^-9, so TMEM
//     holds 2^-9 * sum_k q_k*(code_k + 8) and the promotion subtracts the offset term with the
//     group's activation sum: acc += 512*s*partial - 8*s*sum_k q_k (one more FMA per element;
//     a tcgen05.mma costs the same issue time at N = 16 as at N = 64, so the offset is cheaper
//     in the promotion than as four more MMAs).
//   signed (wide token tiles, prefill): byte = E4M3(code) by byte-permute lookup (12 integer ops
//     per 8 codes against 2-5 unsigned; the unsigned form needs a [G][BN] group-sum table that
//     wide tiles have no shared memory left for).
//
// Hybrid layers pass an expert -> slab map: the launch then takes only its format's experts and
// reads each one's weights from its slab.
//
// Every mbarrier wait is bounded; a timeout sets a CTA-wide abort flag that turns all later
// waits into no-ops (so the named barrier among the promotion warps stays uniform), records
// the device status, and the CTA frees its TMEM and exits.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"
#include "tc_pipe.cuh"

namespace moe {

// The gathering instance (gate/up on narrow token tiles) fetches its activation rows by token
// (row r of a segment is token sorted[r] / k of the per-token FP8 array [T, K]) and takes s_row
// per token; every other instance reads expert-sorted activation rows [P, K] directly, s_row per
// row.
struct WsGemmArgs {
    const float* s_row;     // gathering: [T] per-token scale; otherwise [P] per-row scale
    const uint16_t* s0;     // [E, R0, K/128] bf16 scales of w0 (gate, or down)
    const uint16_t* s1;     // up scales (SwiGLU instance)
    const int32_t* offsets; // [E + 1]
    int E, R0, K, P;
    float* out;             // SwiGLU: h [P, R0]; plain: Y [P, ldo]
    int ldo;
    unsigned* amax;         // SwiGLU: [P] float bits of max|h| per row
    const int32_t* sorted;  // [P] pair of each sorted row (gathering: token = pair / k)
    int k;
    int T;                  // tokens (rows of the gathered activation tensor)
    // unsigned widening: per (activation row, K-group) sums of the FP8 values the GEMM reads
    // (per token when gathering, per sorted row otherwise), for the +8 offset correction
    const float* qsum;
    // hybrid layers: expert -> slab map (null: slab = expert) and the experts this launch takes
    const int32_t* slot_of = nullptr;
    int slot_want = 0;
};


template <int BN, bool kUnsigned>
struct WsCfg {
    // Narrow token tiles (decode) stream weights as fast as HBM allows: the cheap unsigned
    // widening, 8 widening warps, and for BN = 16 two persistent CTAs per SM.  Wide tiles
    // (prefill) keep more smem for the activation tiles, one CTA per SM.
    static constexpr bool kNarrow = BN <= 32;
    // Every pipeline stage carries kGS K-groups: narrow tiles move two per stage, which halves
    // the waits, commits and TMA issues per weight byte of the single-thread TMA and MMA roles.
    static constexpr int kGS = kNarrow ? 2 : 1;
    static constexpr int kRowB = 64 * kGS;                      // packed bytes per row per stage
    static constexpr int kRaw = 128 * kRowB;                    // packed codes, one stage
    static constexpr int kB = BN * 128;                         // activation tile, one group
    static constexpr int kBSlot = ((kB + 1023) / 1024) * 1024;
    static constexpr int kCtasPerSm = (BN <= 16) ? 2 : 1;       // BN = 16: two CTAs per SM
    // Three rings, in stages: packed weights (shared memory), widened A tiles (TMEM) and
    // activation tiles (shared memory).  With kRB >= kRW + kS a free activation slot is always
    // waiting once a weight slot is, so the one producer lane is paced by the weight ring alone
    // and the activation tiles are fetched kRW stages ahead of their MMAs.
    static constexpr int kRW = (BN <= 16) ? 4 : (BN <= 32 ? 6 : (BN <= 64 ? 12 : 8));  // weight ring
    static constexpr int kS = (BN <= 16) ? 2 : (BN <= 32 ? 4 : (BN <= 64 ? 8 : 4));    // A stages
    // Wide tiles instead share one ring between activation and A tiles (kRB = kS: one "ready"
    // barrier counting the widening warps and the activation bytes, one "free" commit), which
    // saves the MMA lane a wait and a commit per group.
    static constexpr bool kSplitB = kNarrow;
    static constexpr int kRB = kSplitB ? kRW + kS : kS;                                 // activation ring
    static constexpr int kNT = kNarrow ? 8 : (BN <= 64 ? 4 : (BN <= 128 ? 3 : 2));  // TMEM partials
    static constexpr int kNTS = kNT / kGS;                       // partial stages (barrier pairs)
    // TMEM columns: partial buffers | widened A tiles (32 columns = 128 E4M3 per row)
    static constexpr int kColA = kNT * BN;
    static constexpr int kTmemNeed = kColA + kS * kGS * 32;
    static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
    static_assert(kTmemNeed <= 512 / kCtasPerSm, "TMEM budget");
    static constexpr int kUsStride = BN + 1;
    static constexpr int kOffB = 0;
    static constexpr int kOffW = kOffB + kRB * kGS * kBSlot;
    static constexpr int kOffUs = kOffW + kRW * kRaw;
    static constexpr int kOffPre = kOffUs + 64 * kUsStride * 4;
    static constexpr int kOffSoff = kOffPre + 1025 * 4;          // segment offsets [0..E]
    static constexpr int kOffSr = kOffSoff + 1025 * 4;           // 2 x BN per-column scales
    static constexpr int kMaxG = 128;                            // K <= 16384
    static constexpr int kOffQs = kOffSr + 2 * BN * 4;           // unsigned: [G][BN] group sums
    static constexpr int kOffBar = ((kOffQs + (kUnsigned ? kMaxG * BN * 4 : 0) + 7) / 8) * 8;
    static constexpr int kNumBars = 2 * kRW + (kSplitB ? 2 * kRB : 0) + 2 * kS + 2 * kNTS;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;     // TMEM slot, abort flag
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    // Warp roles.  Narrow: warps 0-7 widen, 8-11 promote, 12 TMA, 13 MMA.  Wide: warps 0-3
    // widen, 4-11 promote (two warps per TMEM lane quadrant, each owning half of the token
    // columns), 12 TMA, 13 MMA.  A promotion thread issues up to 32 columns of TMEM loads before
    // each wait, so a 128-column group costs two load round trips.
    static constexpr int kNW = kNarrow ? 8 : 4;                 // widening warps
    static constexpr int kNP = kNarrow ? 4 : (BN >= 128 ? 16 : 8);   // promotion / epilogue warps
    static constexpr int kCPW = BN / (kNP / 4);                 // token columns per promotion thread
    static constexpr int kWarpTma = kNW + kNP, kWarpMma = kNW + kNP + 1;
    // TMEM columns per load wait (16 where 704 threads leave 88 registers per thread)
    static constexpr int kLd = kNP > 8 ? 16 : (kCPW < 32 ? kCPW : 32);
    static constexpr int kThreads = 32 * (kNW + kNP + 2);
};

template <int BN, bool kUnsigned, bool kSwiGLU, bool kGather>
__global__ void __launch_bounds__(WsCfg<BN, kUnsigned>::kThreads, WsCfg<BN, kUnsigned>::kCtasPerSm)
    k_gemm_w4a8_ws(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                   const __grid_constant__ CUtensorMap tm_act, const WsGemmArgs a) {
    using C = WsCfg<BN, kUnsigned>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* bring = sm + C::kOffB;
    uint8_t* wring = sm + C::kOffW;
    float* sUs = reinterpret_cast<float*>(sm + C::kOffUs);
    int* pre = reinterpret_cast<int*>(sm + C::kOffPre);
    int* soff = reinterpret_cast<int*>(sm + C::kOffSoff);
    float* sSr = reinterpret_cast<float*>(sm + C::kOffSr);
    float* sQs = reinterpret_cast<float*>(sm + C::kOffQs);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* w_full = bar;                       // weight ring: TMA -> widening warps
    uint64_t* w_empty = w_full + C::kRW;          //              widening warps -> TMA
    uint64_t* s_ready = w_empty + C::kRW;         // widened A stage: widening warps (+ TMA bytes) -> MMA
    uint64_t* s_free = s_ready + C::kS;           //                  MMA commit -> widening warps
    // activation ring (own barriers on narrow tiles; the A stage's otherwise)
    uint64_t* b_full = C::kSplitB ? s_free + C::kS : s_ready;
    uint64_t* b_empty = C::kSplitB ? b_full + C::kRB : s_free;
    uint64_t* t_full = s_free + C::kS + (C::kSplitB ? 2 * C::kRB : 0);   // TMEM partials: MMA -> promotion
    uint64_t* t_empty = t_full + C::kNTS;         //                promotion -> MMA
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.K / kGroup;
    const int nst = (G + C::kGS - 1) / C::kGS;             // stages per tile
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    if (tid == 0) {
        for (int i = 0; i < C::kRW; ++i) { tc::mbar_init(&w_full[i], 1); tc::mbar_init(&w_empty[i], C::kNW); }
        if (C::kSplitB)
            for (int i = 0; i < C::kRB; ++i) { tc::mbar_init(&b_full[i], 1); tc::mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < C::kS; ++i) {
            tc::mbar_init(&s_ready[i], C::kNW + (C::kSplitB ? 0 : 1));
            tc::mbar_init(&s_free[i], 1);
        }
        for (int i = 0; i < C::kNTS; ++i) { tc::mbar_init(&t_full[i], 1); tc::mbar_init(&t_empty[i], C::kNP); }
        *abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == C::kWarpMma) {
        tc::tmem_alloc(tslot, C::kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tslot;
    // Programmatic dependent launch (common.cuh): the set-up above ran under the predecessor's
    // tail.  The gate/up instance reads the expert offsets of the grid just before it, so it
    // waits now.  The down instance's offsets, weights and scales are older than the grid before
    // it (the requantization), so it reads them and streams its first weight stages before
    // waiting; only the activations and their scales wait.
    if constexpr (kSwiGLU) pdl_enter();
    else pdl_trigger();
    const int row_tiles = row_tile_prefix(a.offsets, a.E, BN, pre, soff, a.slot_of, a.slot_want);
    const int64_t n_tiles = (int64_t)row_tiles * m_tiles;
    if ((int64_t)blockIdx.x >= n_tiles) {
        pdl_wait();                                        // no CTA completes before its predecessor
        if (warp == C::kWarpMma) {
            tc::tc_fence_after();
            tc::tmem_dealloc(tmem, C::kTmemCols);
        }
        return;
    }

    if (warp == C::kWarpTma) {
        // ------------------------------------------------------------ TMA producer
        // Lane 0 owns the barriers and the weight tiles.  Activation tiles are either a box of
        // BN expert-sorted rows, or (kGather) only the tile's live token rows, four per
        // tile::gather4 issued by lanes 0..; rows past the segment are never read back.
        if (lane == 0) {
            ws::prefetch_map(&tm_w0);
            if (kSwiGLU) ws::prefetch_map(&tm_w1);
            ws::prefetch_map(&tm_act);
        }
        ws::Ring<C::kRW> rw;
        ws::Ring<C::kRB> rb;
        int pre_w = 0;                        // weight stages of the first tile issued before the wait
        if constexpr (!kSwiGLU) {
            if (lane == 0) {
                const int rt = static_cast<int>(blockIdx.x / m_tiles), mt = static_cast<int>(blockIdx.x % m_tiles);
                const int wb = weight_slab(a.slot_of, expert_of_tile(pre, a.E, rt));
                pre_w = min(nst, C::kRW);
                for (int st = 0; st < pre_w; ++st) {   // a fresh ring: slots 0.. are free, phase 0
                    tc::mbar_arrive_expect_tx(&w_full[st], C::kRaw);
                    ws::tma_load_2d(wring + st * C::kRaw, &tm_w0, st * C::kGS * 64, wb * a.R0 + mt * 128, &w_full[st]);
                }
            }
            pdl_wait();
        }
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            if (__shfl_sync(0xffffffffu, *abort, 0)) break;
            const int rt = static_cast<int>(tile / m_tiles), mt = static_cast<int>(tile % m_tiles);
            const int e = expert_of_tile(pre, a.E, rt);
            const int row0 = soff[e] + (rt - pre[e]) * BN;
            const int nrows = min(BN, soff[e + 1] - row0);
            const int ngather = (nrows + 3) / 4;
            int tok[4] = {0, 0, 0, 0};
            if (kGather && lane < ngather) {
#pragma unroll
                for (int i = 0; i < 4; ++i) tok[i] = a.sorted[row0 + min(4 * lane + i, nrows - 1)] / a.k;
            }
            const uint32_t b_bytes = kGather ? static_cast<uint32_t>(ngather) * 512u : C::kB;
            bool stop = false;
            for (int st = 0; st < nst; ++st, rw.next(), rb.next()) {
                const int g0 = st * C::kGS, ng = min(C::kGS, G - g0);
                const int ws_ = rw.idx, bs = rb.idx;
                int ok = 1;
                const bool w_issued = !kSwiGLU && tile == blockIdx.x && st < pre_w;
                if (lane == 0) {
                    if (!w_issued) {
                        ok = ws::wait(&w_empty[ws_], rw.phase ^ 1u, abort);
                        if (ok) {
                            // a stage past K (odd group count) is filled with zeros by the TMA unit
                            uint8_t* wst = wring + ws_ * C::kRaw;
                            tc::mbar_arrive_expect_tx(&w_full[ws_], C::kRaw);
                            const int wb = weight_slab(a.slot_of, e);
                            if (kSwiGLU) {
                                const int y = wb * a.R0 + mt * 64;
                                ws::tma_load_2d(wst, &tm_w0, g0 * 64, y, &w_full[ws_]);
                                ws::tma_load_2d(wst + 64 * C::kRowB, &tm_w1, g0 * 64, y, &w_full[ws_]);
                            } else {
                                ws::tma_load_2d(wst, &tm_w0, g0 * 64, wb * a.R0 + mt * 128, &w_full[ws_]);
                            }
                        }
                    }
                    if (ok) {
                        ok = ws::wait(&b_empty[bs], rb.phase ^ 1u, abort);
                        if (ok) tc::mbar_arrive_expect_tx(&b_full[bs], b_bytes * ng);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) { stop = true; break; }
                for (int h = 0; h < ng; ++h) {
                    uint8_t* bst = bring + (bs * C::kGS + h) * C::kBSlot;
                    if (kGather) {
                        if (lane < ngather)
                            ws::tma_gather4(bst + lane * 512, &tm_act, (g0 + h) * kGroup, tok[0], tok[1], tok[2],
                                            tok[3], &b_full[bs]);
                    } else if (lane == 0) {
                        ws::tma_load_2d(bst, &tm_act, (g0 + h) * kGroup, row0, &b_full[bs]);
                    }
                }
            }
            if (stop) break;
        }
    } else if (warp == C::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_e4m3_f32(128, BN);
            // descriptor of activation slot 0; slot i starts i * kBSlot / 16 later in the
            // start-address field, and a K step of 32 bytes adds 2 (1024-byte-aligned tiles in
            // the first 256 KB of shared memory keep the 14-bit field from carrying)
            const uint64_t bd0 = tc::sdesc_sw128(tc::smem_u32(bring));
            ws::Ring<C::kS> rs;
            ws::Ring<C::kNTS> rt;
            ws::Ring<C::kRB> rb;
            uint64_t* last_bar = nullptr;                  // the barrier of the last commit
            uint32_t last_bp = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x) {
                for (int st = 0; st < nst; ++st) {
                    const int ng = C::kGS == 1 ? 1 : min(C::kGS, G - st * C::kGS);
                    if (C::kSplitB && !ws::wait(&b_full[rb.idx], rb.phase, abort)) break;
                    if (!ws::wait(&s_ready[rs.idx], rs.phase, abort)) break;
                    if (!ws::wait(&t_empty[rt.idx], rt.phase ^ 1u, abort)) break;
                    tc::tc_fence_after();
                    for (int h = 0; h < ng; ++h) {
                        const uint64_t bd = bd0 + static_cast<uint64_t>((rb.idx * C::kGS + h) * (C::kBSlot >> 4));
                        const uint32_t a_col = tmem + C::kColA + (rs.idx * C::kGS + h) * 32;
                        const uint32_t d = tmem + (rt.idx * C::kGS + h) * BN;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_e4m3_ta(d, a_col + kk * 8, bd + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                    }
                    tc::mma_commit(&t_full[rt.idx]);
                    if (C::kSplitB) {
                        // one commit per stage: the widening warps free the A stage and the
                        // activation slot from the partial's completion (see below)
                        last_bar = &t_full[rt.idx];
                        last_bp = rt.phase;
                    } else {
                        tc::mma_commit(&s_free[rs.idx]);   // = b_empty: A stage + activation slot
                        last_bar = &s_free[rs.idx];
                        last_bp = rs.phase;
                    }
                    rs.next();
                    rt.next();
                    rb.next();
                }
            }
            // the commits complete in order: once the last one has arrived, no tensor-core
            // arrive on this CTA's barriers is still pending
            if (last_bar) ws::wait(last_bar, last_bp, abort);
        }
    } else if (warp < C::kNW) {
        // ------------------------------------------------------------ widening warps
        // A thread owns one A row = one TMEM lane (warp id % 4 selects the lane quadrant); on
        // narrow tiles two warps split each row's K groups.  The packed stage lands with the
        // 64-byte (one group per row) or 128-byte (two) TMA swizzle: 16-byte chunk c of row r sits
        // at chunk c ^ ((r >> 1) & 3), resp. c ^ (r & 7), so the 32 rows a warp reads fall in
        // distinct banks.
        constexpr int kParts = C::kNW / 4;                 // warps per lane quadrant
        constexpr int kChunks = 4 / kParts;                // 16-byte packed chunks per thread per group
        const int quad = warp & 3, part = warp >> 2;
        const int row = quad * 32 + lane;
        const int swz = C::kGS == 1 ? (row >> 1) & 3 : row & 7;
        const uint32_t t_dst = tmem + (static_cast<uint32_t>(quad * 32) << 16) + C::kColA + part * 8 * kChunks;
        ws::Ring<C::kRW> rw;
        ws::Ring<C::kS> ra;
        uint32_t g = 0;                                    // stages so far, in the MMA's order
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            for (int st = 0; st < nst; ++st, rw.next(), ra.next(), ++g) {
                const int ws_ = rw.idx, as = ra.idx;
                ws::wait(&w_full[ws_], rw.phase, abort);
                const uint8_t* raw = wring + ws_ * C::kRaw + row * C::kRowB;
                uint4 w[C::kGS][kChunks];
#pragma unroll
                for (int h = 0; h < C::kGS; ++h)
#pragma unroll
                    for (int p = 0; p < kChunks; ++p)
                        w[h][p] = *reinterpret_cast<const uint4*>(raw + (((4 * h + part * kChunks + p) ^ swz) << 4));
                tc::fence_proxy_async_smem();              // order these reads before the next TMA write
                __syncwarp();                              // this warp's reads of the slot are done
                if (lane == 0) tc::mbar_arrive(&w_empty[ws_]);
                if constexpr (C::kSplitB) {
                    // A stage `as` was last read by the MMAs of stage g - kS, whose completion is
                    // the commit on that stage's partial buffer.  kNTS >= kS, so that buffer's
                    // barrier cannot have completed a later phase yet and its parity is unambiguous.
                    // The same completion frees the activation slot of stage g - kS.
                    static_assert(C::kNTS >= C::kS, "partial ring shorter than the A ring");
                    if (g >= static_cast<uint32_t>(C::kS)) {
                        const uint32_t gp = g - C::kS;
                        ws::wait(&t_full[gp % C::kNTS], (gp / C::kNTS) & 1u, abort);
                        if (warp == 0 && lane == 0) tc::mbar_arrive(&b_empty[gp % C::kRB]);
                    }
                } else {
                    ws::wait(&s_free[as], ra.phase ^ 1u, abort);
                }
                tc::tc_fence_after();
#pragma unroll
                for (int h = 0; h < C::kGS; ++h) {
                    uint32_t o[8 * kChunks];
#pragma unroll
                    for (int p = 0; p < kChunks; ++p) {
                        const uint32_t ww[4] = {w[h][p].x, w[h][p].y, w[h][p].z, w[h][p].w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint2 x = widen8<kUnsigned>(ww[q]);
                            o[8 * p + 2 * q] = x.x;
                            o[8 * p + 2 * q + 1] = x.y;
                        }
                    }
                    const uint32_t dst = t_dst + (as * C::kGS + h) * 32;
                    if constexpr (kChunks == 2) tc::tmem_st16(dst, o);
                    else tc::tmem_st32(dst, o);
                }
                tc::tmem_wait_st();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&s_ready[as]);
            }
        }
    } else if (warp < C::kNW + C::kNP) {
        // ------------------------------------------------------------ promotion + epilogue warps
        if constexpr (!kSwiGLU) pdl_wait();                // s_row: the requantization's scales
        // Promotion warp i owns TMEM lanes 32*(i % 4) .. +31 (warp id % 4 selects the lanes) and
        // the token columns [ch*kCPW, (ch+1)*kCPW) of them.
        constexpr int kCPW = C::kCPW;
        constexpr int kNPT = 32 * C::kNP;
        const int pt = tid - 32 * C::kNW;                 // 0 .. kNPT-1
        const int ch = (warp - C::kNW) >> 2;              // column block of this warp
        const int c_base = ch * kCPW;
        const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int lrow = (warp & 3) * 32 + lane;           // this thread's A row / TMEM lane
        // group-scale row of this thread in a tile; the first scales of the next tile are fetched
        // before the current tile's epilogue so that a tile never starts on a DRAM round trip
        auto scale_row = [&](int64_t t) -> const uint16_t* {
            const int rt_ = static_cast<int>(t / m_tiles), mt_ = static_cast<int>(t % m_tiles);
            const int b_ = weight_slab(a.slot_of, expert_of_tile(pre, a.E, rt_));
            if (kSwiGLU)
                return (lrow < 64 ? a.s0 : a.s1) + ((int64_t)b_ * a.R0 + mt_ * 64 + (lrow & 63)) * G;
            return a.s0 + ((int64_t)b_ * a.R0 + mt_ * 128 + lrow) * G;
        };
        uint16_t first_raw[C::kGS];
        if (kSwiGLU && !C::kNarrow) {
            const uint16_t* s0 = scale_row(blockIdx.x);
#pragma unroll
            for (int h = 0; h < C::kGS; ++h) first_raw[h] = h < G ? __ldg(s0 + h) : uint16_t(0);
        }
        uint32_t tcount = 0;
        ws::Ring<C::kNTS> rq;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const int rt = static_cast<int>(tile / m_tiles), mt = static_cast<int>(tile % m_tiles);
            const int e = expert_of_tile(pre, a.E, rt);
            const int seg0 = soff[e];
            const int r0 = (rt - pre[e]) * BN;
            const int nrows = min(BN, soff[e + 1] - seg0 - r0);
            const int64_t row0 = seg0 + r0;
            // token scale of column pt, fetched now and staged in shared memory for the epilogue
            float my_sr = 0.0f;
            if (pt < nrows) my_sr = kGather ? a.s_row[a.sorted[row0 + pt] / a.k] : a.s_row[row0 + pt];
            float* sr_t = sSr + (tcount & 1) * BN;         // two buffers: tile parity
            ++tcount;
            const uint16_t* ssrc = scale_row(tile);
            (void)mt;
            if constexpr (kUnsigned) {   // the tile's activation group sums, sQs[g * BN + j]
                for (int i = pt; i < G * BN; i += kNPT) {
                    const int j = i / G, g = i - j * G;
                    float v = 0.0f;
                    if (j < nrows) {
                        const int64_t rr = kGather ? (int64_t)(a.sorted[row0 + j] / a.k) : row0 + j;
                        v = a.qsum[rr * G + g];
                    }
                    sQs[g * BN + j] = v;
                }
                ws::named_sync_math<kNPT>();
            }
            float acc[kCPW];
#pragma unroll
            for (int j = 0; j < kCPW; ++j) acc[j] = 0.0f;
            float sc_next[C::kGS];
#pragma unroll
            for (int h = 0; h < C::kGS; ++h)
                sc_next[h] = bf16_bits_to_f32((C::kNarrow || !kSwiGLU) ? (h < G ? __ldg(ssrc + h) : uint16_t(0))
                                                                        : first_raw[h]);
            for (int st = 0; st < nst; ++st, rq.next()) {
                const int g0 = st * C::kGS;
                float scs[C::kGS];
#pragma unroll
                for (int h = 0; h < C::kGS; ++h) {
                    scs[h] = sc_next[h];
                    const int gn = g0 + C::kGS + h;
                    if (gn < G) sc_next[h] = bf16_bits_to_f32(__ldg(ssrc + gn));
                }
                const int ts = rq.idx;
                ws::wait(&t_full[ts], rq.phase, abort);
                tc::tc_fence_after();
#pragma unroll
                for (int h = 0; h < C::kGS; ++h) {
                    const int g = g0 + h;
                    if (g >= G) break;
                    const float sc = kUnsigned ? scs[h] * 512.0f : scs[h];
                    const uint32_t tcol = tmem + t_lane + (ts * C::kGS + h) * BN + c_base;
#pragma unroll
                    for (int c1 = 0; c1 < kCPW; c1 += C::kLd) {    // kLd columns in flight per wait
                        uint32_t v[C::kLd];
#pragma unroll
                        for (int c0 = 0; c0 < C::kLd; c0 += 16)
                            tc::tmem_ld16(tcol + c1 + c0, *reinterpret_cast<uint32_t(*)[16]>(v + c0));
                        tc::tmem_wait_ld();
                        // two columns per packed fp32 FMA (same rounding as two fmaf)
                        const float2 sc2 = make_float2(sc, sc);
#pragma unroll
                        for (int j = 0; j < C::kLd; j += 2) {
                            const float2 r = __ffma2_rn(sc2, make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])),
                                                        make_float2(acc[c1 + j], acc[c1 + j + 1]));
                            acc[c1 + j] = r.x;
                            acc[c1 + j + 1] = r.y;
                        }
                        if constexpr (kUnsigned) {   // minus 8 * s * (group sum of the column's q)
                            const float scm = sc * (-1.0f / 64.0f);
                            const float2 scm2 = make_float2(scm, scm);
                            const float* qg = sQs + g * BN + c_base + c1;
#pragma unroll
                            for (int j = 0; j < C::kLd; j += 2) {
                                const float2 r = __ffma2_rn(scm2, make_float2(qg[j], qg[j + 1]),
                                                            make_float2(acc[c1 + j], acc[c1 + j + 1]));
                                acc[c1 + j] = r.x;
                                acc[c1 + j + 1] = r.y;
                            }
                        }
                    }
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&t_empty[ts]);
            }

            if (kSwiGLU && !C::kNarrow && tile + gridDim.x < n_tiles) {   // wide gate/up tiles only
                const uint16_t* sn = scale_row(tile + gridDim.x);
#pragma unroll
                for (int h = 0; h < C::kGS; ++h) first_raw[h] = h < G ? __ldg(sn + h) : uint16_t(0);
            }

            // ---- epilogue (static indices keep acc[] in registers) ----
            // The column scales come from shared memory, so no load waits behind the stores, and
            // the per-column max|h| is one redux per warp.
            if (pt < BN) sr_t[pt] = my_sr;
            if constexpr (kSwiGLU) {
                // Gate warps (lrow < 64) finish the first half of the columns, up warps the second:
                // each hands the other the half it does not finish through sUs.
                constexpr int kHalf = kCPW / 2;
                const bool gate = lrow < 64;
                const int r64 = lrow & 63;
                const int c_mine = c_base + (gate ? 0 : kHalf);
#pragma unroll
                for (int j = 0; j < kHalf; ++j)
                    sUs[r64 * C::kUsStride + c_base + (gate ? kHalf : 0) + j] = gate ? acc[kHalf + j] : acc[j];
                ws::named_sync_math<kNPT>();
                const int n = mt * 64 + r64;
#pragma unroll
                for (int j = 0; j < kHalf; ++j) {
                    const float sr = sr_t[c_mine + j];
                    const float other = sUs[r64 * C::kUsStride + c_mine + j];
                    const float gv = gate ? acc[j] : other;
                    const float uv = gate ? other : acc[kHalf + j];
                    acc[j] = silu_fast(gv * sr) * (uv * sr);
                }
#pragma unroll
                for (int j = 0; j < kHalf; ++j)
                    if (c_mine + j < nrows) a.out[(row0 + c_mine + j) * a.ldo + n] = acc[j];
#pragma unroll
                for (int j = 0; j < kHalf; ++j) {
                    const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(acc[j])));
                    if (lane == 0 && c_mine + j < nrows) atomicMax(a.amax + row0 + c_mine + j, m);
                }
                ws::named_sync_math<kNPT>();                  // exchange buffer free again
            } else {
                const int m = mt * 128 + lrow;
                ws::named_sync_math<kNPT>();
#pragma unroll
                for (int j = 0; j < kCPW; ++j)
                    if (c_base + j < nrows) a.out[(row0 + c_base + j) * a.ldo + m] = acc[j] * sr_t[c_base + j];
            }
        }
    }

    __syncwarp();          // single-lane roles reconverge before the CTA-wide barrier
    if constexpr (!kSwiGLU) pdl_wait();   // (returns at once in the roles that waited already)
    __syncthreads();
    if (*abort && tid == 0) atomicOr(&g_device_status, kStatusTimeout);
    if (warp == C::kWarpMma) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---- host side --------------------------------------------------------------------------------

template <int BN, bool kUnsigned, bool kSwiGLU, bool kGather>
int launch_gemm_ws_inst(const WsGemmArgs& a, const void* act, const void* w0, const void* w1,
                        int64_t max_row_tiles, cudaStream_t stream) {
    using C = WsCfg<BN, kUnsigned>;
    if (kUnsigned && !a.qsum) return MOE_ERR_INVALID_ARG;   // the +8 offset needs the group sums
    static TcLaunchShape cache[16];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    auto kern = k_gemm_w4a8_ws<BN, kUnsigned, kSwiGLU, kGather>;
    TcLaunchShape& c = cache[dev & 15];
    if (c.sms == 0) {
        int sms = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kAlloc) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        c.ctas_per_sm = C::kCtasPerSm;
        c.sms = sms;
    }
    CUtensorMap m0, m1, mact;
    const int rows_per_load = kSwiGLU ? 64 : 128;
    const CUtensorMapSwizzle wsw = C::kGS == 1 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_map_u8(&m0, w0, a.K / 2, (uint64_t)a.E * a.R0, C::kRowB, rows_per_load, wsw) ||
        !make_map_u8(&m1, kSwiGLU ? w1 : w0, a.K / 2, (uint64_t)a.E * a.R0, C::kRowB, rows_per_load, wsw) ||
        !make_map_u8(&mact, act, a.K, kGather ? (uint64_t)a.T : (uint64_t)a.P, 128, kGather ? 1 : BN,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return MOE_ERR_CUDA;
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    const int64_t grid = std::max<int64_t>(
        1, std::min<int64_t>(max_row_tiles * m_tiles, (int64_t)c.sms * c.ctas_per_sm));
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(C::kThreads), C::kAlloc, stream, m0, m1,
                      mact, a);
}

// Narrow token tiles (decode): the gate/up instance gathers its activation rows by token from the
// per-token FP8 array instead of an expert-sorted copy.
inline bool ws_narrow(int BN) { return BN <= 32; }

// A W4A8 layer on 128-row tiles (segments of 24 to 160 rows on average, typically skewed) runs
// its segments of at most kShortRows rows on 32-row tiles, which widen unsigned and cost a
// quarter of the integer work per weight: at T = 2048 with Zipf routing 84 of 184 128-row tiles
// hold at most 32 rows (5 % of the rows).  Only where both reductions span at least sixteen
// K-groups (H, N >= 2048, the model's depths): the unsigned form's +8-biased sums lose up to half
// an fp32 ulp each, which averages out over many groups but not over a few, and a requantized
// code it tips over moves its token's outputs by ~1/N (measured on random layers: split, a
// 256 x 128 layer put an output at 2.8 x the tolerance, 0.78 x unsplit; at 1024 x 1024 one
// layer reached 1.36 x split; at 4096 x 2048 every case stays within 0.78 x).
inline bool ws_split(int64_t P, int E, int H, int N) {
    return H >= 16 * kGroup && N >= 16 * kGroup && ws_tile_rows(P, E) == 128;
}

// bn: the token-tile width (0: chosen from the average segment length, ws_tile_rows);
// rows_sorted: a narrow gate/up launch reads expert-sorted activation rows instead of gathering
// them by token (the short segments of a layer whose other segments run on wide tiles).
template <bool kSwiGLU>
int launch_gemm_ws(const WsGemmArgs& a, const void* act, const void* w0, const void* w1,
                   cudaStream_t stream, int bn = 0, bool rows_sorted = false) {
    const int BN = bn ? bn : ws_tile_rows(a.P, a.E);
    const int64_t max_row_tiles = ((int64_t)a.P + BN - 1) / BN + a.E;
    switch (BN) {
        // narrow tiles (decode) widen unsigned: the tensor core sums the +8-offset products in fp32
        // without loss (measured: exact, or 0.5 ulp, over 128-wide groups), and the promotion
        // removes the offset with the activation rows' group sums (per token for the gathering
        // gate/up instance, per sorted row otherwise)
        case 16: return launch_gemm_ws_inst<16, true, kSwiGLU, kSwiGLU>(a, act, w0, w1, max_row_tiles, stream);
        case 32:
            if (kSwiGLU && rows_sorted)
                return launch_gemm_ws_inst<32, true, kSwiGLU, false>(a, act, w0, w1, max_row_tiles, stream);
            return launch_gemm_ws_inst<32, true, kSwiGLU, kSwiGLU>(a, act, w0, w1, max_row_tiles, stream);
        case 128: return launch_gemm_ws_inst<128, false, kSwiGLU, false>(a, act, w0, w1, max_row_tiles, stream);
        default: return launch_gemm_ws_inst<192, false, kSwiGLU, false>(a, act, w0, w1, max_row_tiles, stream);
    }
}

}  // namespace moe
