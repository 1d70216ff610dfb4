// gemm_w8a8.cuh — the grouped expert GEMMs of the row-scaled FP8 (W8A8) expert format.
//
// Format: the "Inkling 2 Small FP8 for AMD MI300X" card, "Precision and files": E4M3 expert
// weights with one fp32 scale per expert output channel, run on per-token FP8 activations.
// Both operands are tensor-core types already, so unlike the W4A8 GEMM nothing is widened and
// nothing is promoted per K-group: the tensor core accumulates the whole of K in TMEM and the
// epilogue applies the two scales once,  out[t, n] = (acc[n, t] * s_w[n]) * s_x[t].
//
// Roles (one persistent CTA per SM, 192 threads):
//   warps 0-3  epilogue: thread = TMEM lane = weight row; drains one of two TMEM accumulators
//              while the tensor core fills the other.
//   warp 4     TMA: per 128-wide K step, the 128 weight rows x 128 B and the token tile
//              (BN rows x 128 B; the gathering instance fetches only the tile's live token rows,
//              four per tile::gather4) into one stage of a ring, both landing in the 128-byte
//              swizzle the MMA reads.
//   warp 5     MMA: one lane issues four tcgen05.mma.kind::f8f6f4 (K = 32 each) per stage,
//              commits the stage back to the TMA warp and, after a tile's last stage, the
//              accumulator to the epilogue warps; the warp owns the TMEM.  The MMA's N is the
//              tile's live rows rounded up to 16 (a runtime field of the instruction
//              descriptor), so a segment's last, partly filled tile costs only what it holds.
// Swap AB as in the W4A8 GEMM: MMA M = 128 weight rows (gate/up: 64 gate rows and the same 64
// up rows), N = BN tokens of one expert's segment.  The epilogues are the W4A8 GEMM's: SwiGLU
// with max|h| per row, or the plain projection; the requantization and the combine run as
// their own passes after the GEMMs.
//
// Every mbarrier wait is bounded; a timeout sets the CTA's abort flag, later waits give up at
// once, the device status is recorded and the CTA frees its TMEM and exits.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"
#include "tc_pipe.cuh"

namespace moe {

struct W8GemmArgs {
    const float* s_row;     // gathering: [T] per-token scale; otherwise [P] per-row scale
    const float* rs0;       // [E, R0] fp32 row scales of w0 (gate, or down)
    const float* rs1;       // [E, R0] up row scales (SwiGLU instance)
    const int32_t* offsets; // [E + 1]
    int E, R0, K, P;
    float* out;             // SwiGLU: h [P, R0]; plain: Y [P, ldo]
    int ldo;
    unsigned* amax;         // SwiGLU: [P] float bits of max|h| per row
    const int32_t* sorted;  // [P] pair of each sorted row (gathering: token = pair / k)
    int k;
    int T;                  // tokens (rows of the gathered activation tensor)
};

template <int BN>
struct W8Cfg {
    static constexpr bool kNarrow = BN <= 32;
    static constexpr int kA = 128 * 128;                    // 128 weight rows x 128 E4M3
    static constexpr int kB = BN * 128;                     // BN token rows x 128 E4M3
    static constexpr int kStage = kA + kB;                  // a multiple of 1024
    static_assert(kStage % 1024 == 0, "stage alignment");
    // ring depth: about 190 KB of stages in flight per SM
    static constexpr int kRS = BN <= 32 ? 10 : (BN <= 64 ? 8 : (BN <= 128 ? 6 : 4));
    static constexpr int kChunk = BN < 32 ? BN : 32;        // TMEM columns per epilogue load
    static constexpr int kXStride = kChunk + 1;             // SwiGLU exchange: 64 x kChunk (+1)
    static constexpr int kOffX = kRS * kStage;
    static constexpr int kOffPre = kOffX + 64 * kXStride * 4;
    static constexpr int kOffSoff = kOffPre + 1025 * 4;     // segment offsets [0..E]
    static constexpr int kOffSr = kOffSoff + 1025 * 4;      // 2 x BN column scales
    static constexpr int kOffBar = ((kOffSr + 2 * BN * 4 + 7) / 8) * 8;
    static constexpr int kNumBars = 2 * kRS + 4;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8; // TMEM slot, abort flag
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static constexpr int kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;   // two accumulators
    static constexpr int kThreads = 192;
    static constexpr int kWarpTma = 4, kWarpMma = 5;
};

// The epilogue warps (threads 0..127, thread = TMEM lane = weight row): every tile's accumulator
// times the tile's row scale rs_of(expert, m tile, row) and the column (token) scales, then the
// SwiGLU epilogue (h and max|h| per row) or the plain one (Y rows).  Shared by the FP8 and NVFP4
// expert GEMMs, whose accumulators both hold the whole K.
template <int BN, bool kSwiGLU, bool kGather, class RowScale>
__device__ __forceinline__ void w8_epilogue_warps(const W8GemmArgs& a, int64_t n_tiles, int m_tiles,
                                                  const int* pre, const int* soff, float* sSr, float* sX,
                                                  uint32_t tmem, uint64_t* t_full,
                                                  uint64_t* t_empty, volatile int* abort, RowScale rs_of) {
    constexpr int kXS = (BN < 32 ? BN : 32) + 1;         // SwiGLU exchange row stride
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kNPT = 128;
    constexpr int kCh = BN < 32 ? BN : 32;            // TMEM columns per load
    const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
    const int lrow = tid;                              // A row = TMEM lane
    uint32_t tcount = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tcount) {
        const int rt = static_cast<int>(tile / m_tiles), mt = static_cast<int>(tile % m_tiles);
        const int e = expert_of_tile(pre, a.E, rt);
        const int64_t row0 = soff[e] + (rt - pre[e]) * BN;
        const int nrows = min(BN, soff[e + 1] - static_cast<int>(row0));
        float* sr_t = sSr + (tcount & 1) * BN;         // two buffers: tile parity
        for (int c = tid; c < BN; c += kNPT) {
            float v = 0.0f;
            if (c < nrows) v = kGather ? a.s_row[a.sorted[row0 + c] / a.k] : a.s_row[row0 + c];
            sr_t[c] = v;
        }
        const float rs = rs_of(e, mt, lrow);
        const int tb = tcount & 1;
        ws::wait(&t_full[tb], (tcount >> 1) & 1, abort);
        tc::tc_fence_after();
        ws::named_sync_math<kNPT>();                   // column scales visible
        const uint32_t tcol = tmem + t_lane + tb * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < nrows; c0 += kCh) {       // only the columns the MMA wrote
            uint32_t v[kCh];
            if constexpr (kCh == 32) tc::tmem_ld32(tcol + c0, *reinterpret_cast<uint32_t(*)[32]>(v));
            else tc::tmem_ld16(tcol + c0, *reinterpret_cast<uint32_t(*)[16]>(v));
            tc::tmem_wait_ld();
            float val[kCh];
#pragma unroll
            for (int j = 0; j < kCh; ++j) val[j] = __fmul_rn(__fmul_rn(__uint_as_float(v[j]), rs), sr_t[c0 + j]);
            if constexpr (kSwiGLU) {
                // gate rows finish the first half of the columns, up rows the second; each
                // hands the other the half it does not finish
                constexpr int kHalf = kCh / 2;
                const bool gate = lrow < 64;
                const int r64 = lrow & 63;
#pragma unroll
                for (int j = 0; j < kHalf; ++j)
                    sX[r64 * kXS + (gate ? kHalf : 0) + j] = gate ? val[kHalf + j] : val[j];
                ws::named_sync_math<kNPT>();
                const int cm = c0 + (gate ? 0 : kHalf);
                const int n = mt * 64 + r64;
                float hv[kHalf];
#pragma unroll
                for (int j = 0; j < kHalf; ++j) {
                    const float other = sX[r64 * kXS + (gate ? 0 : kHalf) + j];
                    const float gv = gate ? val[j] : other;
                    const float uv = gate ? other : val[kHalf + j];
                    hv[j] = silu_fast(gv) * uv;
                }
#pragma unroll
                for (int j = 0; j < kHalf; ++j)
                    if (cm + j < nrows) a.out[(row0 + cm + j) * a.ldo + n] = hv[j];
#pragma unroll
                for (int j = 0; j < kHalf; ++j) {
                    const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(hv[j])));
                    if (lane == 0 && cm + j < nrows) atomicMax(a.amax + row0 + cm + j, m);
                }
                ws::named_sync_math<kNPT>();           // exchange buffer free again
            } else {
                const int m = mt * 128 + lrow;
#pragma unroll
                for (int j = 0; j < kCh; ++j)
                    if (c0 + j < nrows) a.out[(row0 + c0 + j) * a.ldo + m] = val[j];
            }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&t_empty[tb]);
    }
}

template <int BN, bool kSwiGLU, bool kGather>
__global__ void __launch_bounds__(W8Cfg<BN>::kThreads, 1)
    k_gemm_w8a8(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                const __grid_constant__ CUtensorMap tm_act, const W8GemmArgs a) {
    pdl_enter();
    using C = W8Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = sm;
    float* sX = reinterpret_cast<float*>(sm + C::kOffX);
    int* pre = reinterpret_cast<int*>(sm + C::kOffPre);
    int* soff = reinterpret_cast<int*>(sm + C::kOffSoff);
    float* sSr = reinterpret_cast<float*>(sm + C::kOffSr);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* full = bar;                  // stage filled: TMA bytes -> MMA
    uint64_t* empty = bar + C::kRS;        // stage read: MMA commit -> TMA
    uint64_t* t_full = bar + 2 * C::kRS;   // accumulator done: MMA commit -> epilogue
    uint64_t* t_empty = t_full + 2;        // accumulator drained: epilogue warps -> MMA
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int steps = a.K / 128;                           // K steps per tile
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    const int row_tiles = row_tile_prefix(a.offsets, a.E, BN, pre, soff);
    const int64_t n_tiles = (int64_t)row_tiles * m_tiles;
    if ((int64_t)blockIdx.x >= n_tiles) return;

    if (tid == 0) {
        for (int i = 0; i < C::kRS; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&t_full[i], 1); tc::mbar_init(&t_empty[i], 4); }
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

    if (warp == C::kWarpTma) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ws::prefetch_map(&tm_w0);
            if (kSwiGLU) ws::prefetch_map(&tm_w1);
            ws::prefetch_map(&tm_act);
        }
        ws::Ring<C::kRS> r;
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
            for (int s = 0; s < steps; ++s, r.next()) {
                uint8_t* st = ring + r.idx * C::kStage;
                int ok = 1;
                if (lane == 0) {
                    ok = ws::wait(&empty[r.idx], r.phase ^ 1u, abort);
                    if (ok) {
                        tc::mbar_arrive_expect_tx(&full[r.idx], C::kA + b_bytes);
                        if (kSwiGLU) {
                            const int y = e * a.R0 + mt * 64;
                            ws::tma_load_2d(st, &tm_w0, s * 128, y, &full[r.idx]);
                            ws::tma_load_2d(st + 64 * 128, &tm_w1, s * 128, y, &full[r.idx]);
                        } else {
                            ws::tma_load_2d(st, &tm_w0, s * 128, e * a.R0 + mt * 128, &full[r.idx]);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) { stop = true; break; }
                if (kGather) {
                    if (lane < ngather)
                        ws::tma_gather4(st + C::kA + lane * 512, &tm_act, s * 128, tok[0], tok[1], tok[2],
                                        tok[3], &full[r.idx]);
                } else if (lane == 0) {
                    ws::tma_load_2d(st + C::kA, &tm_act, s * 128, row0, &full[r.idx]);
                }
            }
            if (stop) break;
        }
    } else if (warp == C::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_full = tc::idesc_e4m3_f32(128, BN);
            // descriptors of stage 0; stage i starts i * kStage / 16 later in the start-address
            // field and a K step of 32 bytes adds 2 (1024-byte-aligned tiles in the first 256 KB
            // of shared memory keep the 14-bit field from carrying)
            const uint64_t ad0 = tc::sdesc_sw128(tc::smem_u32(ring));
            const uint64_t bd0 = tc::sdesc_sw128(tc::smem_u32(ring + C::kA));
            ws::Ring<C::kRS> r;
            uint32_t tcount = 0;
            int last = -1;
            uint32_t last_phase = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x, ++tcount) {
                const int tb = tcount & 1;
                const int rt = static_cast<int>(tile / m_tiles);
                const int e = expert_of_tile(pre, a.E, rt);
                const int nrows = min(BN, soff[e + 1] - soff[e] - (rt - pre[e]) * BN);
                const int n_mma = min(BN, (nrows + 15) & ~15);
                const uint32_t idesc = n_mma == BN ? idesc_full : tc::idesc_e4m3_f32(128, n_mma);
                if (!ws::wait(&t_empty[tb], ((tcount >> 1) & 1) ^ 1u, abort)) break;
                tc::tc_fence_after();
                const uint32_t d = tmem + tb * BN;
                bool stop = false;
                for (int s = 0; s < steps; ++s, r.next()) {
                    if (!ws::wait(&full[r.idx], r.phase, abort)) { stop = true; break; }
                    tc::tc_fence_after();
                    const uint64_t so = static_cast<uint64_t>(r.idx * (C::kStage >> 4));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_e4m3(d, ad0 + so + 2 * kk, bd0 + so + 2 * kk, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&empty[r.idx]);
                    last = r.idx;
                    last_phase = r.phase;
                }
                if (stop) break;
                tc::mma_commit(&t_full[tb]);
            }
            // the commits complete in order: once the last one has arrived, no tensor-core
            // arrive on this CTA's barriers is still pending
            if (last >= 0) ws::wait(&empty[last], last_phase, abort);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps 0-3
        w8_epilogue_warps<BN, kSwiGLU, kGather>(
            a, n_tiles, m_tiles, pre, soff, sSr, sX, tmem, t_full, t_empty, abort,
            [&](int e, int mt, int lrow) {
                return kSwiGLU ? __ldg((lrow < 64 ? a.rs0 : a.rs1) + (int64_t)e * a.R0 + mt * 64 + (lrow & 63))
                               : __ldg(a.rs0 + (int64_t)e * a.R0 + mt * 128 + lrow);
            });
    }

    __syncwarp();          // single-lane roles reconverge before the CTA-wide barrier
    __syncthreads();
    if (*abort && tid == 0) atomicOr(&g_device_status, kStatusTimeout);
    if (warp == C::kWarpMma) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---- host side --------------------------------------------------------------------------------

template <int BN, bool kSwiGLU, bool kGather>
int launch_gemm_w8a8_inst(const W8GemmArgs& a, const void* act, const void* w0, const void* w1,
                          int64_t max_row_tiles, cudaStream_t stream) {
    using C = W8Cfg<BN>;
    static int sms_cache[16] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    auto kern = k_gemm_w8a8<BN, kSwiGLU, kGather>;
    if (sms_cache[dev & 15] == 0) {
        int sms = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kAlloc) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        sms_cache[dev & 15] = sms;
    }
    CUtensorMap m0, m1, mact;
    const int rows_per_load = kSwiGLU ? 64 : 128;
    if (!make_map_u8(&m0, w0, a.K, (uint64_t)a.E * a.R0, 128, rows_per_load, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_u8(&m1, kSwiGLU ? w1 : w0, a.K, (uint64_t)a.E * a.R0, 128, rows_per_load,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_u8(&mact, act, a.K, kGather ? (uint64_t)a.T : (uint64_t)a.P, 128, kGather ? 1 : BN,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return MOE_ERR_CUDA;
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(max_row_tiles * m_tiles, sms_cache[dev & 15]));
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(C::kThreads), C::kAlloc, stream, m0, m1, mact,
                      a);
}

// Token-tile width for the expected rows per expert: the narrow decode widths of the W4A8 GEMM
// (16 / 32 rows), else 256 rows.  A wide tile's MMA N follows its live rows, so short segments
// cost little more than in a narrower tile, while long ones re-read each weight stage for 256
// tokens instead of 64 or 128 (measured: the Zipf T = 2048 gate/up GEMM 0.67 -> 0.46 ms, T =
// 16384 36 -> 50 % of the FP8 peak).  Narrow tiles gather their gate/up activation rows by
// token.
inline int w8_tile_rows(int64_t P, int E) {
    const int BN = tc_tile_rows(P, E);
    return BN <= 32 ? BN : 256;
}

template <bool kSwiGLU>
int launch_gemm_w8a8(const W8GemmArgs& a, const void* act, const void* w0, const void* w1,
                     cudaStream_t stream) {
    const int BN = w8_tile_rows(a.P, a.E);
    const int64_t max_row_tiles = ((int64_t)a.P + BN - 1) / BN + a.E;
    switch (BN) {
        case 16: return launch_gemm_w8a8_inst<16, kSwiGLU, kSwiGLU>(a, act, w0, w1, max_row_tiles, stream);
        case 32: return launch_gemm_w8a8_inst<32, kSwiGLU, kSwiGLU>(a, act, w0, w1, max_row_tiles, stream);
        default: return launch_gemm_w8a8_inst<256, kSwiGLU, false>(a, act, w0, w1, max_row_tiles, stream);
    }
}

}  // namespace moe
