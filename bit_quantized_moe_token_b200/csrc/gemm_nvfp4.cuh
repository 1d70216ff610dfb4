// gemm_nvfp4.cuh — the grouped expert GEMMs of the NVFP4 expert format.
//
// Weights: E2M1 codes with an E4M3 scale per 16 input weights and an fp32 scale2 per expert
// ("Inkling-512k-NVFP4-AQLM-hybrid" card, "Dequant math"), run on the layer's per-token FP8
// activations.  The block scales change every 16 weights along K, so they cannot be promoted
// per K-group like the W4A8 scales, and LUT[code] * scale has up to six significant bits, more
// than E4M3 holds.  It fits f16 exactly (so does every E4M3 activation), and an f16 tcgen05 MMA
// (kind::f16, K = 16 per instruction = one block) accumulates the whole of K in TMEM:
//     out[t, n] = (sum_k f16(LUT[c] * scale)[n, k] * f16(dec q)[t, k]) * scale2 * s_x[t]
// with every product exact in fp32.
//
// Roles (persistent CTAs of 320 threads; two per SM on 16-row tiles, else one):
//   warps 0-3  epilogue (the FP8 GEMM's, with scale2 as the row scale)
//   warps 4-7  widening: thread = weight row = TMEM lane; per 128-wide K step the row's 64 code
//              bytes (from the TMA stage) and its 8 block scales (global, fetched a step ahead)
//              become 128 f16 values written into a TMEM A stage with tcgen05.st
//   warp 8     TMA: per K step the 128 rows x 64 B of codes and the token tile (BN rows x 128
//              f16 as two 128-byte-swizzled boxes; narrow gate/up tiles gather their live token
//              rows four at a time) into one stage of a ring
//   warp 9     MMA: eight tcgen05.mma.kind::f16 per K step, A from TMEM, B from the stage; the
//              warp owns the TMEM
// Every mbarrier wait is bounded, as in the other GEMMs.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"
#include "tc_pipe.cuh"
#include "gemm_w8a8.cuh"

namespace moe {

struct F4GemmArgs {
    W8GemmArgs b;             // shapes, activations (f16 rows), epilogue; b.rs0 / b.rs1 unused
    const uint8_t* bs0;       // [E * R0, K / 16] E4M3 block scales of w0 (gate, or down)
    const uint8_t* bs1;       // up block scales (SwiGLU instance)
    const float* s2_0;        // [E] scale2 of w0
    const float* s2_1;        // [E] scale2 of w1
    // hybrid layers: expert -> slab map (null: slab = expert) and the experts this launch takes
    const int32_t* slot_of = nullptr;
    int slot_want = 0;
};

namespace tc {
// Instruction descriptor: kind::f16 with A = B = F16, D = F32, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
// D[tmem] (+)= A[tmem] * B[smem]^T, one 128 x N x 16 step of f16 inputs (A: two f16 per column).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
}  // namespace tc

// Eight E2M1 codes of one word (code j in bits 4j..4j+3) -> four f16x2 words in K order, each
// multiplied exactly by the block scale s2h (an f16x2 holding the scale twice).  An E2M1 value's
// f16 encoding has a zero low byte; its high byte comes from an 8-entry byte table (prmt) and
// the code's sign bit.
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, __half2 s2h, uint32_t (&o)[4]) {
    constexpr uint32_t kT0 = 0x3E3C3800u, kT1 = 0x46444240u;   // high bytes of 0 .5 1 1.5 | 2 3 4 6
    const uint32_t ws = w << 4;
    const uint32_t blo = prmt(kT0, kT1, w & 0x7777u) | (prmt(ws, w, 0xD9C8u) & 0x80808080u);
    const uint32_t bhi = prmt(kT0, kT1, (w >> 16) & 0x7777u) | (prmt(ws, w, 0xFBEAu) & 0x80808080u);
    const uint32_t h[4] = {prmt(blo, 0u, 0x1404u), prmt(blo, 0u, 0x3424u), prmt(bhi, 0u, 0x1404u),
                           prmt(bhi, 0u, 0x3424u)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&h[i]), s2h);
        o[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
}

template <int BN>
struct F4Cfg {
    static constexpr bool kNarrow = BN <= 32;
    static constexpr int kW = 128 * 64;                     // codes: 128 rows x 128 K
    static constexpr int kBBox = BN * 128;                  // one f16 box: BN rows x 64 K
    static constexpr int kStage = kW + 2 * kBBox;           // a multiple of 1024
    static_assert(kStage % 1024 == 0, "stage alignment");
    // ring stages; 16-row tiles run two CTAs per SM (each with half the ring): the single MMA
    // lane is then shared by fewer bytes per cycle (measured: decode +29 %)
    static constexpr int kRS = kNarrow ? (BN <= 16 ? 8 : 12) : 4;
    static constexpr int kCtasPerSm = BN <= 16 ? 2 : 1;
    static constexpr int kS = kNarrow ? 2 : 4;              // TMEM A stages (64 columns each)
    static constexpr int kColA = 2 * BN;                    // TMEM: two accumulators | A stages
    static constexpr int kTmemNeed = kColA + kS * 64;
    static constexpr int kTmemCols = kTmemNeed <= 256 ? 256 : 512;
    static_assert(kTmemNeed <= 512, "TMEM budget");
    static constexpr int kXStride = (BN < 32 ? BN : 32) + 1;
    static constexpr int kOffX = kRS * kStage;
    static constexpr int kOffPre = kOffX + 64 * kXStride * 4;
    static constexpr int kOffSoff = kOffPre + 1025 * 4;
    static constexpr int kOffSr = kOffSoff + 1025 * 4;
    static constexpr int kOffBar = ((kOffSr + 2 * BN * 4 + 7) / 8) * 8;
    static constexpr int kNumBars = 2 * kRS + 2 * kS + 4;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static constexpr int kThreads = 320;
    static constexpr int kWarpWiden = 4, kWarpTma = 8, kWarpMma = 9;
};

template <int BN, bool kSwiGLU, bool kGather>
__global__ void __launch_bounds__(F4Cfg<BN>::kThreads, F4Cfg<BN>::kCtasPerSm)
    k_gemm_nvfp4(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                 const __grid_constant__ CUtensorMap tm_act, const F4GemmArgs f) {
    pdl_enter();
    using C = F4Cfg<BN>;
    const W8GemmArgs& a = f.b;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = sm;
    float* sX = reinterpret_cast<float*>(sm + C::kOffX);
    int* pre = reinterpret_cast<int*>(sm + C::kOffPre);
    int* soff = reinterpret_cast<int*>(sm + C::kOffSoff);
    float* sSr = reinterpret_cast<float*>(sm + C::kOffSr);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* full = bar;                  // stage filled: TMA bytes -> widening + MMA
    uint64_t* empty = full + C::kRS;       // stage consumed: MMA commit -> TMA
    uint64_t* a_ready = empty + C::kRS;    // A stage written: widening warps -> MMA
    uint64_t* a_free = a_ready + C::kS;    // A stage read: MMA commit -> widening warps
    uint64_t* t_full = a_free + C::kS;     // accumulator done: MMA commit -> epilogue
    uint64_t* t_empty = t_full + 2;        // accumulator drained: epilogue warps -> MMA
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int steps = a.K / 128;
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    const int row_tiles = row_tile_prefix(a.offsets, a.E, BN, pre, soff, f.slot_of, f.slot_want);
    const int64_t n_tiles = (int64_t)row_tiles * m_tiles;
    if ((int64_t)blockIdx.x >= n_tiles) return;

    if (tid == 0) {
        for (int i = 0; i < C::kRS; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
        for (int i = 0; i < C::kS; ++i) { tc::mbar_init(&a_ready[i], 4); tc::mbar_init(&a_free[i], 1); }
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
            const uint32_t b_bytes = kGather ? static_cast<uint32_t>(ngather) * 1024u : 2u * C::kBBox;
            bool stop = false;
            for (int s = 0; s < steps; ++s, r.next()) {
                uint8_t* st = ring + r.idx * C::kStage;
                int ok = 1;
                if (lane == 0) {
                    ok = ws::wait(&empty[r.idx], r.phase ^ 1u, abort);
                    if (ok) {
                        tc::mbar_arrive_expect_tx(&full[r.idx], C::kW + b_bytes);
                        const int wb = weight_slab(f.slot_of, e);
                        if (kSwiGLU) {
                            const int y = wb * a.R0 + mt * 64;
                            ws::tma_load_2d(st, &tm_w0, s * 64, y, &full[r.idx]);
                            ws::tma_load_2d(st + 64 * 64, &tm_w1, s * 64, y, &full[r.idx]);
                        } else {
                            ws::tma_load_2d(st, &tm_w0, s * 64, wb * a.R0 + mt * 128, &full[r.idx]);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) { stop = true; break; }
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {          // the two 64-wide halves of the K step
                    uint8_t* bst = st + C::kW + hb * C::kBBox;
                    const int xb = (s * 128 + hb * 64) * 2;   // byte column of the f16 rows
                    if (kGather) {
                        if (lane < ngather)
                            ws::tma_gather4(bst + lane * 512, &tm_act, xb, tok[0], tok[1], tok[2], tok[3],
                                            &full[r.idx]);
                    } else if (lane == 0) {
                        ws::tma_load_2d(bst, &tm_act, xb, row0, &full[r.idx]);
                    }
                }
            }
            if (stop) break;
        }
    } else if (warp == C::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint64_t bd0 = tc::sdesc_sw128(tc::smem_u32(ring + C::kW));
            ws::Ring<C::kRS> r;
            ws::Ring<C::kS> ra;
            uint32_t tcount = 0;
            int last = -1;
            uint32_t last_phase = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x, ++tcount) {
                const int tb = tcount & 1;
                const int rt = static_cast<int>(tile / m_tiles);
                const int e = expert_of_tile(pre, a.E, rt);
                const int nrows = min(BN, soff[e + 1] - soff[e] - (rt - pre[e]) * BN);
                const int n_mma = min(BN, (nrows + 15) & ~15);
                const uint32_t idesc = tc::idesc_f16_f32(128, n_mma);
                if (!ws::wait(&t_empty[tb], ((tcount >> 1) & 1) ^ 1u, abort)) break;
                tc::tc_fence_after();
                const uint32_t d = tmem + tb * BN;
                bool stop = false;
                for (int s = 0; s < steps; ++s, r.next(), ra.next()) {
                    if (!ws::wait(&full[r.idx], r.phase, abort)) { stop = true; break; }
                    if (!ws::wait(&a_ready[ra.idx], ra.phase, abort)) { stop = true; break; }
                    tc::tc_fence_after();
                    const uint64_t so = static_cast<uint64_t>(r.idx * (C::kStage >> 4));
                    const uint32_t a_col = tmem + C::kColA + ra.idx * 64;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {      // K = 16 each: box kk / 4, 32 bytes apart
                        const uint64_t bd = bd0 + so + static_cast<uint64_t>((kk >> 2) * (C::kBBox >> 4) + 2 * (kk & 3));
                        tc::mma_f16_ta(d, a_col + kk * 8, bd, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&empty[r.idx]);
                    tc::mma_commit(&a_free[ra.idx]);
                    last = ra.idx;
                    last_phase = ra.phase;
                }
                if (stop) break;
                tc::mma_commit(&t_full[tb]);
            }
            if (last >= 0) ws::wait(&a_free[last], last_phase, abort);
        }
    } else if (warp >= C::kWarpWiden) {
        // ------------------------------------------------------------ widening warps
        // A row per thread; the 64 code bytes of a K step land with the 64-byte TMA swizzle
        // (16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3)), so a warp's 32 rows read
        // distinct banks.  The row's block scales are read from global memory one step ahead.
        const int quad = warp - C::kWarpWiden;
        const int row = quad * 32 + lane;
        const int swz = (row >> 1) & 3;
        const uint32_t t_dst = tmem + (static_cast<uint32_t>(quad * 32) << 16) + C::kColA;
        const int kb = a.K / 16;                           // block scales per weight row
        ws::Ring<C::kRS> r;
        ws::Ring<C::kS> ra;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const int rt = static_cast<int>(tile / m_tiles), mt = static_cast<int>(tile % m_tiles);
            const int wb = weight_slab(f.slot_of, expert_of_tile(pre, a.E, rt));
            const uint8_t* srow = kSwiGLU
                ? (row < 64 ? f.bs0 : f.bs1) + ((int64_t)wb * a.R0 + mt * 64 + (row & 63)) * kb
                : f.bs0 + ((int64_t)wb * a.R0 + mt * 128 + row) * kb;
            uint2 sc_next = __ldg(reinterpret_cast<const uint2*>(srow));
            for (int s = 0; s < steps; ++s, r.next(), ra.next()) {
                const uint2 sc = sc_next;
                if (s + 1 < steps) sc_next = __ldg(reinterpret_cast<const uint2*>(srow) + s + 1);
                ws::wait(&full[r.idx], r.phase, abort);
                const uint8_t* raw = ring + r.idx * C::kStage + row * 64;
                uint4 cw[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) cw[p] = *reinterpret_cast<const uint4*>(raw + ((p ^ swz) << 4));
                ws::wait(&a_free[ra.idx], ra.phase ^ 1u, abort);
                tc::tc_fence_after();
                // block scales -> f16 (exact): eight per step, two per conversion
                __half2 s2h[8];
                const uint32_t sw[2] = {sc.x, sc.y};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                        static_cast<__nv_fp8x2_storage_t>((sw[q >> 1] >> (16 * (q & 1))) & 0xFFFFu), __NV_E4M3);
                    const __half2 h2 = *reinterpret_cast<const __half2*>(&hr);
                    s2h[2 * q] = __low2half2(h2);
                    s2h[2 * q + 1] = __high2half2(h2);
                }
#pragma unroll
                for (int half = 0; half < 2; ++half) {    // 64 K (32 TMEM columns) per store
                    uint32_t o[32];
#pragma unroll
                    for (int p2 = 0; p2 < 2; ++p2) {
                        const uint4 c = cw[2 * half + p2];
                        const uint32_t ww[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {      // word q: codes 8q..8q+7 of this chunk
                            const int blk = (2 * half + p2) * 2 + (q >> 1);   // block of 16 in the step
                            uint32_t v[4];
                            e2m1x8_to_f16(ww[q], s2h[blk], v);
#pragma unroll
                            for (int i = 0; i < 4; ++i) o[16 * p2 + 4 * q + i] = v[i];
                        }
                    }
                    tc::tmem_st32(t_dst + ra.idx * 64 + half * 32, o);
                }
                tc::tmem_wait_st();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&a_ready[ra.idx]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue warps 0-3
        w8_epilogue_warps<BN, kSwiGLU, kGather>(
            a, n_tiles, m_tiles, pre, soff, sSr, sX, tmem, t_full, t_empty, abort,
            [&](int e, int, int lrow) {
                const int wb = weight_slab(f.slot_of, e);
                return kSwiGLU ? (lrow < 64 ? f.s2_0[wb] : f.s2_1[wb]) : f.s2_0[wb];
            });
    }

    __syncwarp();
    __syncthreads();
    if (*abort && tid == 0) atomicOr(&g_device_status, kStatusTimeout);
    if (warp == C::kWarpMma) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---- host side --------------------------------------------------------------------------------

template <int BN, bool kSwiGLU, bool kGather>
int launch_gemm_nvfp4_inst(const F4GemmArgs& f, const void* act_f16, const void* w0, const void* w1,
                           int64_t max_row_tiles, cudaStream_t stream) {
    using C = F4Cfg<BN>;
    const W8GemmArgs& a = f.b;
    static int sms_cache[16] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    auto kern = k_gemm_nvfp4<BN, kSwiGLU, kGather>;
    if (sms_cache[dev & 15] == 0) {
        int sms = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kAlloc) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        sms_cache[dev & 15] = sms;
    }
    CUtensorMap m0, m1, mact;
    const int rows_per_load = kSwiGLU ? 64 : 128;
    if (!make_map_u8(&m0, w0, a.K / 2, (uint64_t)a.E * a.R0, 64, rows_per_load, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_u8(&m1, kSwiGLU ? w1 : w0, a.K / 2, (uint64_t)a.E * a.R0, 64, rows_per_load,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_u8(&mact, act_f16, (uint64_t)a.K * 2, kGather ? (uint64_t)a.T : (uint64_t)a.P, 128,
                     kGather ? 1 : BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return MOE_ERR_CUDA;
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    const int64_t grid = std::max<int64_t>(
        1, std::min<int64_t>(max_row_tiles * m_tiles, (int64_t)sms_cache[dev & 15] * C::kCtasPerSm));
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(C::kThreads), C::kAlloc, stream, m0, m1, mact,
                      f);
}

template <bool kSwiGLU>
int launch_gemm_nvfp4(const F4GemmArgs& f, const void* act_f16, const void* w0, const void* w1,
                      cudaStream_t stream) {
    const W8GemmArgs& a = f.b;
    const int BN = tc_tile_rows(a.P, a.E);
    const int64_t max_row_tiles = ((int64_t)a.P + BN - 1) / BN + a.E;
    switch (BN) {
        case 16: return launch_gemm_nvfp4_inst<16, kSwiGLU, kSwiGLU>(f, act_f16, w0, w1, max_row_tiles, stream);
        case 32: return launch_gemm_nvfp4_inst<32, kSwiGLU, kSwiGLU>(f, act_f16, w0, w1, max_row_tiles, stream);
        default: return launch_gemm_nvfp4_inst<128, kSwiGLU, false>(f, act_f16, w0, w1, max_row_tiles, stream);
    }
}

}  // namespace moe
