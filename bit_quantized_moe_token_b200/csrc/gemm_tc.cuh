// gemm_tc.cuh — S4/S6: grouped W4A8 GEMM on the 5th-generation tensor cores (tcgen05).
//
// Layout ("swap AB"): the MMA's M side is 128 weight rows (output features), its N side is
// BN routed token rows of one expert segment, K runs over the input features.  Per K-group
// of 128 the packed INT4 codes are widened exactly to E4M3 into shared memory (every value
// in -8..7 is an E4M3 number), four 128 x BN x 32 tcgen05.mma steps accumulate the group's
// partial sum in TMEM, and the epilogue threads promote it into an fp32 register
// accumulator with the group's bf16 scale:  acc[n,t] += s[n,g] * partial_g[n,t].  The token
// (row) scale is applied last.  TMEM partials and shared-memory stages are double-buffered,
// so the widening of group g+1 and the promotion of group g-1 overlap the MMAs of group g.
//
// Two widenings:
//  * signed: byte = E4M3(code) through two byte-permute table lookups (12 integer ops per
//    8 codes); promotion is one FMA per element.  Used for wide token tiles (prefill).
//  * unsigned: byte = the nibble itself (code + 8).  Bytes 0x00..0x0F are the E4M3 values
//    0..15 x 2^-9 (subnormals and the first normal binade are one equally spaced ladder), so
//    the MMA computes 2^-9 * sum q*(code+8) with 2-5 ops per 8 codes, and the promotion
//    removes the offset with the precomputed per-(row, group) sum of the activations:
//        acc += (512 s) * (partial - c),   c = (sum_{k in g} q_k) / 64.
//    Used for narrow token tiles (decode), where the widening dominates the issue slots.
//
// The forward's gate/up instance fuses SwiGLU: a 128-row M tile holds 64 gate rows and the
// same 64 up rows; the epilogue writes h = silu(G) * U in fp32 and folds max|h| of each token
// row into a global per-row maximum (for the requantization that follows).
#pragma once
#include "common.cuh"
#include "tc_ptx.cuh"

namespace moe {

struct TcGemmArgs {
    const uint8_t* act;     // [P, K] E4M3 activations, expert-sorted rows
    const float* s_row;     // [P] per-row activation scale
    const float* csum;      // [P, K/128] per-row group sums / 64 (unsigned widening only)
    const int32_t* w0;      // [E, R0, K/8] packed codes (gate, or down)
    const uint16_t* s0;     // [E, R0, K/128] bf16 scales
    const int32_t* w1;      // up projection (SwiGLU instance only)
    const uint16_t* s1;
    const int32_t* offsets; // [E + 1] segment offsets
    int E, R0, K;
    float* out;             // SwiGLU: h [P, R0]; plain: Y [P, ldo]
    int ldo;
    unsigned* amax;         // SwiGLU: [P] float bits of max|h| per row
};

// ---- widening ------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Eight codes of one packed word -> eight E4M3 bytes in K order (lo = codes 0..3).
template <bool kUnsigned>
__device__ __forceinline__ uint2 widen8(uint32_t w) {
    if constexpr (kUnsigned) {
        const uint32_t e = w & 0x0F0F0F0Fu;          // nibbles 0, 2, 4, 6
        const uint32_t o = (w >> 4) & 0x0F0F0F0Fu;   // nibbles 1, 3, 5, 7
        return make_uint2(prmt(e, o, 0x5140u), prmt(e, o, 0x7362u));
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

// Per-expert prefix of row tiles (ceil(len / BN)) into shared `pre[0..E]`; returns the total.
__device__ int row_tile_prefix(const int32_t* __restrict__ offsets, int E, int BN, int* pre) {
    __shared__ int s_total;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int run = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int n = (e < E) ? (offsets[e + 1] - offsets[e] + BN - 1) / BN : 0;
            int inc = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (e < E) pre[e] = run + inc - n;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) { pre[E] = run; s_total = run; }
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

constexpr int kTcThreads = 128;

template <int BN>
struct TcSmem {
    static constexpr int kA = 128 * 128;          // one widened A stage (bytes)
    static constexpr int kB = BN * 128;           // one activation stage
    static constexpr int kUsStride = BN + 1;      // SwiGLU exchange row stride (floats)
    static constexpr int kOffA = 0;
    static constexpr int kOffB = 2 * kA;
    static constexpr int kOffC = kOffB + ((2 * kB + 1023) / 1024) * 1024;
    static constexpr int kOffUs = kOffC + 3 * BN * 4;
    static constexpr int kOffPre = kOffUs + 64 * kUsStride * 4;   // (E + 1) ints, E <= 1024
    static constexpr int kOffBar = ((kOffPre + 1025 * 4 + 7) / 8) * 8;
    static constexpr int kOffSlot = kOffBar + 16;
    static constexpr int kBytes = kOffSlot + 16;
    static constexpr int kAlloc = kBytes + 1024;                  // slack for 1024-B alignment
    static constexpr int kTmemCols = (2 * BN < 32) ? 32 : 2 * BN;
};

template <int BN, bool kUnsigned, bool kSwiGLU>
__global__ void __launch_bounds__(kTcThreads) k_gemm_w4a8_tc(const TcGemmArgs a) {
    using L = TcSmem<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = sm + L::kOffA;
    uint8_t* sB = sm + L::kOffB;
    float* sC = reinterpret_cast<float*>(sm + L::kOffC);
    float* sUs = reinterpret_cast<float*>(sm + L::kOffUs);
    int* pre = reinterpret_cast<int*>(sm + L::kOffPre);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kOffSlot);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.K / kGroup;
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    const int row_tiles = row_tile_prefix(a.offsets, a.E, BN, pre);
    const int64_t n_tiles = (int64_t)row_tiles * m_tiles;
    if ((int64_t)blockIdx.x >= n_tiles) return;

    if (warp == 0) {
        tc::tmem_alloc(tslot, L::kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(&bars[0], 1);
        tc::mbar_init(&bars[1], 1);
        tc::fence_mbar_init();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
    constexpr uint32_t idesc = tc::idesc_e4m3_f32(128, BN);
    bool ok = true;
    uint32_t it = 0;   // groups processed by this CTA (stage / phase counter)

    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int rt = static_cast<int>(tile / m_tiles);
        const int mt = static_cast<int>(tile % m_tiles);
        const int e = expert_of_tile(pre, a.E, rt);
        const int seg0 = a.offsets[e];
        const int r0 = (rt - pre[e]) * BN;
        const int nrows = min(BN, a.offsets[e + 1] - seg0 - r0);
        const int64_t row0 = seg0 + r0;

        // A row `tid` of this tile: weight row of w0 (or of w1 for the upper half, SwiGLU)
        const int32_t* wsrc;
        const uint16_t* ssrc;
        if (kSwiGLU) {
            const int n = mt * 64 + (tid & 63);
            const int32_t* W = tid < 64 ? a.w0 : a.w1;
            const uint16_t* S = tid < 64 ? a.s0 : a.s1;
            wsrc = W + ((int64_t)e * a.R0 + n) * (a.K / 8);
            ssrc = S + ((int64_t)e * a.R0 + n) * G;
        } else {
            const int m = mt * 128 + tid;
            wsrc = a.w0 + ((int64_t)e * a.R0 + m) * (a.K / 8);
            ssrc = a.s0 + ((int64_t)e * a.R0 + m) * G;
        }
        const uint4* wv = reinterpret_cast<const uint4*>(wsrc);

        float acc[BN];
#pragma unroll
        for (int j = 0; j < BN; ++j) acc[j] = 0.0f;

        uint4 wnext[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) wnext[q] = __ldg(wv + q);

        auto promote = [&](int g, uint32_t itg) {
            const int s = itg & 1;
            if (ok && !tc::mbar_wait(&bars[s], (itg >> 1) & 1)) ok = false;
            tc::tc_fence_after();
            float sc = bf16_bits_to_f32(__ldg(ssrc + g));
            if (kUnsigned) sc *= 512.0f;
            const float* cg = sC + (itg % 3) * BN;
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += (BN >= 32 ? 32 : 16)) {
                if constexpr (BN >= 32) {
                    uint32_t v[32];
                    tc::tmem_ld32(tmem + t_lane + s * BN + c0, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float p = __uint_as_float(v[j]);
                        acc[c0 + j] = kUnsigned ? fmaf(sc, p - cg[c0 + j], acc[c0 + j])
                                                : fmaf(sc, p, acc[c0 + j]);
                    }
                } else {
                    uint32_t v[16];
                    tc::tmem_ld16(tmem + t_lane + s * BN + c0, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float p = __uint_as_float(v[j]);
                        acc[c0 + j] = kUnsigned ? fmaf(sc, p - cg[c0 + j], acc[c0 + j])
                                                : fmaf(sc, p, acc[c0 + j]);
                    }
                }
            }
            tc::tc_fence_before();
        };

        for (int g = 0; g < G; ++g, ++it) {
            const int s = it & 1;
            // ---- stage s: widened weights, activations, group sums ----
            uint8_t* a_st = sA + s * L::kA;
            uint4 wcur[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) wcur[q] = wnext[q];
            if (g + 1 < G) {
#pragma unroll
                for (int q = 0; q < 4; ++q) wnext[q] = __ldg(wv + (g + 1) * 4 + q);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint2 w0 = widen8<kUnsigned>(wcur[q].x);
                const uint2 w1 = widen8<kUnsigned>(wcur[q].y);
                const uint2 w2 = widen8<kUnsigned>(wcur[q].z);
                const uint2 w3 = widen8<kUnsigned>(wcur[q].w);
                // words 4q..4q+3 = K bytes 32q..32q+31 = chunks 2q, 2q+1
                *reinterpret_cast<uint4*>(a_st + sw128_off(tid, 2 * q)) = make_uint4(w0.x, w0.y, w1.x, w1.y);
                *reinterpret_cast<uint4*>(a_st + sw128_off(tid, 2 * q + 1)) = make_uint4(w2.x, w2.y, w3.x, w3.y);
            }
            uint8_t* b_st = sB + s * L::kB;
            for (int c = tid; c < BN * 8; c += kTcThreads) {
                const int r = c >> 3, j = c & 7;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (r < nrows)
                    v = __ldg(reinterpret_cast<const uint4*>(a.act + (row0 + r) * a.K + g * kGroup) + j);
                *reinterpret_cast<uint4*>(b_st + sw128_off(r, j)) = v;
            }
            if (kUnsigned && tid < BN)
                sC[(it % 3) * BN + tid] = (tid < nrows) ? a.csum[(row0 + tid) * G + g] : 0.0f;
            tc::fence_proxy_async_smem();
            __syncthreads();
            // ---- MMAs of group g into TMEM buffer s ----
            if (tid == 0) {
                tc::tc_fence_after();
                const uint32_t a_addr = tc::smem_u32(a_st), b_addr = tc::smem_u32(b_st);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_e4m3(tmem + s * BN, tc::sdesc_sw128(a_addr + kk * 32),
                                 tc::sdesc_sw128(b_addr + kk * 32), idesc, kk > 0 ? 1u : 0u);
                tc::mma_commit(&bars[s]);
            }
            // ---- promote group g-1 while the tensor core runs group g ----
            if (g > 0) promote(g - 1, it - 1);
        }
        promote(G - 1, it - 1);
        ok = __syncthreads_and(ok) != 0;   // uniform across the CTA before any further barrier
        if (!ok) break;

        // ---- epilogue (static indices keep acc[] in registers) ----
        if constexpr (kSwiGLU) {
            if (tid >= 64) {
#pragma unroll
                for (int j = 0; j < BN; ++j) sUs[(tid - 64) * L::kUsStride + j] = acc[j];
            }
            __syncthreads();
            if (tid < 64) {
                const int n = mt * 64 + tid;
#pragma unroll
                for (int j = 0; j < BN; ++j) {
                    if (j < nrows) {   // uniform across the CTA
                        const float sr = a.s_row[row0 + j];
                        const float h = silu(acc[j] * sr) * (sUs[tid * L::kUsStride + j] * sr);
                        a.out[(row0 + j) * a.ldo + n] = h;
                        const float m = warp_max(fabsf(h));
                        if (lane == 0) atomicMax(a.amax + row0 + j, __float_as_uint(m));
                    }
                }
            }
            __syncthreads();
        } else {
            const int m = mt * 128 + tid;
#pragma unroll
            for (int j = 0; j < BN; ++j)
                if (j < nrows) a.out[(row0 + j) * a.ldo + m] = acc[j] * a.s_row[row0 + j];
        }
    }
    if (!ok && tid == 0) atomicExch(&g_device_status, 1);
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, L::kTmemCols);
}

// Launch shape of one kernel instance on one device (set once; later calls only read it).
struct TcLaunchShape {
    int sms = 0, ctas_per_sm = 0;
};

template <int BN, bool kUnsigned, bool kSwiGLU>
int tc_launch_shape(TcLaunchShape* out) {
    static TcLaunchShape cache[16];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    TcLaunchShape& c = cache[dev & 15];
    if (c.sms == 0) {
        auto kern = k_gemm_w4a8_tc<BN, kUnsigned, kSwiGLU>;
        constexpr int smem = TcSmem<BN>::kAlloc;
        int sms = 0, occ = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kTcThreads, smem) != cudaSuccess)
            return MOE_ERR_CUDA;
        // TMEM: the resident CTAs of an SM share its 512 columns
        c.ctas_per_sm = std::max(1, std::min(occ, 512 / TcSmem<BN>::kTmemCols));
        c.sms = sms;
    }
    *out = c;
    return MOE_OK;
}

template <int BN, bool kUnsigned, bool kSwiGLU>
int launch_gemm_tc_inst(const TcGemmArgs& a, int64_t max_row_tiles, cudaStream_t stream) {
    TcLaunchShape shape;
    if (tc_launch_shape<BN, kUnsigned, kSwiGLU>(&shape) != MOE_OK) return MOE_ERR_CUDA;
    const int m_tiles = kSwiGLU ? a.R0 / 64 : a.R0 / 128;
    const int64_t max_tiles = max_row_tiles * m_tiles;
    const int64_t grid =
        std::max<int64_t>(1, std::min<int64_t>(max_tiles, (int64_t)shape.sms * shape.ctas_per_sm));
    k_gemm_w4a8_tc<BN, kUnsigned, kSwiGLU>
        <<<static_cast<unsigned>(grid), kTcThreads, TcSmem<BN>::kAlloc, stream>>>(a);
    return launch_status();
}

// Token-tile width for the expected rows per expert; narrow tiles use the unsigned widening.
inline int tc_tile_rows(int64_t P, int E) {
    const int64_t avg = (P + E - 1) / E;
    return avg <= 8 ? 16 : avg <= 24 ? 32 : avg <= 64 ? 64 : 128;
}
inline bool tc_unsigned(int BN) { return BN <= 32; }

template <bool kSwiGLU>
int launch_gemm_tc(const TcGemmArgs& a, int64_t P, cudaStream_t stream) {
    const int BN = tc_tile_rows(P, a.E);
    const int64_t max_row_tiles = (P + BN - 1) / BN + a.E;
    switch (BN) {
        case 16: return launch_gemm_tc_inst<16, true, kSwiGLU>(a, max_row_tiles, stream);
        case 32: return launch_gemm_tc_inst<32, true, kSwiGLU>(a, max_row_tiles, stream);
        case 64: return launch_gemm_tc_inst<64, false, kSwiGLU>(a, max_row_tiles, stream);
        default: return launch_gemm_tc_inst<128, false, kSwiGLU>(a, max_row_tiles, stream);
    }
}

}  // namespace moe
