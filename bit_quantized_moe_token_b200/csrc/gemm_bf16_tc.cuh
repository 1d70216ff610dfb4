// gemm_bf16_tc.cuh — S8: the always-on shared experts as bf16 GEMMs on tcgen05.
//
// The shared experts keep their bf16 weights (Inkling-Small card, section 1: shared-expert
// parameters stay BF16).  Their n_shared SwiGLU MLPs are summed, which is one MLP of width
// n_shared * Ns: the gate/up GEMM runs over the stacked [n_shared * Ns, H] weights, and the
// down GEMM reduces over (expert, n) with a 3-D tensor map over [n_shared, H, Ns].
//
// Same warp roles as gemm_ws.cuh: warp 4 streams 128 x 64 bf16 weight tiles and BN x 64 token
// tiles (both landing in the 128-byte swizzle the MMA reads) through a 4-stage ring, warp 5
// issues four tcgen05.mma.kind::f16 (bf16 in, fp32 accumulate) per 64-wide K chunk into one
// of two TMEM accumulators (2 x BN columns), and warps 0-3 drain a finished accumulator while
// the tensor core fills the other.  Swap AB again: MMA M = 128 weight rows, N = BN tokens.
//   SwiGLU instance: M tile = 64 gate rows + the same 64 up rows; the epilogue writes
//     a = silu(gate . x) * (up . x) as f16(a * 2^-8): the layer keeps this activation in fp32,
//     bf16 would move outputs by up to ~1 % (its 8-bit significand), f16 carries 11 bits, and
//     the 2^-8 prescale keeps |a| up to 2^24 inside its range (values below 2^-6 lose relative
//     precision as f16 subnormals, never more than 2^-17 absolute).
//   plain instance, kF16: the shared down projection as an f16 MMA over those activations and an
//     f16 copy of the bf16 down weights (every bf16 weight of magnitude 2^-14 .. 65504 is exact
//     in f16), Y[t, m] = 256 * acc in fp32; the weights of K index k are those of k mod Kw.
//   plain instance, bf16: Y[t, m] fp32 (not used by the layer).
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tc_pipe.cuh"

namespace moe {

struct Bf16GemmArgs {
    int M;       // output rows of one projection (SwiGLU: n_shared*Ns; plain: H)
    int T;       // tokens
    int K;       // reduction length of the activations (SwiGLU: H; plain: n_shared*Ns)
    int Ks;      // plain: K extent per shared expert (Ns); the 3-D weight map's inner dim
    void* out;   // SwiGLU: f16 [T, ldo] (a * 2^-8, ldo >= M); plain: fp32 [T, ldo]
    int ldo;
    int Kw;      // plain: K extent of the weights (n_shared*Ns); activation column k uses k mod Kw
};

namespace tc {
// Instruction descriptor: kind::f16 with A = B = BF16, D = F32, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
// The same with A = B = F16.
__host__ __device__ constexpr uint32_t idesc_h16_f32(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
}  // namespace tc

namespace ws {
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(tc::smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(tc::smem_u32(bar)),
          "r"(x), "r"(y), "r"(z)
        : "memory");
}
}  // namespace ws

template <int BN>
struct Bf16Cfg {
    static constexpr int kA = 128 * 128;                  // 128 rows x 64 bf16
    static constexpr int kB = BN * 128;
    static constexpr int kStage = kA + kB;                // multiple of 1024
    static constexpr int kRS = 4;
    static constexpr int kXStride = 33;                   // SwiGLU exchange: 64 x 32 (+1) floats
    static constexpr int kOffX = kRS * kStage;
    static constexpr int kOffBar = kOffX + 64 * kXStride * 4;
    static constexpr int kOffMisc = kOffBar + (2 * kRS + 4) * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kTmemCols = 2 * BN;
};

template <int BN, bool kSwiGLU, bool kF16 = false>
__global__ void __launch_bounds__(192, 1)
    k_gemm_bf16_ws(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                   const __grid_constant__ CUtensorMap tm_act, const Bf16GemmArgs a) {
    pdl_enter();
    using C = Bf16Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = sm;
    float* sX = reinterpret_cast<float*>(sm + C::kOffX);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
    uint64_t* full = bar;
    uint64_t* empty = bar + C::kRS;
    uint64_t* t_full = bar + 2 * C::kRS;
    uint64_t* t_empty = t_full + 2;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + C::kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m_tiles = kSwiGLU ? a.M / 64 : a.M / 128;
    const int n_tok_tiles = (a.T + BN - 1) / BN;
    const int64_t n_tiles = (int64_t)m_tiles * n_tok_tiles;
    const int chunks = a.K / 64;
    if ((int64_t)blockIdx.x >= n_tiles) return;

    if (tid == 0) {
        for (int i = 0; i < C::kRS; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&t_full[i], 1); tc::mbar_init(&t_empty[i], 128); }
        *abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 5) {
        tc::tmem_alloc(tslot, C::kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp == 4) {
        if (lane == 0) {
            ws::prefetch_map(&tm_w0);
            if (kSwiGLU) ws::prefetch_map(&tm_w1);
            ws::prefetch_map(&tm_act);
            uint32_t it = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x) {
                const int nt = static_cast<int>(tile / m_tiles), mt = static_cast<int>(tile % m_tiles);
                for (int c = 0; c < chunks; ++c, ++it) {
                    const int s = it % C::kRS;
                    if (!ws::wait(&empty[s], ((it / C::kRS) & 1) ^ 1, abort)) break;
                    uint8_t* st = ring + s * C::kStage;
                    tc::mbar_arrive_expect_tx(&full[s], C::kStage);
                    ws::tma_load_2d(st + C::kA, &tm_act, c * 64, nt * BN, &full[s]);
                    if (kSwiGLU) {
                        ws::tma_load_2d(st, &tm_w0, c * 64, mt * 64, &full[s]);
                        ws::tma_load_2d(st + 64 * 128, &tm_w1, c * 64, mt * 64, &full[s]);
                    } else {
                        const int k0 = (c * 64) % a.Kw;
                        ws::tma_load_3d(st, &tm_w0, k0 % a.Ks, mt * 128, k0 / a.Ks, &full[s]);
                    }
                }
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // the SwiGLU instance multiplies bf16 tokens and weights; the plain kF16 instance f16 ones
            constexpr uint32_t idesc = (!kSwiGLU && kF16) ? tc::idesc_h16_f32(128, BN) : tc::idesc_bf16_f32(128, BN);
            uint32_t it = 0, tcount = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort; tile += gridDim.x, ++tcount) {
                const int tb = tcount & 1;
                if (!ws::wait(&t_empty[tb], ((tcount >> 1) & 1) ^ 1, abort)) break;
                tc::tc_fence_after();
                const uint32_t d = tmem + tb * BN;
                for (int c = 0; c < chunks; ++c, ++it) {
                    const int s = it % C::kRS;
                    if (!ws::wait(&full[s], (it / C::kRS) & 1, abort)) break;
                    tc::tc_fence_after();
                    const uint32_t a_addr = tc::smem_u32(ring + s * C::kStage);
                    const uint32_t b_addr = a_addr + C::kA;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(d, tc::sdesc_sw128(a_addr + kk * 32), tc::sdesc_sw128(b_addr + kk * 32),
                                     idesc, (c > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&empty[s]);
                }
                tc::mma_commit(&t_full[tb]);
            }
            if (it > 0) ws::wait(&empty[(it - 1) % C::kRS], ((it - 1) / C::kRS) & 1, abort);
        }
    } else {
        const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
        uint32_t tcount = 0;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tcount) {
            const int nt = static_cast<int>(tile / m_tiles), mt = static_cast<int>(tile % m_tiles);
            const int tb = tcount & 1;
            const int n0 = nt * BN;
            ws::wait(&t_full[tb], (tcount >> 1) & 1, abort);
            tc::tc_fence_after();
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                tc::tmem_ld32(tmem + t_lane + tb * BN + c0, v);
                tc::tmem_wait_ld();
                if constexpr (kSwiGLU) {
                    if (tid >= 64) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) sX[(tid - 64) * C::kXStride + j] = __uint_as_float(v[j]);
                    }
                    ws::named_sync_math();
                    if (tid < 64) {
                        __half* out = static_cast<__half*>(a.out);
                        const int n = mt * 64 + tid;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int t = n0 + c0 + j;
                            if (t < a.T) {
                                const float h = silu(__uint_as_float(v[j])) * sX[tid * C::kXStride + j];
                                out[(int64_t)t * a.ldo + n] = __float2half_rn(h * 0.00390625f);   // h * 2^-8
                            }
                        }
                    }
                    ws::named_sync_math();
                } else {
                    float* out = static_cast<float*>(a.out);
                    const int m = mt * 128 + tid;
                    constexpr float kUnscale = kF16 ? 256.0f : 1.0f;   // undo the activations' 2^-8
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = n0 + c0 + j;
                        if (t < a.T) out[(int64_t)t * a.ldo + m] = __uint_as_float(v[j]) * kUnscale;
                    }
                }
            }
            tc::tc_fence_before();
            tc::mbar_arrive(&t_empty[tb]);
        }
    }

    __syncwarp();
    __syncthreads();
    if (*abort && tid == 0) atomicOr(&g_device_status, kStatusTimeout);
    if (warp == 5) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, C::kTmemCols);
    }
}

// bf16 -> f16, eight values per thread (round to nearest even; exact for magnitudes 2^-14 .. 65504).
__global__ void __launch_bounds__(256) k_bf16_to_f16(const uint4* __restrict__ in, uint4* __restrict__ out,
                                                     int64_t n8) {
    pdl_enter();
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const uint4 v = in[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __half2 h = __floats2half2_rn(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xFFFF0000u));
        o[q] = *reinterpret_cast<const uint32_t*>(&h);
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

// ---- host side -----------------------------------------------------------------------------

inline bool make_map_bf16_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                             uint32_t box_cols, uint32_t box_rows) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// [d2, d1, d0] bf16 tensor (d0 innermost) with a box of 1 x box1 x box0.
inline bool make_map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                             uint32_t box0, uint32_t box1) {
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    const cuuint32_t box[3] = {box0, box1, 1};
    return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// kF16: the plain instance as the shared down projection (f16 operands, output x 256); the router
// logits use the plain bf16 instance.
template <bool kSwiGLU, bool kF16 = false>
int launch_gemm_bf16_ws(const Bf16GemmArgs& a, const void* act, const void* w0, const void* w1,
                        cudaStream_t stream) {
    constexpr int BN = 256;
    using C = Bf16Cfg<BN>;
    // plain instance: the weights' K extent Kw is a whole number of Ks-wide slices, and the
    // activations' K a whole number of Kw
    if (!kSwiGLU && (a.Ks <= 0 || a.Kw <= 0 || a.Kw % a.Ks || a.K % a.Kw || a.Kw % 64))
        return MOE_ERR_INVALID_ARG;
    static int sms_cache[16] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    auto kern = k_gemm_bf16_ws<BN, kSwiGLU, kF16>;
    if (sms_cache[dev & 15] == 0) {
        int sms = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kAlloc) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        sms_cache[dev & 15] = sms;
    }
    CUtensorMap m0, m1, mact;
    bool ok;
    if (kSwiGLU) {
        ok = make_map_bf16_2d(&m0, w0, a.K, a.M, 64, 64) && make_map_bf16_2d(&m1, w1, a.K, a.M, 64, 64);
    } else {
        ok = make_map_bf16_3d(&m0, w0, a.Ks, a.M, a.Kw / a.Ks, 64, 128);
        m1 = m0;
    }
    ok = ok && make_map_bf16_2d(&mact, act, a.K, a.T, 64, BN);
    if (!ok) return MOE_ERR_CUDA;
    const int m_tiles = kSwiGLU ? a.M / 64 : a.M / 128;
    const int64_t tiles = (int64_t)m_tiles * ((a.T + BN - 1) / BN);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(tiles, sms_cache[dev & 15]));
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(192), C::kAlloc, stream, m0, m1, mact, a);
}

}  // namespace moe
