// router.cuh — router logits x . wr^T over the bf16 router weight: the step upstream of S2.
//
// The router stays in its source precision ("Baekpica/Inkling-Small-Mixed-Quant-GGUF" card,
// "Precision differences": router tensors are native; "Inkling-512k-NVFP4-AQLM-hybrid" card,
// "Layout summary": the gate is copied verbatim), so the logits are a bf16 x bf16 product with
// fp32 accumulation and no bias.
//   T <= 16 (decode): one CTA per expert, its 8 warps splitting K; each thread reads one 16-byte
//     weight chunk per step and the tokens' matching chunks from L2, and a fixed-order shared-
//     memory reduction finishes every logit (deterministic, no workspace).
//   16 < T < 256: CTAs of 8 experts x 16 tokens, the tokens staged in shared memory, one warp
//     per expert.
//   large T: the bf16 tcgen05 GEMM of the shared experts (gemm_bf16_tc.cuh), plain instance,
//     with the router weight as its 128-row M tiles.
//
// Router + top-k (moe_router_topk): the two CUDA-core paths finish with S2 in the same kernel.
// Every CTA counts itself done on a device-scope counter of its token block after a fence; the
// CTA that completes the block ranks those tokens' logits (read back through L2) into the top-k
// ids and softmax gates, so the logits never make a second trip through a separate launch.  At
// decode (T <= 16) the CTAs of the first T experts also quantize one token each to FP8 (S1),
// so router, quantization and top-k are one launch.  The tensor-core path (T >= 256) writes the
// logits and runs the top-k kernel after it.
#pragma once
#include "common.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "gemm_bf16_tc.cuh"

namespace moe {

__device__ __forceinline__ void bf16x8_to_f32(uint4 v, float (&f)[8]) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        f[2 * q] = __uint_as_float(u[q] << 16);
        f[2 * q + 1] = __uint_as_float(u[q] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// x [T, H] and wr [E, H] as 16-byte chunks (HC = H / 8 per row); logits [T, E] fp32.
// Expert e's logits of all T <= kT tokens by one CTA of 256 threads; thread i takes chunks i,
// i + 256, ... of the expert's row.
template <int kT>
__device__ __forceinline__ void router_rows_cta(const uint4* __restrict__ x, const uint4* __restrict__ wr,
                                                int T, int HC, int E, int e, float* __restrict__ logits) {
    __shared__ float part[8][kT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[kT];
#pragma unroll
    for (int j = 0; j < kT; ++j) acc[j] = 0.0f;
    const uint4* wrow = wr + (int64_t)e * HC;
    for (int c = threadIdx.x; c < HC; c += blockDim.x) {
        float wf[8];
        bf16x8_to_f32(__ldg(wrow + c), wf);
#pragma unroll
        for (int j = 0; j < kT; ++j) {
            if (j < T) {
                float xf[8];
                bf16x8_to_f32(__ldg(x + (int64_t)j * HC + c), xf);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[j] = fmaf(xf[q], wf[q], acc[j]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kT; ++j) {
        const float s = warp_sum(acc[j]);
        if (lane == 0) part[warp][j] = s;
    }
    __syncthreads();
    if (threadIdx.x < T) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += part[w][threadIdx.x];
        logits[(int64_t)threadIdx.x * E + e] = s;
    }
}

template <int kT>
__global__ void __launch_bounds__(256) k_router_rows(const uint4* __restrict__ x,
                                                     const uint4* __restrict__ wr, int T, int HC,
                                                     int E, float* __restrict__ logits) {
    pdl_enter();
    router_rows_cta<kT>(x, wr, T, HC, E, blockIdx.x, logits);
}

// Counts this CTA done on `counter` (after its logits are stored) and returns, to every thread,
// whether it completed the count of `n` (the last CTA then resets the counter to zero).
__device__ __forceinline__ bool last_of(unsigned* counter, unsigned n) {
    __shared__ int s_last;
    __syncthreads();                                 // every thread's logits are stored
    if (threadIdx.x == 0) {
        __threadfence();                             // cumulative: publishes the CTA's stores
        s_last = atomicAdd(counter, 1u) == n - 1;
        if (s_last) *counter = 0u;                   // all n arrivals are in: ready for the next call
    }
    __syncthreads();
    if (s_last) __threadfence();                     // acquire side before reading the others' logits
    return s_last != 0;
}

// Decode front (T <= kT): the logits of expert blockIdx.x, S1 of token blockIdx.x when
// blockIdx.x < T and xq is given, and S2 of every token by the last CTA.
template <int kT, int EPL>
__global__ void __launch_bounds__(256) k_router_front(const uint4* __restrict__ x,
                                                      const uint4* __restrict__ wr, int T, int HC,
                                                      int E, int k, float* __restrict__ logits,
                                                      int32_t* __restrict__ ids, float* __restrict__ gates,
                                                      unsigned* __restrict__ counter,
                                                      uint8_t* __restrict__ xq, float* __restrict__ s_x,
                                                      float* __restrict__ qsum) {
    pdl_enter();
    __shared__ float red[32];
    router_rows_cta<kT>(x, wr, T, HC, E, blockIdx.x, logits);
    if (xq && (int)blockIdx.x < T)
        quant_token_cta(reinterpret_cast<const uint16_t*>(x), blockIdx.x, HC * 8, xq, s_x, qsum, red);
    if (!last_of(counter, gridDim.x)) return;
    const int warp = threadIdx.x >> 5;
    for (int t = warp; t < T; t += 8)
        topk_row<EPL, true>(logits + (int64_t)t * E, E, k, ids + (int64_t)t * k, gates + (int64_t)t * k,
                            threadIdx.x & 31);
}

// CTAs of 8 experts (one warp each) x kTB tokens (blockIdx.y), the tokens staged in shared memory.
// With kTopk, the last of the gridDim.x CTAs of token block blockIdx.y runs S2 for its tokens.
template <int kTB, bool kTopk = false, int EPL = 1>
__global__ void __launch_bounds__(256) k_router_gemv(const uint4* __restrict__ x,
                                                     const uint4* __restrict__ wr, int T, int HC,
                                                     int E, float* __restrict__ logits, int k = 0,
                                                     int32_t* __restrict__ ids = nullptr,
                                                     float* __restrict__ gates = nullptr,
                                                     unsigned* __restrict__ counters = nullptr) {
    pdl_enter();
    extern __shared__ uint4 sx[];                    // [kTB][HC]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + warp;
    {
        const int t0 = blockIdx.y * kTB;
        const int nt = min(kTB, T - t0);
        for (int i = threadIdx.x; i < nt * HC; i += blockDim.x) sx[i] = __ldg(x + (int64_t)t0 * HC + i);
        __syncthreads();
        if (e < E) {                                 // warp-uniform
            float acc[kTB];
#pragma unroll
            for (int j = 0; j < kTB; ++j) acc[j] = 0.0f;
            const uint4* wrow = wr + (int64_t)e * HC;
            for (int c = lane; c < HC; c += 32) {
                float wf[8];
                bf16x8_to_f32(__ldg(wrow + c), wf);
#pragma unroll
                for (int j = 0; j < kTB; ++j) {
                    if (j < nt) {
                        float xf[8];
                        bf16x8_to_f32(sx[j * HC + c], xf);
#pragma unroll
                        for (int q = 0; q < 8; ++q) acc[j] = fmaf(xf[q], wf[q], acc[j]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < kTB; ++j) {
                const float s = warp_sum(acc[j]);
                if (lane == 0 && j < nt) logits[(int64_t)(t0 + j) * E + e] = s;
            }
        }
        if constexpr (kTopk) {
            if (!last_of(counters + blockIdx.y, gridDim.x)) return;
            for (int j = warp; j < nt; j += 8) {
                const int64_t t = t0 + j;
                topk_row<EPL, true>(logits + t * E, E, k, ids + t * k, gates + t * k, lane);
            }
        }
    }
}

template <int kTB, bool kTopk = false, int EPL = 1>
int launch_router_gemv(const uint16_t* x, const uint16_t* wr, int64_t T, int H, int E, float* logits,
                       cudaStream_t stream, int k = 0, int32_t* ids = nullptr, float* gates = nullptr,
                       unsigned* counters = nullptr) {
    const size_t smem = static_cast<size_t>(kTB) * H * 2;
    auto kern = k_router_gemv<kTB, kTopk, EPL>;
    static int smem_set[16] = {0};                   // per device: the largest opt-in so far
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (smem > 48 * 1024 && static_cast<int>(smem) > smem_set[dev & 15]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        smem_set[dev & 15] = static_cast<int>(smem);
    }
    const dim3 grid(static_cast<unsigned>((E + 7) / 8), static_cast<unsigned>((T + kTB - 1) / kTB));
    return launch_pdl(kern, grid, dim3(256), smem, stream, reinterpret_cast<const uint4*>(x),
                      reinterpret_cast<const uint4*>(wr), static_cast<int>(T), H / 8, E, logits, k, ids, gates,
                      counters);
}

inline bool router_uses_tensor_cores(int64_t T, int H, int E) {
    return T >= 256 && E % 128 == 0 && H % 64 == 0;
}

// Counter words the fused router + top-k needs (zero on entry of the first call; every call
// leaves them zero).
inline int64_t router_counter_words(int64_t T) { return (T + 3) / 4 + 1; }

// Router logits + S2 (and, with xq non-null and T <= 16, S1) in as few launches as the path
// allows; *launches receives their number.  `counters` must hold router_counter_words(T) zero
// words (they are left zero).
inline int launch_router_topk(const uint16_t* x, const uint16_t* wr, int64_t T, int H, int E, int k,
                              float* logits, int32_t* ids, float* gates, unsigned* counters,
                              uint8_t* xq, float* s_x, float* qsum, cudaStream_t stream, int* launches) {
    const int epl = (E + 31) / 32;
    *launches = 0;
    if (router_uses_tensor_cores(T, H, E)) {
        Bf16GemmArgs a{E, static_cast<int>(T), H, H, logits, E, H};
        int st = launch_gemm_bf16_ws<false>(a, x, wr, nullptr, stream);
        if (st != MOE_OK) return st;
        *launches = 2;
        return launch_topk(logits, T, E, k, ids, gates, stream);
    }
    *launches = 1;
    const uint4* x4 = reinterpret_cast<const uint4*>(x);
    const uint4* w4 = reinterpret_cast<const uint4*>(wr);
    if (T <= 16) {
#define MOE_RF(N) launch_pdl(k_router_front<16, N>, dim3(static_cast<unsigned>(E)), dim3(256), 0, stream, x4, w4, \
                             static_cast<int>(T), H / 8, E, k, logits, ids, gates, counters, xq, s_x, qsum)
        if (epl <= 1) return MOE_RF(1);
        if (epl <= 2) return MOE_RF(2);
        if (epl <= 4) return MOE_RF(4);
        if (epl <= 8) return MOE_RF(8);
        if (epl <= 16) return MOE_RF(16);
        return MOE_RF(32);
#undef MOE_RF
    }
#define MOE_RG(TB, N) launch_router_gemv<TB, true, N>(x, wr, T, H, E, logits, stream, k, ids, gates, counters)
#define MOE_RG_E(TB) (epl <= 1 ? MOE_RG(TB, 1) : epl <= 2 ? MOE_RG(TB, 2) : epl <= 4 ? MOE_RG(TB, 4) \
                      : epl <= 8 ? MOE_RG(TB, 8) : epl <= 16 ? MOE_RG(TB, 16) : MOE_RG(TB, 32))
    return H <= 4096 ? MOE_RG_E(16) : MOE_RG_E(4);
#undef MOE_RG_E
#undef MOE_RG
}

inline int router_args_ok(int64_t T, int H, int E) {
    if (T < 0 || H <= 0 || E < 1) return MOE_ERR_INVALID_ARG;
    if (H % 8 != 0 || H > 16384 || E > 1024 || T > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

}  // namespace moe

extern "C" int moe_router_logits(const uint16_t* x_bf16, const uint16_t* wr_bf16, int64_t T, int H, int E,
                                 float* logits, moe_stream_t stream) {
    using namespace moe;
    const int st = router_args_ok(T, H, E);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !wr_bf16 || !logits) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(wr_bf16, 16) || !aligned(logits, 4)) return MOE_ERR_MISALIGNED;
    if (router_uses_tensor_cores(T, H, E)) {
        Bf16GemmArgs a{E, static_cast<int>(T), H, H, logits, E, H};
        return launch_gemm_bf16_ws<false>(a, x_bf16, wr_bf16, nullptr, stream);
    }
    if (T <= 16) {
        return launch_pdl(k_router_rows<16>, dim3(static_cast<unsigned>(E)), dim3(256), 0, stream,
                          reinterpret_cast<const uint4*>(x_bf16), reinterpret_cast<const uint4*>(wr_bf16),
                          static_cast<int>(T), H / 8, E, logits);
    }
    return H <= 4096 ? launch_router_gemv<16>(x_bf16, wr_bf16, T, H, E, logits, stream)
                     : launch_router_gemv<4>(x_bf16, wr_bf16, T, H, E, logits, stream);
}

extern "C" size_t moe_router_topk_workspace_bytes(int64_t T, int E, int k) {
    if (moe::router_args_ok(T, 8, E) != MOE_OK || moe::route_args_ok(T, E, k) != MOE_OK) return 0;
    return moe::align_up(static_cast<size_t>(moe::router_counter_words(T)) * 4, 256);
}

extern "C" int moe_router_topk(const uint16_t* x_bf16, const uint16_t* wr_bf16, int64_t T, int H, int E,
                               int k, float* logits, int32_t* topk_ids, float* topk_w, void* ws,
                               size_t ws_bytes, moe_stream_t stream) {
    using namespace moe;
    int st = router_args_ok(T, H, E);
    if (st != MOE_OK) return st;
    if ((st = route_args_ok(T, E, k)) != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !wr_bf16 || !logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < moe_router_topk_workspace_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
    if (!aligned(x_bf16, 16) || !aligned(wr_bf16, 16) || !aligned(logits, 4) || !aligned(topk_ids, 4) ||
        !aligned(topk_w, 4) || !aligned(ws, 256))
        return MOE_ERR_MISALIGNED;
    unsigned* cnt = static_cast<unsigned*>(ws);
    if (cudaMemsetAsync(cnt, 0, router_counter_words(T) * 4, stream) != cudaSuccess) return MOE_ERR_CUDA;
    int launches = 0;
    return launch_router_topk(x_bf16, wr_bf16, T, H, E, k, logits, topk_ids, topk_w, cnt, nullptr, nullptr,
                              nullptr, stream, &launches);
}