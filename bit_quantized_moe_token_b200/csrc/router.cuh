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
#pragma once
#include "common.cuh"
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
// One CTA per expert, T <= kT; thread i takes chunks i, i + 256, ... of the expert's row.
template <int kT>
__global__ void __launch_bounds__(256) k_router_rows(const uint4* __restrict__ x,
                                                     const uint4* __restrict__ wr, int T, int HC,
                                                     int E, float* __restrict__ logits) {
    __shared__ float part[8][kT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x;
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

// CTAs of 8 experts (one warp each) x kTB tokens (blockIdx.y), the tokens staged in shared memory.
template <int kTB>
__global__ void __launch_bounds__(256) k_router_gemv(const uint4* __restrict__ x,
                                                     const uint4* __restrict__ wr, int T, int HC,
                                                     int E, float* __restrict__ logits) {
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
    }
}

template <int kTB>
int launch_router_gemv(const uint16_t* x, const uint16_t* wr, int64_t T, int H, int E, float* logits,
                       cudaStream_t stream) {
    const size_t smem = static_cast<size_t>(kTB) * H * 2;
    auto kern = k_router_gemv<kTB>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>((E + 7) / 8), static_cast<unsigned>((T + kTB - 1) / kTB));
    kern<<<grid, 256, smem, stream>>>(
        reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(wr), static_cast<int>(T), H / 8, E,
        logits);
    return launch_status();
}

inline bool router_uses_tensor_cores(int64_t T, int H, int E) {
    return T >= 256 && E % 128 == 0 && H % 64 == 0;
}

}  // namespace moe

extern "C" int moe_router_logits(const uint16_t* x_bf16, const uint16_t* wr_bf16, int64_t T, int H, int E,
                                 float* logits, moe_stream_t stream) {
    using namespace moe;
    if (T < 0 || H <= 0 || E < 1) return MOE_ERR_INVALID_ARG;
    if (H % 8 != 0 || H > 16384 || E > 1024 || T > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !wr_bf16 || !logits) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(wr_bf16, 16) || !aligned(logits, 4)) return MOE_ERR_MISALIGNED;
    if (router_uses_tensor_cores(T, H, E)) {
        Bf16GemmArgs a{E, static_cast<int>(T), H, H, logits, E};
        return launch_gemm_bf16_ws<false>(a, x_bf16, wr_bf16, nullptr, 1, stream);
    }
    if (T <= 16) {
        k_router_rows<16><<<static_cast<unsigned>(E), 256, 0, stream>>>(
            reinterpret_cast<const uint4*>(x_bf16), reinterpret_cast<const uint4*>(wr_bf16),
            static_cast<int>(T), H / 8, E, logits);
        return launch_status();
    }
    return H <= 4096 ? launch_router_gemv<16>(x_bf16, wr_bf16, T, H, E, logits, stream)
                     : launch_router_gemv<4>(x_bf16, wr_bf16, T, H, E, logits, stream);
}
