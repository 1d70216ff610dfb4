// gemm_simple.cuh — CUDA-core bf16 GEMM (shared experts, S8): a plain 64x64 smem-tiled
// kernel with fp32 accumulation.
#pragma once
#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------------------------------
// C[M, Nc] (+)= A[M, K] * B[Nc, K]^T with B bf16 and A bf16 or fp32, fp32 accumulate.
// 64x64 tile, 256 threads, 4x4 outputs per thread.  Used for the shared experts.
// ------------------------------------------------------------------------------------------
template <typename TA>
__device__ __forceinline__ float load_a(const TA* p);
template <>
__device__ __forceinline__ float load_a<uint16_t>(const uint16_t* p) { return bf16_bits_to_f32(*p); }
template <>
__device__ __forceinline__ float load_a<float>(const float* p) { return *p; }

template <typename TA>
__global__ void __launch_bounds__(256) k_gemm_bf16_simple(const TA* __restrict__ A,
                                                          const uint16_t* __restrict__ B, int M,
                                                          int Nc, int K, float* __restrict__ C,
                                                          int ldc, int accumulate) {
    __shared__ float As[16][64 + 1];
    __shared__ float Bs[16][64 + 1];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int i = threadIdx.x; i < 16 * 64; i += 256) {
            const int kk = i & 15, rr = i >> 4;
            const int m = m0 + rr, n = n0 + rr;
            As[kk][rr] = (m < M) ? load_a<TA>(A + (int64_t)m * K + k0 + kk) : 0.0f;
            Bs[kk][rr] = (n < Nc) ? bf16_bits_to_f32(B[(int64_t)n * K + k0 + kk]) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
            if (m < M && n < Nc) {
                float* c = C + (int64_t)m * ldc + n;
                *c = accumulate ? *c + acc[i][j] : acc[i][j];
            }
        }
}

template <typename TA>
inline int launch_gemm_bf16_simple(const TA* A, const uint16_t* B, int M, int Nc, int K, float* C,
                                   int ldc, bool accumulate, cudaStream_t stream) {
    dim3 grid((Nc + 63) / 64, (M + 63) / 64);
    k_gemm_bf16_simple<TA><<<grid, 256, 0, stream>>>(A, B, M, Nc, K, C, ldc, accumulate ? 1 : 0);
    return launch_status();
}

}  // namespace moe
