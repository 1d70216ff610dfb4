// gemm_simple.cuh — CUDA-core grouped W4A8 GEMM and bf16 GEMM.
//
// These are the plain, straightforward versions of S4/S6 (and S8): one output element per
// thread and row, weights unpacked in registers, activations staged one K-group at a time in
// shared memory.  They define the arithmetic the tensor-core kernels must reproduce and give
// a second, independent GPU route for cross-checks in tests.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kSimpleRows = 8;    // activation rows per CTA
constexpr int kSimpleCols = 128;  // weight rows (outputs) per CTA = threads

// Map a linear row-tile index to (expert, first row of the tile) given per-expert segments.
// Warp 0 scans; returns false when the tile index is past the last tile.
__device__ bool find_row_tile(const int32_t* __restrict__ offsets, int E, int rows_per_tile,
                              int64_t tile, int* e_out, int* r0_out) {
    __shared__ int s_e, s_r0;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int64_t acc = 0;
        int found_e = -1, found_r0 = 0;
        for (int e0 = 0; e0 < E && found_e < 0; e0 += 32) {
            const int e = e0 + lane;
            int n = 0;
            if (e < E) {
                const int len = offsets[e + 1] - offsets[e];
                n = (len + rows_per_tile - 1) / rows_per_tile;
            }
            int inc = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            const int64_t lo = acc + inc - n, hi = acc + inc;
            const unsigned hit = __ballot_sync(0xffffffffu, tile >= lo && tile < hi);
            if (hit) {
                const int src = __ffs(hit) - 1;
                found_e = e0 + src;
                const int64_t lo_src = __shfl_sync(0xffffffffu, lo, src);
                found_r0 = static_cast<int>((tile - lo_src) * rows_per_tile);
            }
            acc += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) { s_e = found_e; s_r0 = found_r0; }
    }
    __syncthreads();
    *e_out = s_e;
    *r0_out = s_r0;
    return s_e >= 0;
}

// Out[r, n] = s_row[r] * sum_g scale[e,n,g] * sum_{k in g} dec(A[r,k]) * code[e,n,k]
//   A      [P, K]  E4M3, rows in expert-sorted order (segment e = rows offsets[e]..offsets[e+1])
//   W      [E, R, K/8] packed int4;  S [E, R, K/128] bf16
//   Out    [P, ldo] fp32 (column block starting at out_col)
__global__ void __launch_bounds__(kSimpleCols) k_gemm_w4a8_simple(
    const uint8_t* __restrict__ A, const float* __restrict__ s_row,
    const int32_t* __restrict__ W, const uint16_t* __restrict__ S,
    const int32_t* __restrict__ offsets, int E, int R, int K, float* __restrict__ Out, int ldo) {
    __shared__ float As[kSimpleRows][kGroup];
    int e, r0;
    if (!find_row_tile(offsets, E, kSimpleRows, blockIdx.y, &e, &r0)) return;
    const int seg0 = offsets[e];
    const int nrows = min(kSimpleRows, offsets[e + 1] - seg0 - r0);
    const int n = blockIdx.x * kSimpleCols + threadIdx.x;
    const int G = K / kGroup;
    const uint4* wrow = reinterpret_cast<const uint4*>(W + ((int64_t)e * R + n) * (K / 8));
    const uint16_t* srow = S + ((int64_t)e * R + n) * G;
    float acc[kSimpleRows];
#pragma unroll
    for (int r = 0; r < kSimpleRows; ++r) acc[r] = 0.0f;
    for (int g = 0; g < G; ++g) {
        __syncthreads();
        {
            const int r = threadIdx.x >> 4, c = (threadIdx.x & 15) * 8;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (r < nrows) {
                const uint2 q = *reinterpret_cast<const uint2*>(
                    A + (int64_t)(seg0 + r0 + r) * K + g * kGroup + c);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    v[i] = e4m3_to_f32(static_cast<uint8_t>(((i < 4 ? q.x : q.y) >> (8 * (i & 3))) & 0xFF));
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) As[r][c + i] = v[i];
        }
        __syncthreads();
        float part[kSimpleRows];
#pragma unroll
        for (int r = 0; r < kSimpleRows; ++r) part[r] = 0.0f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const uint4 w4 = __ldg(wrow + g * 4 + q4);
            const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float c = static_cast<float>(static_cast<int>((ws[q] >> (4 * i)) & 15u) - 8);
                    const int kk = (q4 * 4 + q) * 8 + i;
#pragma unroll
                    for (int r = 0; r < kSimpleRows; ++r) part[r] = __fmaf_rn(As[r][kk], c, part[r]);
                }
            }
        }
        const float sc = bf16_bits_to_f32(__ldg(srow + g));
#pragma unroll
        for (int r = 0; r < kSimpleRows; ++r) acc[r] = __fadd_rn(acc[r], __fmul_rn(part[r], sc));
    }
    for (int r = 0; r < nrows; ++r) {
        const int64_t row = seg0 + r0 + r;
        Out[row * ldo + n] = __fmul_rn(acc[r], s_row[row]);
    }
}

inline int launch_gemm_w4a8_simple(const uint8_t* A, const float* s_row, const int32_t* W,
                                   const uint16_t* S, const int32_t* offsets, int E, int R, int K,
                                   int64_t P, float* Out, int ldo, cudaStream_t stream) {
    const int64_t max_tiles = (P + kSimpleRows - 1) / kSimpleRows + E;
    dim3 grid(R / kSimpleCols, static_cast<unsigned>(max_tiles));
    k_gemm_w4a8_simple<<<grid, kSimpleCols, 0, stream>>>(A, s_row, W, S, offsets, E, R, K, Out, ldo);
    return launch_status();
}

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
