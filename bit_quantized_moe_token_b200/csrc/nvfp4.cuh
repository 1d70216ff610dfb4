// nvfp4.cuh — NVFP4 expert weights: quantization from bf16, and the FP8 -> f16 activation copy
// the NVFP4 GEMM reads.
//
// Storage ("Inkling-512k-NVFP4-AQLM-hybrid" card, "On-disk tensor format" and "Dequant math"):
// two E2M1 codes per byte, the first weight of a pair in the low nibble; one E4M3 scale per
// block of 16 input weights; one fp32 scale2 per expert projection; W = LUT[code] * scale *
// scale2 with LUT = 0, .5, 1, 1.5, 2, 3, 4, 6 for codes 0..7 and the negatives for 8..15.
// Quantization (the page's slabs come from an NVFP4 base this library does not have):
//   scale2 = amax / (6 * 448) over the expert projection,
//   scale  = E4M3(amax_block / (6 * scale2))            (round to nearest even, saturating),
//   code   = nearest E2M1 value of w / (dec(scale) * scale2), ties to the even code, +-6 at
//            most, the sign kept; a zero scale gives codes 0.
#pragma once
#include "common.cuh"

namespace moe {

constexpr float kE2M1Max = 6.0f;

// Nearest E2M1 code of x: the decision points are the midpoints of the grid; at a midpoint the
// even code wins (0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2.0, 2.5 -> 2.0, 3.5 -> 4.0,
// 5 -> 4.0).
__device__ __forceinline__ uint32_t e2m1_code(float x) {
    const float a = fabsf(x);
    const uint32_t m = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
                     : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.0f ? 6u : 7u;
    return m | (signbit(x) ? 8u : 0u);
}

// amax over each expert projection (float bits, atomic max; the target words start at 0).
__global__ void __launch_bounds__(256) k_nvfp4_amax(const uint4* __restrict__ w, int64_t chunks_per_expert,
                                                     unsigned* __restrict__ amax_bits) {
    pdl_enter();
    const int64_t e = blockIdx.y;
    const uint4* we = w + e * chunks_per_expert;
    float a = 0.0f;
    for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < chunks_per_expert;
         c += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = __ldg(we + c);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            a = fmaxf(a, fabsf(__uint_as_float(u[q] << 16)));
            a = fmaxf(a, fabsf(__uint_as_float(u[q] & 0xFFFF0000u)));
        }
    }
    a = warp_max(a);
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + e, __float_as_uint(a));
}

// One thread per block of 16 weights: its E4M3 scale and eight code bytes.
__global__ void __launch_bounds__(256) k_nvfp4_quant(const uint4* __restrict__ w, int64_t blocks_per_expert,
                                                      int64_t experts, const unsigned* __restrict__ amax_bits,
                                                      uint2* __restrict__ codes, uint8_t* __restrict__ scales) {
    pdl_enter();
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= blocks_per_expert * experts) return;
    const int64_t e = i / blocks_per_expert;
    const float s2 = __fdiv_rn(__uint_as_float(amax_bits[e]), 6.0f * kFp8Max);
    const uint4 v0 = __ldg(w + 2 * i), v1 = __ldg(w + 2 * i + 1);
    const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float x[16];
    float ab = 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        x[2 * q] = __uint_as_float(u[q] << 16);
        x[2 * q + 1] = __uint_as_float(u[q] & 0xFFFF0000u);
        ab = fmaxf(ab, fmaxf(fabsf(x[2 * q]), fabsf(x[2 * q + 1])));
    }
    uint8_t sc = 0;
    if (s2 != 0.0f) sc = static_cast<uint8_t>(f32x2_to_e4m3x2(__fdiv_rn(ab, __fmul_rn(6.0f, s2)), 0.0f) & 0xFF);
    const float d = __fmul_rn(e4m3_to_f32(sc), s2);
    uint32_t out[2] = {0u, 0u};
    if (d != 0.0f) {
#pragma unroll
        for (int j = 0; j < 16; ++j) out[j >> 3] |= e2m1_code(__fdiv_rn(x[j], d)) << (4 * (j & 7));
    }
    codes[i] = make_uint2(out[0], out[1]);
    scales[i] = sc;
}

__global__ void k_nvfp4_finish(unsigned* __restrict__ s2_bits, int64_t experts) {
    pdl_enter();
    const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (e < experts) s2_bits[e] = __float_as_uint(__fdiv_rn(__uint_as_float(s2_bits[e]), 6.0f * kFp8Max));
}

// FP8 E4M3 codes -> f16 values (exact), eight per thread; with `unperm` the codes are in the
// narrow W4A8 tiles' K order (perm8) and the f16 values come out in column order.
__global__ void __launch_bounds__(256) k_e4m3_to_f16(const uint2* __restrict__ q, int64_t n8,
                                                     uint4* __restrict__ out, bool unperm) {
    pdl_enter();
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const uint2 c = unperm ? unperm8(__ldg(q + i)) : __ldg(q + i);
    const uint32_t w[2] = {c.x, c.y};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((w[h >> 1] >> (16 * (h & 1))) & 0xFFFFu), __NV_E4M3);
        o[h] = static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

inline int launch_e4m3_to_f16(const uint8_t* q, int64_t n, uint16_t* out, cudaStream_t stream,
                              bool unperm = false) {
    if (n == 0) return MOE_OK;
    const int64_t n8 = n / 8;
    return launch_pdl(k_e4m3_to_f16, dim3(static_cast<unsigned>((n8 + 255) / 256)), dim3(256), 0, stream,
                      reinterpret_cast<const uint2*>(q), n8, reinterpret_cast<uint4*>(out), unperm);
}

}  // namespace moe

extern "C" int nvfp4_quant_weights(const uint16_t* w_bf16, int64_t experts, int64_t rows, int64_t K,
                                   uint8_t* codes, uint8_t* scales, float* scale2,
                                   moe_stream_t stream) {
    using namespace moe;
    if (experts < 0 || rows < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
    if (K % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (experts == 0 || rows == 0) return MOE_OK;
    if (!w_bf16 || !codes || !scales || !scale2) return MOE_ERR_INVALID_ARG;
    if (!aligned(w_bf16, 16) || !aligned(codes, 8) || !aligned(scale2, 4)) return MOE_ERR_MISALIGNED;
    if (experts > 65535) return MOE_ERR_UNSUPPORTED_SHAPE;
    unsigned* amax = reinterpret_cast<unsigned*>(scale2);
    if (cudaMemsetAsync(amax, 0, experts * sizeof(float), stream) != cudaSuccess) return MOE_ERR_CUDA;
    const int64_t chunks = rows * K / 8;
    const int64_t bx = std::min<int64_t>((chunks + 255) / 256, 64);
    k_nvfp4_amax<<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(experts)), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(w_bf16), chunks, amax);
    const int64_t blocks = rows * K / 16;
    const int64_t total = blocks * experts;
    k_nvfp4_quant<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(w_bf16), blocks, experts, amax, reinterpret_cast<uint2*>(codes), scales);
    k_nvfp4_finish<<<static_cast<unsigned>((experts + 255) / 256), 256, 0, stream>>>(amax, experts);
    return launch_status();
}
