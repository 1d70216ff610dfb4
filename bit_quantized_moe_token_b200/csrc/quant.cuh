// quant.cuh — S1: dynamic per-token FP8 E4M3 quantization (Inkling-Small W4A8-G128 card,
// section 1: FP8 input activations scaled per token at run time).  scale = amax / 448, q = e4m3_rn_sat(x / scale).
#pragma once
#include "common.cuh"

namespace moe {

__device__ __forceinline__ float block_max(float v, float* red) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    if (w == 0) {
        v = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.0f;
        v = warp_max(v);
        if (l == 0) red[0] = v;
    }
    __syncthreads();
    return red[0];
}

// Eight bf16 (one 16-byte chunk) -> eight E4M3 codes of x / scale (scale 0 -> zeros).
__device__ __forceinline__ uint2 quant8(uint4 v, float scale) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0u, 0u};
    if (scale != 0.0f) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = __fdiv_rn(__uint_as_float(u[q] << 16), scale);
            const float hi = __fdiv_rn(__uint_as_float(u[q] & 0xFFFF0000u), scale);
            o[q >> 1] |= static_cast<uint32_t>(f32x2_to_e4m3x2(lo, hi)) << (16 * (q & 1));
        }
    }
    return make_uint2(o[0], o[1]);
}

__device__ __forceinline__ float amax8(uint4 v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    float a = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        a = fmaxf(a, fabsf(__uint_as_float(u[q] << 16)));
        a = fmaxf(a, fabsf(__uint_as_float(u[q] & 0xFFFF0000u)));
    }
    return a;
}

// One CTA per token row.  With `row_of_pair` non-null the codes and scale of token t are
// written to its k expert-sorted rows (the forward's gathered activation matrix) and, when
// q_tok / s_tok are non-null, also to row t of those; otherwise to row t of q / scale.
__global__ void __launch_bounds__(256) k_quant_tokens(const uint16_t* __restrict__ x, int H,
                                                      uint8_t* __restrict__ q,
                                                      float* __restrict__ scale,
                                                      const int32_t* __restrict__ row_of_pair,
                                                      int k, uint8_t* __restrict__ q_tok,
                                                      float* __restrict__ s_tok) {
    pdl_enter();
    __shared__ float red[32];
    const int64_t t = blockIdx.x;
    const uint4* row = reinterpret_cast<const uint4*>(x + t * H);
    const int chunks = H >> 3;
    float a = 0.0f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) a = fmaxf(a, amax8(__ldg(row + c)));
    a = block_max(a, red);
    const float s = __fdiv_rn(a, kFp8Max);
    const int ncopy = row_of_pair ? k : 1;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        const uint2 codes = quant8(__ldg(row + c), s);
        for (int j = 0; j < ncopy; ++j) {
            const int64_t r = row_of_pair ? row_of_pair[t * k + j] : t;
            reinterpret_cast<uint2*>(q + r * H)[c] = codes;
        }
        if (q_tok) reinterpret_cast<uint2*>(q_tok + t * H)[c] = codes;
    }
    if (threadIdx.x == 0) {
        for (int j = 0; j < ncopy; ++j) scale[row_of_pair ? row_of_pair[t * k + j] : t] = s;
        if (s_tok) s_tok[t] = s;
    }
}

// S1 for token t by the whole CTA: amax, scale = amax / 448, the FP8 codes written once per
// token, and (qsum non-null) per K-group of 128 (16 chunks = one half-warp) the sum of the
// decoded codes.  Same arithmetic as k_quant_tokens.  The group sums serve the narrow W4A8
// tiles' unsigned widening, which reads the codes in its own K order: with qsum non-null the
// codes are stored in that order (perm8).
__device__ __forceinline__ void quant_token_cta(const uint16_t* __restrict__ x, int64_t t, int H,
                                                uint8_t* __restrict__ xq, float* __restrict__ s_x,
                                                float* __restrict__ qsum, float* red) {
    const uint4* row = reinterpret_cast<const uint4*>(x + t * H);
    const int chunks = H >> 3;
    float a = 0.0f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) a = fmaxf(a, amax8(__ldg(row + c)));
    a = block_max(a, red);
    const float s = __fdiv_rn(a, kFp8Max);
    const int G = H / kGroup;
    for (int base = 0; base < chunks; base += blockDim.x) {
        const int c = base + threadIdx.x;
        const bool live = c < chunks;
        const uint2 codes = live ? quant8(__ldg(row + c), s) : make_uint2(0u, 0u);
        if (live) reinterpret_cast<uint2*>(xq + t * H)[c] = qsum ? perm8(codes) : codes;
        const float gs = halfwarp_sum(e4m3x8_sum(codes));
        if (qsum && live && (threadIdx.x & 15) == 0) qsum[t * G + c / 16] = gs;
    }
    if (threadIdx.x == 0) s_x[t] = s;
}

inline int launch_quant_tokens(const uint16_t* x, int64_t T, int64_t H, uint8_t* q, float* s,
                               const int32_t* row_of_pair, int k, cudaStream_t stream,
                               uint8_t* q_tok = nullptr, float* s_tok = nullptr) {
    if (T == 0) return MOE_OK;
    return launch_pdl(k_quant_tokens, dim3(static_cast<unsigned>(T)), dim3(256), 0, stream, x, static_cast<int>(H),
                      q, s, row_of_pair, k, q_tok, s_tok);
}

}  // namespace moe

extern "C" int fp8_quant_tokens(const uint16_t* x_bf16, int64_t T, int64_t H, uint8_t* q_e4m3,
                                float* scale, moe_stream_t stream) {
    using namespace moe;
    if (T < 0 || H <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 8 != 0 || H > 65536) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !q_e4m3 || !scale) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 16) || !aligned(scale, 4)) return MOE_ERR_MISALIGNED;
    if (T > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED_SHAPE;
    return launch_quant_tokens(x_bf16, T, H, q_e4m3, scale, nullptr, 1, stream);
}

// Row-scaled FP8 weights ("Inkling 2 Small FP8 for AMD MI300X" card, "Precision and files": one
// fp32 scale per output channel, the row's max |w| over the largest FP8 value): the per-token
// rule above applied to weight rows.
extern "C" int w8a8_quant_weights(const uint16_t* w_bf16, int64_t rows, int64_t K, uint8_t* q_e4m3,
                                  float* row_scale, moe_stream_t stream) {
    return fp8_quant_tokens(w_bf16, rows, K, q_e4m3, row_scale, stream);
}
