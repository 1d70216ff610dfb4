// pack.cuh — S0: symmetric RTN INT4 quantization into pack-quantized storage.
//
// "Inkling-Small: GPTQ W4A8-FP8 creation and INT4 export recovery", section 1 (symmetric
// INT4 in 128-wide groups) and section 7 "Recover and physically pack INT4" (nibble = code + 8,
// eight codes along K per little-endian I32, first code in the least significant nibble).
#pragma once
#include "common.cuh"

namespace moe {

// One thread per packed word (8 consecutive K); the 16 threads of a half-warp cover one
// K-group of 128 and agree on its scale through shuffles.  Because K/8 is a multiple of 16,
// group boundaries fall on half-warp boundaries and a half-warp is entirely live or dead.
__global__ void __launch_bounds__(256) k_pack_weights(const uint4* __restrict__ w, int64_t words,
                                                      int64_t words_per_row,
                                                      int32_t* __restrict__ packed,
                                                      uint16_t* __restrict__ scales) {
    pdl_enter();
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const bool live = i < words;
    const uint4 v = live ? __ldg(w + i) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    float x[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        x[2 * q] = __uint_as_float(u[q] << 16);
        x[2 * q + 1] = __uint_as_float(u[q] & 0xFFFF0000u);
    }
    float a = 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) a = fmaxf(a, fabsf(x[q]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const uint16_t sb = f32_to_bf16_bits(__fdiv_rn(a, 7.0f));
    const float s = bf16_bits_to_f32(sb);
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        int c = 0;
        if (s != 0.0f) {
            float r = rintf(__fdiv_rn(x[q], s));
            r = fminf(fmaxf(r, -8.0f), 7.0f);
            c = static_cast<int>(r);
        }
        word |= static_cast<uint32_t>(c + 8) << (4 * q);
    }
    if (live) {
        packed[i] = static_cast<int32_t>(word);
        if ((threadIdx.x & 15) == 0) scales[i >> 4] = sb;
    }
    (void)words_per_row;
}

}  // namespace moe

extern "C" int w4a8_pack_weights(const uint16_t* w_bf16, int64_t rows, int64_t K, int group,
                                 int32_t* packed, uint16_t* scales_bf16, moe_stream_t stream) {
    using namespace moe;
    if (rows < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
    if (group != kGroup || K % kGroup != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0) return MOE_OK;
    if (!w_bf16 || !packed || !scales_bf16) return MOE_ERR_INVALID_ARG;
    if (!aligned(w_bf16, 16) || !aligned(packed, 16) || !aligned(scales_bf16, 2))
        return MOE_ERR_MISALIGNED;
    const int64_t words = rows * (K / 8);
    const int64_t blocks = (words + 255) / 256;
    k_pack_weights<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(w_bf16), words, K / 8, packed, scales_bf16);
    return launch_status();
}
