// common.cuh — small device helpers shared by the kernels of libmoe_w4a8.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "moe_w4a8.h"

namespace moe {

constexpr int kGroup = 128;   // K-group of the INT4 scales
constexpr float kFp8Max = 448.0f;

// ---- host-side argument checks ---------------------------------------------------------------

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- programmatic dependent launch ------------------------------------------------------------
//
// The layer's kernels follow one rule: a grid waits for the grid launched before it on the
// stream (its completion and memory visibility, griddepcontrol.wait) before it touches any
// buffer that grid writes or reads, and lets the next grid launch only after that wait.  A
// grid that has started therefore knows that every grid two or more launches back has
// completed, and a grid may read data written that far back (expert offsets, weights) before
// its own wait.  The overlap gained: a grid's launch, prologue (barriers, TMEM allocation,
// descriptor prefetch) and any such early reads run under its predecessor's tail.  Both
// instructions are no-ops for a grid launched without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
    pdl_wait();
    pdl_trigger();
}

// Launches `kern` on `stream` with programmatic stream serialization (the kernel must follow the
// rule above).
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess) return MOE_OK;
    (void)cudaGetLastError();   // a rejected launch leaves no error behind for later calls
    return MOE_ERR_CUDA;
}

// ---- conversions -------------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Round to nearest even, subnormals kept (hardware cvt.rn.bf16.f32).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

// Two floats -> two E4M3 bytes, round to nearest even with saturation to +-448 (the
// hardware cvt.rn.satfinite.e4m3x2.f32).  Byte 0 holds `lo`.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    __nv_fp8x2_storage_t r = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
    return static_cast<uint16_t>(r);
}

// E4M3 byte -> float (exact).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
    return __half2float(*reinterpret_cast<__half*>(&h));
}

// Sum of the eight E4M3 values in `codes` (byte 0 of .x first), each decoded exactly.
__device__ __forceinline__ float e4m3x8_sum(uint2 codes) {
    const uint32_t w[2] = {codes.x, codes.y};
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int hgh = 0; hgh < 2; ++hgh) {
            const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * hgh)) & 0xFFFFu), __NV_E4M3);
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
            s += f.x + f.y;
        }
    }
    return s;
}

// The K order of the FP8 activations that narrow W4A8 token tiles read: within each block of
// 8 columns, columns 0,2,4,6,1,3,5,7 (the order in which the GEMM's unsigned widening splits a
// packed word into its even and odd nibbles, so that it needs no byte interleave).  perm8 maps
// eight codes in column order (byte i of .x/.y = column i / i+4) to that order; unperm8 inverts it.
__device__ __forceinline__ uint2 perm8(uint2 c) {
    return make_uint2(__byte_perm(c.x, c.y, 0x6420), __byte_perm(c.x, c.y, 0x7531));
}
__device__ __forceinline__ uint2 unperm8(uint2 c) {
    return make_uint2(__byte_perm(c.x, c.y, 0x5140), __byte_perm(c.x, c.y, 0x7362));
}

// Sum over the 16 lanes of each half-warp (all 32 lanes take part).
__device__ __forceinline__ float halfwarp_sum(float v) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// g * sigmoid(g) with the hardware exp2-based exponential and fast division: a few ulp from
// the IEEE form below, orders of magnitude under the FP8 rounding step that follows it.
__device__ __forceinline__ float silu_fast(float g) {
    return __fdividef(g, 1.0f + __expf(-g));
}

__device__ __forceinline__ float silu(float g) {
    // g * sigmoid(g) with IEEE division; expf is CUDA's (max 2 ulp).
    return g * __fdiv_rn(1.0f, 1.0f + expf(-g));
}

}  // namespace moe
