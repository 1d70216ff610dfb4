// tc_pipe.cuh — pieces shared by the warp-specialised tcgen05 GEMMs (gemm_ws.cuh, gemm_w8a8.cuh,
// gemm_bf16_tc.cuh): TMA issue helpers, ring counters, the bounded barrier wait, the fused
// requantization of one row, and the host-side tensor-map encoders.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace ws {

// Four rows (r0..r3) of a 2-D tensor, `box_w` wide from column x, into four consecutive
// box rows at dst (the tensor map's box is one row high).
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, int x, int r0, int r1,
                                            int r2, int r3, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
        ::"r"(tc::smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(tc::smem_u32(bar)),
          "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        ::"r"(tc::smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(tc::smem_u32(bar)),
          "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Named barrier 1 among the promotion / epilogue warps only.
template <int kThreads = 128>
__device__ __forceinline__ void named_sync_math() {
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}


// Slot and phase parity of a ring of N stages, advanced once per stage (no division).
template <int N>
struct Ring {
    int idx = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next() {
        if (++idx == N) { idx = 0; phase ^= 1u; }
    }
};

// Bounded wait that gives up at once after an abort.
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (tc::mbar_try_wait(bar, parity)) return true;      // completed phase: no flag read
    if (*abort) return false;
    if (tc::mbar_wait(bar, parity)) return true;
    *abort = 1;
    return false;
}

}  // namespace ws

// ---- host side --------------------------------------------------------------------------------

using PFN_encodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline PFN_encodeTiled encode_fn() {
    static const PFN_encodeTiled fn = [] {   // looked up once (thread-safe static initialisation)
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<PFN_encodeTiled>(nullptr);
        return reinterpret_cast<PFN_encodeTiled>(p);
    }();
    return fn;
}

// cuTensorMapEncodeTiled (element strides 1, no interleave, 256-byte L2 promotion, zero fill).
inline bool encode_tiled(CUtensorMap* m, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                         const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                         CUtensorMapSwizzle swizzle) {
    PFN_encodeTiled fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dtype, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D byte tensor [rows, row_bytes] (row-major) with a box of box_rows x box_bytes.
inline bool make_map_u8(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                        uint32_t box_bytes, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_bytes, box_rows};
    return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, swizzle);
}

}  // namespace moe
