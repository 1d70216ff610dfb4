// route.cuh — S2 top-k routing with a softmax over the selected logits, and S3 the stable
// permutation of routed pairs into per-expert segments (Inkling-512k-NVFP4-AQLM-hybrid card:
// 256 routed experts per layer with 6 active, opening paragraph; its fused MoE kernels run
// all experts of a layer in one grouped GEMM, section "Serving").
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 8;
constexpr int kChunk = 1024;          // pairs per permutation chunk (one per thread)
constexpr int kSinglePassMaxP = 4096; // above this the permutation runs on one CTA per chunk

// ------------------------------------------------------------------------------------------
// top-k: one warp per token; lane l holds experts l, l+32, ..., (EPL slots)
// ------------------------------------------------------------------------------------------
// kCoherent: read the logits through L2 (they were written by other CTAs of the same kernel).
template <int EPL, bool kCoherent = false>
__device__ __forceinline__ void topk_row(const float* __restrict__ l, int E, int k,
                                         int32_t* __restrict__ ids, float* __restrict__ gates,
                                         int lane) {
    float v[EPL];
    uint32_t taken = 0;
#pragma unroll
    for (int s = 0; s < EPL; ++s) {
        const int e = lane + 32 * s;
        float x = (e < E) ? (kCoherent ? __ldcg(l + e) : __ldg(l + e)) : -INFINITY;
        v[s] = isnan(x) ? -INFINITY : x;
        if (e >= E) taken |= 1u << s;
    }
    float sel[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        sel[j] = 0.0f;
        if (j >= k) continue;
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int s = 0; s < EPL; ++s) {
            const int e = lane + 32 * s;
            if (!((taken >> s) & 1u) && (bi == 0x7FFFFFFF || v[s] > bv)) { bv = v[s]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi != 0x7FFFFFFF && (bi == 0x7FFFFFFF || ov > bv || (ov == bv && oi < bi))) {
                bv = ov;
                bi = oi;
            }
        }
        if (lane == (bi & 31)) taken |= 1u << (bi >> 5);
        if (lane == 0) ids[j] = bi;
        sel[j] = bv;
    }
    if (lane == 0) {
        float ex[kMaxK];
        float sum = 0.0f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            ex[j] = 0.0f;
            if (j < k) {
                ex[j] = expf(sel[j] - sel[0]);
                sum = __fadd_rn(sum, ex[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j < k) gates[j] = __fdiv_rn(ex[j], sum);
    }
}

template <int EPL>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits, int64_t T, int E,
                                              int k, int32_t* __restrict__ ids,
                                              float* __restrict__ gates) {
    pdl_enter();
    const int64_t t = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;  // uniform per warp
    topk_row<EPL>(logits + t * E, E, k, ids + t * k, gates + t * k, threadIdx.x & 31);
}

inline int launch_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* gates,
                       cudaStream_t stream) {
    const int64_t warps = T;
    const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
    const int epl = (E + 31) / 32;
#define MOE_TK(N) launch_pdl(k_topk<N>, dim3(blocks), dim3(256), 0, stream, logits, T, E, k, ids, gates)
    if (epl <= 1) return MOE_TK(1);
    if (epl <= 2) return MOE_TK(2);
    if (epl <= 4) return MOE_TK(4);
    if (epl <= 8) return MOE_TK(8);
    if (epl <= 16) return MOE_TK(16);
    return MOE_TK(32);
#undef MOE_TK
}

// ------------------------------------------------------------------------------------------
// permutation
// ------------------------------------------------------------------------------------------

// Exclusive scan of cnt[0..E) in shared memory (E <= blockDim.x = 1024) into out[] (shared),
// returning the total.  All threads must call it.
__device__ int block_exclusive_scan(const int* cnt, int* out, int E, int* warp_tot) {
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    int v = (t < E) ? cnt[t] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_tot[w] = inc;
    __syncthreads();
    if (w == 0) {
        int s = warp_tot[lane];
        int si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += n;
        }
        warp_tot[lane] = si - s;   // exclusive prefix of warp totals
        if (lane == 31) warp_tot[32] = si;
    }
    __syncthreads();
    if (t < E) out[t] = warp_tot[w] + inc - v;
    const int total = warp_tot[32];
    __syncthreads();
    return total;
}

// Place one chunk of up to 1024 pairs (p0 + threadIdx.x).  base[e] (shared) holds the sorted
// row of the first pair of expert e in this chunk and is advanced past the chunk.
// wc is a shared [32][E] scratch.  Stable: within the chunk, pairs keep increasing p.
__device__ void scatter_chunk(const int32_t* __restrict__ ids, int64_t P, int64_t p0, int E,
                              int* base, int* wc, int32_t* __restrict__ sorted,
                              int32_t* __restrict__ rop) {
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    for (int i = t; i < 32 * E; i += blockDim.x) wc[i] = 0;
    const int64_t p = p0 + t;
    const int e = (p < P) ? ids[p] : -1;
    __syncthreads();
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const unsigned lt = (1u << lane) - 1u;
    const int wrank = __popc(peers & lt);
    if (e >= 0 && (peers & lt) == 0) wc[w * E + e] = __popc(peers);
    __syncthreads();
    if (t < E) {
        int s = base[t];
        for (int ww = 0; ww < 32; ++ww) {
            const int c = wc[ww * E + t];
            wc[ww * E + t] = s;
            s += c;
        }
        base[t] = s;
    }
    __syncthreads();
    if (e >= 0) {
        const int r = wc[w * E + e] + wrank;
        sorted[r] = static_cast<int32_t>(p);
        rop[p] = r;
    }
    __syncthreads();
}

// Whole permutation inside one CTA of 1024 threads (small P); `sm` holds (2E + 33 + 32E) ints.
__device__ void permute_block(const int32_t* __restrict__ ids, int64_t P, int E,
                              int32_t* __restrict__ offsets, int32_t* __restrict__ sorted,
                              int32_t* __restrict__ rop, int* sm) {
    int* cnt = sm;            // E
    int* base = cnt + E;      // E
    int* wt = base + E;       // 33
    int* wc = wt + 33;        // 32 * E
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    for (int64_t p = threadIdx.x; p < P; p += blockDim.x) atomicAdd(&cnt[ids[p]], 1);
    __syncthreads();
    block_exclusive_scan(cnt, base, E, wt);
    for (int i = threadIdx.x; i < E; i += blockDim.x) offsets[i] = base[i];
    if (threadIdx.x == 0) offsets[E] = static_cast<int32_t>(P);
    for (int64_t p0 = 0; p0 < P; p0 += kChunk) scatter_chunk(ids, P, p0, E, base, wc, sorted, rop);
}

inline size_t permute_block_smem(int E) { return (2 * E + 33 + 32 * E) * sizeof(int); }

__global__ void __launch_bounds__(1024) k_permute_single(const int32_t* __restrict__ ids, int64_t P,
                                                         int E, int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ sorted,
                                                         int32_t* __restrict__ rop,
                                                         unsigned* __restrict__ zero, int64_t n_zero) {
    pdl_enter();
    extern __shared__ int sm[];
    for (int64_t i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0u;
    permute_block(ids, P, E, offsets, sorted, rop, sm);
}

// Large P, pass 1: per-chunk expert histogram -> counts[c][E].
__global__ void __launch_bounds__(1024) k_chunk_hist(const int32_t* __restrict__ ids, int64_t P,
                                                     int E, int32_t* __restrict__ counts) {
    pdl_enter();
    extern __shared__ int sm[];
    for (int i = threadIdx.x; i < E; i += blockDim.x) sm[i] = 0;
    __syncthreads();
    const int64_t p = blockIdx.x * (int64_t)kChunk + threadIdx.x;
    if (p < P) atomicAdd(&sm[ids[p]], 1);
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) counts[blockIdx.x * (int64_t)E + i] = sm[i];
}

// Large P, pass 2 (one CTA): offsets, and counts[c][e] := first sorted row of expert e in chunk c.
__global__ void __launch_bounds__(1024) k_chunk_scan(int32_t* __restrict__ counts, int64_t nchunks,
                                                     int64_t P, int E,
                                                     int32_t* __restrict__ offsets) {
    pdl_enter();
    extern __shared__ int sm[];
    int* tot = sm;          // E
    int* base = tot + E;    // E
    int* wt = base + E;     // 33
    const int e = threadIdx.x;
    if (e < E) {
        int s = 0;
        for (int64_t c = 0; c < nchunks; ++c) {
            const int v = counts[c * E + e];
            counts[c * E + e] = s;
            s += v;
        }
        tot[e] = s;
    }
    __syncthreads();
    block_exclusive_scan(tot, base, E, wt);
    if (e < E) {
        offsets[e] = base[e];
        for (int64_t c = 0; c < nchunks; ++c) counts[c * E + e] += base[e];
    }
    if (e == 0) offsets[E] = static_cast<int32_t>(P);
}

// Large P, pass 3: one CTA per chunk.
__global__ void __launch_bounds__(1024) k_chunk_scatter(const int32_t* __restrict__ ids, int64_t P,
                                                        int E, const int32_t* __restrict__ counts,
                                                        int32_t* __restrict__ sorted,
                                                        int32_t* __restrict__ rop) {
    pdl_enter();
    extern __shared__ int sm[];
    int* base = sm;         // E
    int* wc = base + E;     // 32 * E
    for (int i = threadIdx.x; i < E; i += blockDim.x) base[i] = counts[blockIdx.x * (int64_t)E + i];
    __syncthreads();
    scatter_chunk(ids, P, blockIdx.x * (int64_t)kChunk, E, base, wc, sorted, rop);
}

inline size_t route_ws_bytes(int64_t T, int E, int k) {
    const int64_t P = T * k;
    const int64_t nchunks = (P + kChunk - 1) / kChunk;
    return align_up(static_cast<size_t>(nchunks > 0 ? nchunks : 1) * E * sizeof(int32_t), 256);
}

inline int set_smem(const void* fn, size_t bytes) {
    if (bytes <= 48 * 1024) return MOE_OK;
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(bytes)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Also zeroes `n_zero` words at `zero` (may be null) for the forward's accumulators.
inline int launch_permute(const int32_t* ids, int64_t T, int E, int k, int32_t* offsets,
                          int32_t* sorted, int32_t* rop, int32_t* counts, cudaStream_t stream,
                          unsigned* zero = nullptr, int64_t n_zero = 0) {
    const int64_t P = T * k;
    if (P <= kSinglePassMaxP) {
        const size_t smem = permute_block_smem(E);
        if (set_smem((const void*)k_permute_single, smem)) return MOE_ERR_CUDA;
        return launch_pdl(k_permute_single, dim3(1), dim3(1024), smem, stream, ids, P, E, offsets, sorted, rop, zero,
                          n_zero);
    }
    if (zero && cudaMemsetAsync(zero, 0, n_zero * sizeof(unsigned), stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    const int64_t nchunks = (P + kChunk - 1) / kChunk;
    int st = launch_pdl(k_chunk_hist, dim3(static_cast<unsigned>(nchunks)), dim3(1024), E * sizeof(int), stream, ids,
                        P, E, counts);
    if (st == MOE_OK)
        st = launch_pdl(k_chunk_scan, dim3(1), dim3(1024), (2 * E + 33) * sizeof(int), stream, counts, nchunks, P, E,
                        offsets);
    const size_t smem = (E + 32 * E) * sizeof(int);
    if (st == MOE_OK && set_smem((const void*)k_chunk_scatter, smem)) return MOE_ERR_CUDA;
    if (st == MOE_OK)
        st = launch_pdl(k_chunk_scatter, dim3(static_cast<unsigned>(nchunks)), dim3(1024), smem, stream, ids, P, E,
                        counts, sorted, rop);
    return st;
}

inline int route_args_ok(int64_t T, int E, int k) {
    if (T < 0 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
    if (k > E || k > kMaxK || E > kMaxE) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T * k > 0x7FFFFFFFLL) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

}  // namespace moe

extern "C" size_t moe_route_workspace_bytes(int64_t T, int E, int k) {
    if (moe::route_args_ok(T, E, k) != MOE_OK) return 0;
    return moe::route_ws_bytes(T, E, k);
}

extern "C" int moe_route_topk(const float* logits, int64_t T, int E, int k, int32_t* topk_ids,
                              float* topk_w, int32_t* expert_offsets, int32_t* sorted_pairs,
                              int32_t* row_of_pair, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
    using namespace moe;
    int st = route_args_ok(T, E, k);
    if (st != MOE_OK) return st;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_ids || !topk_w || !sorted_pairs || !row_of_pair))
        return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < route_ws_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_w, 4) ||
        !aligned(expert_offsets, 4) || !aligned(sorted_pairs, 4) || !aligned(row_of_pair, 4))
        return MOE_ERR_MISALIGNED;
    if (T == 0) {
        if (cudaMemsetAsync(expert_offsets, 0, (E + 1) * sizeof(int32_t), stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    st = launch_topk(logits, T, E, k, topk_ids, topk_w, stream);
    if (st != MOE_OK) return st;
    return launch_permute(topk_ids, T, E, k, expert_offsets, sorted_pairs, row_of_pair,
                          static_cast<int32_t*>(ws), stream);
}
