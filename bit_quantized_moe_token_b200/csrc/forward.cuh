// forward.cuh — S5 SwiGLU + per-row FP8 requantization, S7 combine, the workspace plan and
// the layer entry points (moe_w4a8_forward, and moe_w8a8_forward for row-scaled FP8 experts).
#pragma once
#include "common.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "gemm_ws.cuh"
#include "gemm_w8a8.cuh"
#include "gemm_nvfp4.cuh"
#include "nvfp4.cuh"
#include "gemm_bf16_tc.cuh"
#include "router.cuh"

namespace moe {

// S5 requantization of the SwiGLU activations h (fp32, one expert-sorted row per CTA, written
// by the gate/up GEMM together with max|h| per row): s_h = max|h| / 448, Hq = e4m3(h / s_h).
// With qsum non-null it also writes each row's per-128-column sums of the FP8 values (the down
// GEMM's unsigned widening removes its +8 offset with them; a half-warp covers one group).  With
// perm the codes are stored in the narrow W4A8 tiles' K order (perm8).
// With `offsets` non-null (a layer whose short segments run on narrow tiles) the order and the
// sums are per row instead: the rows of segments of at most kShortRows rows in the K order with
// their sums, the others in column order without.
__global__ void __launch_bounds__(256) k_requant(const float* __restrict__ h, int N,
                                                 const unsigned* __restrict__ amax,
                                                 uint8_t* __restrict__ hq, float* __restrict__ s_h,
                                                 float* __restrict__ qsum, bool perm,
                                                 const int32_t* __restrict__ offsets, int E) {
    pdl_enter();
    const int64_t r = blockIdx.x;
    if (offsets) {   // the segment of row r: offsets[e] <= r < offsets[e + 1]
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offsets[mid] <= r) lo = mid; else hi = mid - 1;
        }
        perm = offsets[lo + 1] - offsets[lo] <= kShortRows;
        if (!perm) qsum = nullptr;
    }
    const float s = __fdiv_rn(__uint_as_float(amax[r]), kFp8Max);
    const float4* src = reinterpret_cast<const float4*>(h + r * N);
    const int G = N / kGroup;
    for (int c = threadIdx.x; c < (N >> 3); c += blockDim.x) {   // blockDim = 256: whole half-warps
        uint2 codes = make_uint2(0u, 0u);
        if (s != 0.0f) {
            const float4 a = src[2 * c], b = src[2 * c + 1];
            codes.x = static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s))) |
                      (static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(a.z, s), __fdiv_rn(a.w, s))) << 16);
            codes.y = static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(b.x, s), __fdiv_rn(b.y, s))) |
                      (static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(b.z, s), __fdiv_rn(b.w, s))) << 16);
        }
        reinterpret_cast<uint2*>(hq + r * N)[c] = perm ? perm8(codes) : codes;
        if (qsum) {
            const float gs = halfwarp_sum(e4m3x8_sum(codes));
            if ((threadIdx.x & 15) == 0) qsum[r * G + c / 16] = gs;
        }
    }
    if (threadIdx.x == 0) s_h[r] = s;
}

// out[t, m] = bf16( sum_j gate[t,j] * Y[row(t,j), m]  (+ shared[t, m]) ), j in selection
// order.  One thread per (token, 4 consecutive m): the k row indices and gates first, then the k
// float4 loads of the routed rows all in flight at once, then the sum in order.
__global__ void __launch_bounds__(256) k_combine(const float* __restrict__ Y,
                                                 const float* __restrict__ gates,
                                                 const int32_t* __restrict__ rop, int k, int H,
                                                 int64_t T, const float* __restrict__ shared,
                                                 uint16_t* __restrict__ out) {
    pdl_enter();
    const int q = H >> 2;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= T * q) return;
    const int64_t t = i / q;
    const int m4 = static_cast<int>(i % q);
    int row[kMaxK];
    float g[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        row[j] = j < k ? rop[t * k + j] : 0;
        g[j] = j < k ? gates[t * k + j] : 0.0f;
    }
    float4 y[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
        if (j < k) y[j] = reinterpret_cast<const float4*>(Y + (int64_t)row[j] * H)[m4];
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        if (j < k) {
            o.x = __fadd_rn(o.x, __fmul_rn(g[j], y[j].x));
            o.y = __fadd_rn(o.y, __fmul_rn(g[j], y[j].y));
            o.z = __fadd_rn(o.z, __fmul_rn(g[j], y[j].z));
            o.w = __fadd_rn(o.w, __fmul_rn(g[j], y[j].w));
        }
    }
    if (shared) {
        const float4 sh = reinterpret_cast<const float4*>(shared + t * H)[m4];
        o.x = __fadd_rn(o.x, sh.x);
        o.y = __fadd_rn(o.y, sh.y);
        o.z = __fadd_rn(o.z, sh.z);
        o.w = __fadd_rn(o.w, sh.w);
    }
    uint2 packed;
    packed.x = static_cast<uint32_t>(f32_to_bf16_bits(o.x)) | (static_cast<uint32_t>(f32_to_bf16_bits(o.y)) << 16);
    packed.y = static_cast<uint32_t>(f32_to_bf16_bits(o.z)) | (static_cast<uint32_t>(f32_to_bf16_bits(o.w)) << 16);
    reinterpret_cast<uint2*>(out + t * H)[m4] = packed;
}

// S1 + S2 for one token per CTA: warp 0 ranks the token's router logits (top-k, softmax
// gate) while all threads quantize its hidden state to FP8 (amax, scale, codes), written once
// per token; the grouped GEMM gathers the rows it needs by token index.  Same arithmetic as
// k_topk and k_quant_tokens.  kTopk = false: quantization only (the routing came from the
// fused router front).
template <int EPL, bool kTopk = true>
__global__ void __launch_bounds__(256) k_quant_topk(const float* __restrict__ logits,
                                                    const uint16_t* __restrict__ x, int E, int k,
                                                    int H, int32_t* __restrict__ ids,
                                                    float* __restrict__ gates,
                                                    uint8_t* __restrict__ xq,
                                                    float* __restrict__ s_x,
                                                    float* __restrict__ qsum) {
    pdl_enter();
    __shared__ float red[32];
    const int64_t t = blockIdx.x;
    if (kTopk && threadIdx.x < 32) topk_row<EPL>(logits + t * E, E, k, ids + t * k, gates + t * k, threadIdx.x);
    quant_token_cta(x, t, H, xq, s_x, qsum, red);
}

inline int launch_quant_topk(const float* logits, const uint16_t* x, int64_t T, int E, int k, int H,
                             int32_t* ids, float* gates, uint8_t* xq, float* s_x, float* qsum,
                             cudaStream_t stream, bool topk = true) {
    const int epl = (E + 31) / 32;
    const unsigned grid = static_cast<unsigned>(T);
    if (!topk)
        return launch_pdl(k_quant_topk<1, false>, dim3(grid), dim3(256), 0, stream, logits, x, E, k, H, ids, gates,
                          xq, s_x, qsum);
#define MOE_QT(N) launch_pdl(k_quant_topk<N>, dim3(grid), dim3(256), 0, stream, logits, x, E, k, H, ids, gates, xq, \
                             s_x, qsum)
    if (epl <= 1) return MOE_QT(1);
    if (epl <= 2) return MOE_QT(2);
    if (epl <= 4) return MOE_QT(4);
    if (epl <= 8) return MOE_QT(8);
    if (epl <= 16) return MOE_QT(16);
    return MOE_QT(32);
#undef MOE_QT
}

// S1 for token t (one CTA, the arithmetic of k_quant_tokens) written to its k expert-sorted rows
// and to row t of q_tok / s_tok, for a layer whose short segments (at most kShortRows rows) run on
// narrow tiles: rows of short segments get the codes in the narrow tiles' K order (perm8) and
// their per-128-column sums in qsum_rows [P, H / 128], the other rows the codes in column order.
__global__ void __launch_bounds__(256) k_quant_tokens_split(const uint16_t* __restrict__ x, int H, int k,
                                                            const int32_t* __restrict__ ids,
                                                            const int32_t* __restrict__ rop,
                                                            const int32_t* __restrict__ offsets,
                                                            uint8_t* __restrict__ q, float* __restrict__ scale,
                                                            float* __restrict__ qsum_rows,
                                                            uint8_t* __restrict__ q_tok,
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
    int32_t r_[kMaxK];
    bool short_[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        r_[j] = j < k ? rop[t * k + j] : 0;
        const int e = j < k ? ids[t * k + j] : 0;
        short_[j] = j < k && offsets[e + 1] - offsets[e] <= kShortRows;
    }
    const int G = H / kGroup;
    for (int base = 0; base < chunks; base += blockDim.x) {   // blockDim = 256: whole half-warps
        const int c = base + threadIdx.x;
        const bool live = c < chunks;
        const uint2 codes = live ? quant8(__ldg(row + c), s) : make_uint2(0u, 0u);
        const uint2 pc = perm8(codes);
        if (live) {
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                if (j < k) reinterpret_cast<uint2*>(q + (int64_t)r_[j] * H)[c] = short_[j] ? pc : codes;
            reinterpret_cast<uint2*>(q_tok + t * H)[c] = codes;
        }
        const float gs = halfwarp_sum(e4m3x8_sum(codes));
        if (live && (threadIdx.x & 15) == 0) {
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                if (j < k && short_[j]) qsum_rows[(int64_t)r_[j] * G + c / 16] = gs;
        }
    }
    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j < k) scale[r_[j]] = s;
        s_tok[t] = s;
    }
}

// ------------------------------------------------------------------------------------------
// workspace
// ------------------------------------------------------------------------------------------
struct WsPlan {
    size_t topk_ids, topk_w, offsets, sorted, rop, route_ws;
    size_t xq, s_x, x_sorted, s_x_sorted, h, zero, hq, s_h, y;
    size_t qs_x;         // per (token, K-group) sums of the FP8 values (narrow W4A8 tiles)
    size_t qs_h;         // per (sorted row, N-group) sums of the requantized values (W4A8 down GEMM)
    size_t qs_xr;        // per (sorted row, K-group) sums of the FP8 input rows (short segments, split layers)
    size_t logits, rcnt; // router logits [T, E] and the fused router's counters (router entry points)
    size_t act16;        // NVFP4 experts: f16 copies of the GEMM inputs (max of [T|P, H] and [P, N])
    size_t slot_of;      // hybrid layers: expert -> slab map [E]
    int64_t n_zero;   // u32 words at `zero`: max|h| per row [P]
    size_t sh_a, sh_y, sh_wd;
    size_t total;
};

// fmt: 0 W4A8, 1 row-scaled FP8, 2 NVFP4, 3 hybrid (2 and 3 need the f16 activation copies).
inline WsPlan plan_workspace(const moe_w4a8_layer& L, int64_t T, int k, int fmt = 0) {
    WsPlan p{};
    const int64_t P = T * k;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + (bytes ? bytes : 1), 256);
        return at;
    };
    p.topk_ids = take(P * 4);
    p.topk_w = take(P * 4);
    p.offsets = take((L.E + 1) * 4);
    p.sorted = take(P * 4);
    p.rop = take(P * 4);
    p.route_ws = take(route_ws_bytes(T, L.E, k));
    p.xq = take((size_t)T * L.H);
    p.s_x = take(T * 4);
    p.x_sorted = take((size_t)P * L.H);
    p.s_x_sorted = take(P * 4);
    p.h = take((size_t)P * L.N * 4);
    p.n_zero = P;
    p.zero = take((size_t)p.n_zero * 4);
    p.hq = take((size_t)P * L.N);
    p.s_h = take(P * 4);
    p.y = take((size_t)P * L.H * 4);
    p.qs_x = take((size_t)T * (L.H / 128) * 4);
    p.qs_h = take((size_t)P * (L.N / 128) * 4);
    p.qs_xr = take((size_t)P * (L.H / 128) * 4);
    p.logits = take((size_t)T * L.E * 4);
    p.rcnt = take((size_t)router_counter_words(T) * 4);
    p.act16 = fmt >= 2 ? take((size_t)P * (L.H > L.N ? L.H : L.N) * 2) : 0;
    p.slot_of = fmt == 3 ? take((size_t)L.E * 4) : 0;
    if (L.n_shared > 0) {
        p.sh_a = take((size_t)T * L.n_shared * L.shared_N * 2);      // f16 SwiGLU activations
        p.sh_y = take((size_t)T * L.H * 4);
        p.sh_wd = take((size_t)L.n_shared * L.H * L.shared_N * 2);   // f16 copy of the down weights
    }
    p.total = off;
    return p;
}

inline int layer_args_ok(const moe_w4a8_layer* L, int64_t T, int k) {
    if (!L || T < 0) return MOE_ERR_INVALID_ARG;
    if (L->E < 1 || L->H <= 0 || L->N <= 0 || k < 1) return MOE_ERR_INVALID_ARG;
    if (L->group != kGroup || L->H % 128 || L->N % 128 || L->H > 16384 || L->N > 8192)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    int st = route_args_ok(T, L->E, k);
    if (st != MOE_OK) return st;
    if (L->n_shared < 0) return MOE_ERR_INVALID_ARG;
    if (L->n_shared > 0 && (L->shared_N <= 0 || L->shared_N % 128)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

}  // namespace moe

extern "C" size_t moe_w4a8_workspace_bytes(const moe_w4a8_layer* layer, int64_t T, int k) {
    if (moe::layer_args_ok(layer, T, k) != MOE_OK) return 0;
    return moe::plan_workspace(*layer, T, k).total;
}

extern "C" int moe_w4a8_workspace_layout(const moe_w4a8_layer* layer, int64_t T, int k,
                                         moe_w4a8_ws_layout* out) {
    int st = moe::layer_args_ok(layer, T, k);
    if (st != MOE_OK) return st;
    if (!out) return MOE_ERR_INVALID_ARG;
    const moe::WsPlan p = moe::plan_workspace(*layer, T, k);
    out->topk_ids = p.topk_ids;
    out->topk_w = p.topk_w;
    out->expert_offsets = p.offsets;
    out->sorted_pairs = p.sorted;
    out->row_of_pair = p.rop;
    out->xq = p.xq;
    out->s_x = p.s_x;
    out->hq = p.hq;
    out->s_h = p.s_h;
    out->total = p.total;
    // W4A8 layer: see the header
    out->act_order = moe::ws_narrow(moe::ws_tile_rows(T * k, layer->E)) ? 1 : moe::ws_split(T * k, layer->E, layer->H, layer->N) ? 2 : 0;
    return MOE_OK;
}

namespace moe {

// Routed-expert weights of one layer in any of the three formats.
enum ExpertFmt { kFmtW4A8 = 0, kFmtW8A8 = 1, kFmtNvfp4 = 2, kFmtHybrid = 3 };
struct ExpertSet {
    int fmt;
    // W4A8: int32 [E,R,K/8]; W8A8: E4M3 [E,R,K]; NVFP4: [E,R,K/2]; hybrid: the cold W4A8 slabs
    const void *gate, *up, *down;
    // W4A8: bf16 [E,R,K/128]; W8A8: fp32 [E,R]; NVFP4: E4M3 [E,R,K/16]; hybrid: the cold scales
    const void *gate_s, *up_s, *down_s;
    const float *gate_s2 = nullptr, *up_s2 = nullptr, *down_s2 = nullptr;   // NVFP4: fp32 [E]
    // hybrid: the hot NVFP4 slabs and the slab lists
    const void *h_gate = nullptr, *h_up = nullptr, *h_down = nullptr;
    const void *h_gate_s = nullptr, *h_up_s = nullptr, *h_down_s = nullptr;
    const float *h_gate_s2 = nullptr, *h_up_s2 = nullptr, *h_down_s2 = nullptr;
    const int32_t *hot_ids = nullptr, *cold_ids = nullptr;
    int n_hot = 0, n_cold = 0;
};

// Hybrid layers: slot_of[e] = i for the expert of hot slab i, -(j + 1) for that of cold slab j,
// kSlotNone for an expert in neither list (ids outside [0, E) are ignored).
__global__ void __launch_bounds__(1024) k_slot_map(const int32_t* __restrict__ hot_ids, int n_hot,
                                                   const int32_t* __restrict__ cold_ids, int n_cold, int E,
                                                   int32_t* __restrict__ slot_of) {
    pdl_enter();
    for (int e = threadIdx.x; e < E; e += blockDim.x) slot_of[e] = kSlotNone;
    __syncthreads();
    for (int i = threadIdx.x; i < n_hot + n_cold; i += blockDim.x) {
        const int hot = i < n_hot;
        const int32_t e = hot ? hot_ids[i] : cold_ids[i - n_hot];
        if (e >= 0 && e < E) slot_of[e] = hot ? i : -(i - n_hot) - 1;
    }
}

inline ExpertSet experts_of(const moe_w4a8_layer& L) {
    return ExpertSet{kFmtW4A8, L.gate_packed, L.up_packed, L.down_packed, L.gate_scales, L.up_scales,
                     L.down_scales};
}

// Records stage-boundary events when profiling; counts kernel launches.
struct StageMarks {
    void* const* ev;
    int n;
    int launches;
    void mark(int i, cudaStream_t s) const {
        if (ev && i < n && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
    }
};

// `layer` gives the shapes and the shared experts; `xs` the routed experts' weights.  With
// `router_w` non-null the router logits are computed from it (into the workspace) and
// `router_logits` is ignored.
int forward_impl(const moe_w4a8_layer* layer, const ExpertSet& xs, const uint16_t* x_bf16,
                 const float* router_logits, int64_t T, int k, uint16_t* out_bf16, void* ws,
                 size_t ws_bytes, cudaStream_t stream, StageMarks& sm,
                 const uint16_t* router_w = nullptr);

}  // namespace moe

extern "C" int moe_w4a8_forward(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                                const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe::StageMarks sm{nullptr, 0, 0};
    if (!layer) return MOE_ERR_INVALID_ARG;
    return moe::forward_impl(layer, moe::experts_of(*layer), x_bf16, router_logits, T, k, out_bf16, ws,
                             ws_bytes, stream, sm);
}

extern "C" int moe_w4a8_forward_profiled(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                                         const float* router_logits, int64_t T, int k,
                                         uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                         moe_stream_t stream, void* const* events, int n_events,
                                         int* n_launches) {
    if (events && n_events < MOE_W4A8_N_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{events, n_events, 0};
    if (!layer) return MOE_ERR_INVALID_ARG;
    const int st = moe::forward_impl(layer, moe::experts_of(*layer), x_bf16, router_logits, T, k,
                                     out_bf16, ws, ws_bytes, stream, sm);
    if (n_launches) *n_launches = sm.launches;
    return st;
}

namespace moe {
// S8: the shared experts, summed = one SwiGLU MLP of width n_shared * shared_N, into y fp32
// [T, H] through sa (the SwiGLU activations as f16 [T, n_shared shared_N], prescaled by 2^-8)
// and wd (an f16 copy of the down weights [n_shared, H, shared_N]); *shared = y, or null for a
// layer without shared experts.
inline int run_shared(const moe_w4a8_layer& L, uint16_t* sa, uint16_t* wd, float* y, const uint16_t* x_bf16,
                      int64_t T, cudaStream_t stream, StageMarks& sm, float** shared) {
    *shared = nullptr;
    if (L.n_shared <= 0) return MOE_OK;
    const int Wsh = L.n_shared * L.shared_N;
    Bf16GemmArgs g{Wsh, (int)T, L.H, 0, sa, Wsh, 0};
    int st = launch_gemm_bf16_ws<true>(g, x_bf16, L.sh_gate, L.sh_up, stream);
    if (st) return st;
    const int64_t n8 = (int64_t)Wsh * L.H / 8;
    if ((st = launch_pdl(k_bf16_to_f16, dim3(static_cast<unsigned>((n8 + 255) / 256)), dim3(256), 0, stream,
                         reinterpret_cast<const uint4*>(L.sh_down), reinterpret_cast<uint4*>(wd), n8)))
        return st;
    Bf16GemmArgs d{L.H, (int)T, Wsh, L.shared_N, y, L.H, Wsh};
    if ((st = launch_gemm_bf16_ws<false, true>(d, sa, wd, nullptr, stream))) return st;
    sm.launches += 3;
    *shared = y;
    return MOE_OK;
}

// Where S4's routed rows are: narrow tiles (gather) read the per-token codes xq / sx (token =
// pair / k) and, for the W4A8 unsigned widening, the group sums qs_x; wide tiles read the
// expert-sorted copies xs / sxs.
struct RoutedRows {
    const int32_t *offsets, *sorted;
    int64_t P, T;
    int k;
    bool gather, act_perm;
    const uint8_t* xq;
    const float* sx;
    const uint8_t* xs;
    const float* sxs;
    float* qs_x;
    // W4A8 layers on wide tiles: segments of at most kShortRows rows run on narrow tiles (their
    // sorted rows in the narrow tiles' K order, with per-row group sums qs_xr)
    bool split = false;
    const float* qs_xr = nullptr;
};

// S4-S6 on routed rows: gate/up GEMM with the SwiGLU epilogue (h, max|h| per row), the
// requantization, and the down GEMM into the workspace's y [P, H] fp32, expert-sorted rows.
inline int run_experts(const moe_w4a8_layer& L, const ExpertSet& xw, const WsPlan& p, char* w,
                       const RoutedRows& rr, const int32_t* slot_of, cudaStream_t stream, StageMarks& sm) {
    auto at = [&](size_t off) { return static_cast<void*>(w + off); };
    const int32_t* offsets = rr.offsets;
    const int32_t* sorted = rr.sorted;
    const int64_t P = rr.P, T = rr.T;
    const int k = rr.k;
    const bool gather = rr.gather, act_perm = rr.act_perm;
    const uint8_t *xq = rr.xq, *xs = rr.xs;
    const float *sx = rr.sx, *sxs = rr.sxs;
    float* qs_x = rr.qs_x;
    float* h = (float*)at(p.h);
    unsigned* amax = (unsigned*)at(p.zero);
    uint8_t* hq = (uint8_t*)at(p.hq);
    float* sh = (float*)at(p.s_h);
    float* y = (float*)at(p.y);
    float* qs_h = (float*)at(p.qs_h);
    uint16_t* act16 = xw.fmt >= kFmtNvfp4 ? (uint16_t*)at(p.act16) : nullptr;
    const bool hybrid = xw.fmt == kFmtHybrid;
    // the two launches of a hybrid layer's GEMM: W4A8 on the cold experts, NVFP4 on the hot ones
    const bool run_w4 = xw.fmt == kFmtW4A8 || (hybrid && xw.n_cold > 0);
    const bool run_f4 = xw.fmt == kFmtNvfp4 || (hybrid && xw.n_hot > 0);
    const void* f4_gate = hybrid ? xw.h_gate : xw.gate;
    const void* f4_up = hybrid ? xw.h_up : xw.up;
    const void* f4_down = hybrid ? xw.h_down : xw.down;
    const uint8_t* f4_gs = (const uint8_t*)(hybrid ? xw.h_gate_s : xw.gate_s);
    const uint8_t* f4_us = (const uint8_t*)(hybrid ? xw.h_up_s : xw.up_s);
    const uint8_t* f4_ds = (const uint8_t*)(hybrid ? xw.h_down_s : xw.down_s);
    const float* f4_g2 = hybrid ? xw.h_gate_s2 : xw.gate_s2;
    const float* f4_u2 = hybrid ? xw.h_up_s2 : xw.up_s2;
    const float* f4_d2 = hybrid ? xw.h_down_s2 : xw.down_s2;
    int st = MOE_OK;
    // S4 + SwiGLU: h = silu(G) * U, max|h| per row
    if (run_f4) {
        // f16 copy of the FP8 activations (exact), then the f16 tensor-core GEMM
        // (in a narrow hybrid layer the per-token codes are in the W4A8 tiles' K order)
        if ((st = launch_e4m3_to_f16(gather ? xq : xs, (gather ? T : P) * L.H, act16, stream, act_perm)))
            return st;
        F4GemmArgs f{W8GemmArgs{gather ? sx : sxs, nullptr, nullptr, offsets, L.E, L.N, L.H, (int)P, h, L.N,
                                amax, sorted, k, (int)T},
                     f4_gs, f4_us, f4_g2, f4_u2, slot_of, hybrid ? kSlotHot : kSlotAll};
        if ((st = launch_gemm_nvfp4<true>(f, act16, f4_gate, f4_up, stream))) return st;
        sm.launches += 2;
    }
    if (xw.fmt == kFmtW8A8) {
        W8GemmArgs a{gather ? sx : sxs, (const float*)xw.gate_s, (const float*)xw.up_s, offsets, L.E, L.N,
                     L.H, (int)P, h, L.N, amax, sorted, k, (int)T};
        if ((st = launch_gemm_w8a8<true>(a, gather ? (const void*)xq : (const void*)xs, xw.gate, xw.up,
                                         stream)))
            return st;
        sm.launches += 1;
    } else if (run_w4 && rr.split) {
        // the short segments on narrow tiles, then the others on wide tiles
        WsGemmArgs a{sxs, (const uint16_t*)xw.gate_s, (const uint16_t*)xw.up_s, offsets, L.E, L.N, L.H, (int)P, h,
                     L.N, amax, sorted, k, (int)T, rr.qs_xr, nullptr, kSlotShort};
        if ((st = launch_gemm_ws<true>(a, xs, xw.gate, xw.up, stream, kShortRows, true))) return st;
        a.qsum = nullptr;
        a.slot_want = kSlotLong;
        if ((st = launch_gemm_ws<true>(a, xs, xw.gate, xw.up, stream))) return st;
        sm.launches += 2;
    } else if (run_w4) {
        WsGemmArgs a{gather ? sx : sxs, (const uint16_t*)xw.gate_s, (const uint16_t*)xw.up_s, offsets, L.E,
                     L.N, L.H, (int)P, h, L.N, amax, sorted, k, (int)T, gather ? qs_x : nullptr, slot_of,
                     hybrid ? kSlotCold : kSlotAll};
        if ((st = launch_gemm_ws<true>(a, gather ? (const void*)xq : (const void*)xs, xw.gate, xw.up,
                                       stream)))
            return st;
        sm.launches += 1;
    }
    sm.mark(4, stream);
    // S5
    // the W4A8 down GEMM widens its narrow tiles unsigned and needs the requantized rows' group sums;
    // hq, like xq, is stored in those tiles' K order whenever a W4A8 or hybrid layer runs narrow
    const bool down_sums = run_w4 && gather;
    if ((st = launch_pdl(k_requant, dim3(static_cast<unsigned>(P)), dim3(256), 0, stream, h, L.N, amax, hq, sh,
                         (down_sums || rr.split) ? qs_h : nullptr, act_perm,
                         rr.split ? offsets : (const int32_t*)nullptr, L.E)))
        return st;
    sm.launches += 1;
    sm.mark(5, stream);
    // S6
    if (run_f4) {
        if ((st = launch_e4m3_to_f16(hq, P * L.N, act16, stream, act_perm))) return st;
        F4GemmArgs f{W8GemmArgs{sh, nullptr, nullptr, offsets, L.E, L.H, L.N, (int)P, y, L.H, nullptr, sorted,
                                k, (int)T},
                     f4_ds, nullptr, f4_d2, nullptr, slot_of, hybrid ? kSlotHot : kSlotAll};
        if ((st = launch_gemm_nvfp4<false>(f, act16, f4_down, nullptr, stream))) return st;
        sm.launches += 2;
    }
    if (xw.fmt == kFmtW8A8) {
        W8GemmArgs a{sh, (const float*)xw.down_s, nullptr, offsets, L.E, L.H, L.N, (int)P, y, L.H, nullptr,
                     sorted, k, (int)T};
        if ((st = launch_gemm_w8a8<false>(a, hq, xw.down, nullptr, stream))) return st;
        sm.launches += 1;
    } else if (run_w4 && rr.split) {
        WsGemmArgs a{sh, (const uint16_t*)xw.down_s, nullptr, offsets, L.E, L.H, L.N, (int)P, y, L.H, nullptr, sorted,
                     k, (int)T, qs_h, nullptr, kSlotShort};
        if ((st = launch_gemm_ws<false>(a, hq, xw.down, nullptr, stream, kShortRows))) return st;
        a.qsum = nullptr;
        a.slot_want = kSlotLong;
        if ((st = launch_gemm_ws<false>(a, hq, xw.down, nullptr, stream))) return st;
        sm.launches += 2;
    } else if (run_w4) {
        WsGemmArgs a{sh, (const uint16_t*)xw.down_s, nullptr, offsets, L.E, L.H, L.N, (int)P, y, L.H,
                     nullptr, sorted, k, (int)T, down_sums ? qs_h : nullptr, slot_of, hybrid ? kSlotCold : kSlotAll};
        if ((st = launch_gemm_ws<false>(a, hq, xw.down, nullptr, stream))) return st;
        sm.launches += 1;
    }
    sm.mark(6, stream);
    return MOE_OK;
}

}  // namespace moe

int moe::forward_impl(const moe_w4a8_layer* layer, const ExpertSet& xw, const uint16_t* x_bf16,
                      const float* router_logits, int64_t T, int k, uint16_t* out_bf16, void* ws,
                      size_t ws_bytes, cudaStream_t stream, StageMarks& sm, const uint16_t* router_w) {
    using namespace moe;
    int st = layer_args_ok(layer, T, k);
    if (st != MOE_OK) return st;
    const moe_w4a8_layer& L = *layer;
    if (T == 0) return MOE_OK;
    const bool need_base = xw.fmt != kFmtHybrid || xw.n_cold > 0;   // a hybrid may have no cold slab
    if (!x_bf16 || (!router_logits && !router_w) || !out_bf16 ||
        (need_base && (!xw.gate || !xw.up || !xw.down || !xw.gate_s || !xw.up_s || !xw.down_s)))
        return MOE_ERR_INVALID_ARG;
    if (router_w && !aligned(router_w, 16)) return MOE_ERR_MISALIGNED;
    if (L.n_shared > 0 && (!L.sh_gate || !L.sh_up || !L.sh_down)) return MOE_ERR_INVALID_ARG;
    if (L.n_shared > 0 && (!aligned(L.sh_gate, 16) || !aligned(L.sh_up, 16) || !aligned(L.sh_down, 16)))
        return MOE_ERR_MISALIGNED;
    const WsPlan p = plan_workspace(L, T, k, xw.fmt);
    if (!ws || ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    const size_t s_al = xw.fmt == kFmtW8A8 ? 4 : xw.fmt == kFmtNvfp4 ? 8 : 2;   // scale alignment
    if (xw.fmt == kFmtNvfp4 && (!xw.gate_s2 || !xw.up_s2 || !xw.down_s2)) return MOE_ERR_INVALID_ARG;
    if (xw.fmt == kFmtHybrid) {
        if (xw.n_hot < 0 || xw.n_cold < 0 || (xw.n_hot > 0 && !xw.hot_ids) || (xw.n_cold > 0 && !xw.cold_ids))
            return MOE_ERR_INVALID_ARG;
        if (xw.n_hot > 0 && (!xw.h_gate || !xw.h_up || !xw.h_down || !xw.h_gate_s || !xw.h_up_s ||
                             !xw.h_down_s || !xw.h_gate_s2 || !xw.h_up_s2 || !xw.h_down_s2))
            return MOE_ERR_INVALID_ARG;
        if (xw.n_hot > 0 && (!aligned(xw.h_gate, 16) || !aligned(xw.h_up, 16) || !aligned(xw.h_down, 16) ||
                             !aligned(xw.h_gate_s, 8) || !aligned(xw.h_up_s, 8) || !aligned(xw.h_down_s, 8)))
            return MOE_ERR_MISALIGNED;
    }
    if (!aligned(ws, 256) || !aligned(x_bf16, 16) || !aligned(out_bf16, 16) ||
        !aligned(router_logits, 4) || !aligned(xw.gate, 16) || !aligned(xw.up, 16) ||
        !aligned(xw.down, 16) || !aligned(xw.gate_s, s_al) || !aligned(xw.up_s, s_al) ||
        !aligned(xw.down_s, s_al))
        return MOE_ERR_MISALIGNED;      // (null pointers count as aligned)

    const int64_t P = T * k;
    char* w = static_cast<char*>(ws);
    auto at = [&](size_t off) { return static_cast<void*>(w + off); };
    int32_t* ids = (int32_t*)at(p.topk_ids);
    float* gates = (float*)at(p.topk_w);
    int32_t* offsets = (int32_t*)at(p.offsets);
    int32_t* sorted = (int32_t*)at(p.sorted);
    int32_t* rop = (int32_t*)at(p.rop);
    uint8_t* xq = (uint8_t*)at(p.xq);
    float* sx = (float*)at(p.s_x);
    uint8_t* xs = (uint8_t*)at(p.x_sorted);
    float* sxs = (float*)at(p.s_x_sorted);
    unsigned* zero = (unsigned*)at(p.zero);
    float* y = (float*)at(p.y);
    float* qs_x = (float*)at(p.qs_x);
    // narrow token tiles (decode): codes written once per token and gathered by the GEMM; wide
    // tiles (prefill): codes copied to expert-sorted rows.  Either way the requantization (S5)
    // and the combine (S7) run as their own passes: fused into the GEMM epilogues behind
    // device-scope counters they cost every tile a fence and an atomic round trip while the
    // tensor core waited (measured: 7-26 % slower decode layers).
    const bool gather = ws_narrow(tc_tile_rows(P, L.E));
    const bool hybrid = xw.fmt == kFmtHybrid;
    float* qsum_x = (xw.fmt == kFmtW4A8 || hybrid) ? qs_x : nullptr;   // the unsigned widening only
    // narrow W4A8 / hybrid layers store xq and hq in the unsigned widening's K order (perm8); the
    // token quantization writes xq that way exactly when it is given the group sums
    const bool act_perm = gather && qsum_x != nullptr;
    // a W4A8 layer on 128-row tiles runs its short segments on narrow tiles (ws_split)
    const bool split = xw.fmt == kFmtW4A8 && ws_split(P, L.E, L.H, L.N);
    float* qs_xr = (float*)at(p.qs_xr);
    // S1 into the expert-sorted rows (wide tiles) and per token
    auto quant_rows = [&]() -> int {
        if (split)
            return launch_pdl(k_quant_tokens_split, dim3(static_cast<unsigned>(T)), dim3(256), 0, stream, x_bf16,
                              L.H, k, (const int32_t*)ids, (const int32_t*)rop, (const int32_t*)offsets, xs, sxs,
                              qs_xr, xq, sx);
        return launch_quant_tokens(x_bf16, T, L.H, xs, sxs, rop, k, stream, xq, sx);
    };
    int32_t* slot_of = hybrid ? (int32_t*)at(p.slot_of) : nullptr;
    if (hybrid) {
        if ((st = launch_pdl(k_slot_map, dim3(1), dim3(1024), 0, stream, xw.hot_ids, xw.n_hot, xw.cold_ids,
                             xw.n_cold, L.E, slot_of)))
            return st;
        sm.launches += 1;
    }

    sm.mark(0, stream);
    if (router_w) {
        // router logits + S2 (+ S1 at decode) from the router weight
        float* lg = (float*)at(p.logits);
        unsigned* rc = (unsigned*)at(p.rcnt);
        if (cudaMemsetAsync(rc, 0, router_counter_words(T) * 4, stream) != cudaSuccess) return MOE_ERR_CUDA;
        const bool front_quant = gather && T <= 16;
        int nl = 0;
        if ((st = launch_router_topk(x_bf16, router_w, T, L.H, L.E, k, lg, ids, gates, rc,
                                     front_quant ? xq : nullptr, sx, qsum_x, stream, &nl)))
            return st;
        sm.launches += nl;
        sm.mark(1, stream);
        if (gather) {
            if (!front_quant) {
                if ((st = launch_quant_topk(nullptr, x_bf16, T, L.E, k, L.H, ids, gates, xq, sx, qsum_x,
                                            stream, false)))
                    return st;
                sm.launches += 1;
            }
            if ((st = launch_permute(ids, T, L.E, k, offsets, sorted, rop, (int32_t*)at(p.route_ws), stream,
                                     zero, p.n_zero)))
                return st;
            sm.launches += (P <= kSinglePassMaxP ? 1 : 3);
        } else {
            if ((st = launch_permute(ids, T, L.E, k, offsets, sorted, rop, (int32_t*)at(p.route_ws), stream,
                                     zero, p.n_zero)))
                return st;
            if ((st = quant_rows())) return st;
            sm.launches += (P <= kSinglePassMaxP ? 1 : 3) + 1;
        }
        sm.mark(2, stream);
    } else if (gather) {
        // S1 + S2: per-token FP8 codes and top-k
        if ((st = launch_quant_topk(router_logits, x_bf16, T, L.E, k, L.H, ids, gates, xq, sx, qsum_x,
                                    stream)))
            return st;
        sm.launches += 1;
        sm.mark(1, stream);
        // S3 (+ zeroing of the per-row maxima)
        if ((st = launch_permute(ids, T, L.E, k, offsets, sorted, rop, (int32_t*)at(p.route_ws), stream,
                                 zero, p.n_zero)))
            return st;
        sm.launches += (P <= kSinglePassMaxP ? 1 : 3);
        sm.mark(2, stream);
    } else {
        // S2 + S3 (+ zeroing)
        if ((st = launch_topk(router_logits, T, L.E, k, ids, gates, stream))) return st;
        if ((st = launch_permute(ids, T, L.E, k, offsets, sorted, rop, (int32_t*)at(p.route_ws), stream,
                                 zero, p.n_zero)))
            return st;
        sm.launches += 1 + (P <= kSinglePassMaxP ? 1 : 3);
        sm.mark(1, stream);
        // S1, written to the token's k expert-sorted rows and to its own row
        if ((st = quant_rows())) return st;
        sm.launches += 1;
        sm.mark(2, stream);
    }
    // S8
    float* shared = nullptr;
    if ((st = run_shared(L, (uint16_t*)at(p.sh_a), (uint16_t*)at(p.sh_wd), (float*)at(p.sh_y), x_bf16, T, stream,
                         sm, &shared)))
        return st;
    sm.mark(3, stream);
    {
        RoutedRows rr{offsets, sorted, P, T, k, gather, act_perm, xq, sx, xs, sxs, qs_x, split, qs_xr};
        if ((st = run_experts(L, xw, p, w, rr, slot_of, stream, sm))) return st;
    }
    // S7
    {
        const int64_t n = T * (L.H / 4);
        if ((st = launch_pdl(k_combine, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, stream, y,
                             gates, rop, k, L.H, T, shared, out_bf16)))
            return st;
        sm.launches += 1;
    }
    sm.mark(7, stream);
    return MOE_OK;
}

// ---- row-scaled FP8 experts ------------------------------------------------------------------

namespace moe {
// The shape / shared-expert view of a W8A8 layer (group 128: the GEMM's K step).
inline moe_w4a8_layer shape_of(const moe_w8a8_layer& L) {
    return moe_w4a8_layer{L.E, L.H, L.N, kGroup, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                          L.n_shared, L.shared_N, L.sh_gate, L.sh_up, L.sh_down};
}
inline ExpertSet experts_of(const moe_w8a8_layer& L) {
    return ExpertSet{kFmtW8A8, L.gate_w8, L.up_w8, L.down_w8, L.gate_rs, L.up_rs, L.down_rs};
}
}  // namespace moe

extern "C" size_t moe_w8a8_workspace_bytes(const moe_w8a8_layer* layer, int64_t T, int k) {
    if (!layer) return 0;
    const moe_w4a8_layer s = moe::shape_of(*layer);
    return moe_w4a8_workspace_bytes(&s, T, k);
}

extern "C" int moe_w8a8_workspace_layout(const moe_w8a8_layer* layer, int64_t T, int k,
                                         moe_w4a8_ws_layout* out) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    const moe_w4a8_layer s = moe::shape_of(*layer);
    const int st = moe_w4a8_workspace_layout(&s, T, k, out);
    if (st == MOE_OK) out->act_order = 0;          // row-scaled FP8 tiles read the codes in column order
    return st;
}

extern "C" int moe_w8a8_forward(const moe_w8a8_layer* layer, const uint16_t* x_bf16,
                                const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{nullptr, 0, 0};
    const moe_w4a8_layer s = moe::shape_of(*layer);
    return moe::forward_impl(&s, moe::experts_of(*layer), x_bf16, router_logits, T, k, out_bf16, ws,
                             ws_bytes, stream, sm);
}

extern "C" int moe_w8a8_forward_profiled(const moe_w8a8_layer* layer, const uint16_t* x_bf16,
                                         const float* router_logits, int64_t T, int k,
                                         uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                         moe_stream_t stream, void* const* events, int n_events,
                                         int* n_launches) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    if (events && n_events < MOE_W4A8_N_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{events, n_events, 0};
    const moe_w4a8_layer s = moe::shape_of(*layer);
    const int st = moe::forward_impl(&s, moe::experts_of(*layer), x_bf16, router_logits, T, k,
                                     out_bf16, ws, ws_bytes, stream, sm);
    if (n_launches) *n_launches = sm.launches;
    return st;
}

// ---- the layer from the router weight ----------------------------------------------------------

extern "C" int moe_w4a8_forward_router(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                                       const uint16_t* router_w_bf16, int64_t T, int k,
                                       uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                       moe_stream_t stream) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !router_w_bf16) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{nullptr, 0, 0};
    return moe::forward_impl(layer, moe::experts_of(*layer), x_bf16, nullptr, T, k, out_bf16, ws, ws_bytes,
                             stream, sm, router_w_bf16);
}

extern "C" int moe_w8a8_forward_router(const moe_w8a8_layer* layer, const uint16_t* x_bf16,
                                       const uint16_t* router_w_bf16, int64_t T, int k,
                                       uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                       moe_stream_t stream) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !router_w_bf16) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{nullptr, 0, 0};
    const moe_w4a8_layer s = moe::shape_of(*layer);
    return moe::forward_impl(&s, moe::experts_of(*layer), x_bf16, nullptr, T, k, out_bf16, ws, ws_bytes,
                             stream, sm, router_w_bf16);
}

// ---- NVFP4 experts ----------------------------------------------------------------------------

namespace moe {
inline moe_w4a8_layer shape_of(const moe_nvfp4_layer& L) {
    return moe_w4a8_layer{L.E, L.H, L.N, kGroup, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                          L.n_shared, L.shared_N, L.sh_gate, L.sh_up, L.sh_down};
}
inline ExpertSet experts_of(const moe_nvfp4_layer& L) {
    return ExpertSet{kFmtNvfp4, L.gate_f4, L.up_f4, L.down_f4, L.gate_bs, L.up_bs, L.down_bs,
                     L.gate_s2, L.up_s2, L.down_s2};
}
}  // namespace moe

extern "C" size_t moe_nvfp4_workspace_bytes(const moe_nvfp4_layer* layer, int64_t T, int k) {
    if (!layer) return 0;
    const moe_w4a8_layer s = moe::shape_of(*layer);
    if (moe::layer_args_ok(&s, T, k) != MOE_OK) return 0;
    return moe::plan_workspace(s, T, k, moe::kFmtNvfp4).total;
}

extern "C" int moe_nvfp4_workspace_layout(const moe_nvfp4_layer* layer, int64_t T, int k,
                                          moe_w4a8_ws_layout* out) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    const moe_w4a8_layer s = moe::shape_of(*layer);
    int st = moe_w4a8_workspace_layout(&s, T, k, out);
    if (st == MOE_OK) {
        out->total = moe::plan_workspace(s, T, k, moe::kFmtNvfp4).total;
        out->act_order = 0;                        // NVFP4 layers keep the codes in column order
    }
    return st;
}

extern "C" int moe_nvfp4_forward_profiled(const moe_nvfp4_layer* layer, const uint16_t* x_bf16,
                                          const float* router_logits, int64_t T, int k,
                                          uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                          moe_stream_t stream, void* const* events, int n_events,
                                          int* n_launches) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    if (events && n_events < MOE_W4A8_N_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{events, n_events, 0};
    const moe_w4a8_layer s = moe::shape_of(*layer);
    const int st = moe::forward_impl(&s, moe::experts_of(*layer), x_bf16, router_logits, T, k,
                                     out_bf16, ws, ws_bytes, stream, sm);
    if (n_launches) *n_launches = sm.launches;
    return st;
}

extern "C" int moe_nvfp4_forward(const moe_nvfp4_layer* layer, const uint16_t* x_bf16,
                                 const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                                 void* ws, size_t ws_bytes, moe_stream_t stream) {
    return moe_nvfp4_forward_profiled(layer, x_bf16, router_logits, T, k, out_bf16, ws, ws_bytes, stream,
                                      nullptr, 0, nullptr);
}

extern "C" int moe_nvfp4_forward_router(const moe_nvfp4_layer* layer, const uint16_t* x_bf16,
                                        const uint16_t* router_w_bf16, int64_t T, int k,
                                        uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                        moe_stream_t stream) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !router_w_bf16) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{nullptr, 0, 0};
    const moe_w4a8_layer s = moe::shape_of(*layer);
    return moe::forward_impl(&s, moe::experts_of(*layer), x_bf16, nullptr, T, k, out_bf16, ws, ws_bytes,
                             stream, sm, router_w_bf16);
}

// ---- hybrid layers: NVFP4 hot experts, W4A8 cold experts -------------------------------------

namespace moe {
inline moe_w4a8_layer shape_of(const moe_hybrid_layer& L) {
    return moe_w4a8_layer{L.E, L.H, L.N, kGroup, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                          L.n_shared, L.shared_N, L.sh_gate, L.sh_up, L.sh_down};
}
inline ExpertSet experts_of(const moe_hybrid_layer& L) {
    ExpertSet x{kFmtHybrid, L.cold_gate_packed, L.cold_up_packed, L.cold_down_packed, L.cold_gate_scales,
                L.cold_up_scales, L.cold_down_scales};
    x.h_gate = L.hot_gate_f4;
    x.h_up = L.hot_up_f4;
    x.h_down = L.hot_down_f4;
    x.h_gate_s = L.hot_gate_bs;
    x.h_up_s = L.hot_up_bs;
    x.h_down_s = L.hot_down_bs;
    x.h_gate_s2 = L.hot_gate_s2;
    x.h_up_s2 = L.hot_up_s2;
    x.h_down_s2 = L.hot_down_s2;
    x.hot_ids = L.hot_ids;
    x.cold_ids = L.cold_ids;
    x.n_hot = L.n_hot;
    x.n_cold = L.n_cold;
    return x;
}
}  // namespace moe

extern "C" size_t moe_hybrid_workspace_bytes(const moe_hybrid_layer* layer, int64_t T, int k) {
    if (!layer) return 0;
    const moe_w4a8_layer s = moe::shape_of(*layer);
    if (moe::layer_args_ok(&s, T, k) != MOE_OK) return 0;
    return moe::plan_workspace(s, T, k, moe::kFmtHybrid).total;
}

extern "C" int moe_hybrid_workspace_layout(const moe_hybrid_layer* layer, int64_t T, int k,
                                           moe_w4a8_ws_layout* out) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    const moe_w4a8_layer s = moe::shape_of(*layer);
    int st = moe_w4a8_workspace_layout(&s, T, k, out);
    if (st == MOE_OK) {
        out->total = moe::plan_workspace(s, T, k, moe::kFmtHybrid).total;
        if (out->act_order == 2) out->act_order = 0;   // hybrid layers do not split by segment length
    }
    return st;
}

extern "C" int moe_hybrid_forward_profiled(const moe_hybrid_layer* layer, const uint16_t* x_bf16,
                                           const float* router_logits, int64_t T, int k,
                                           uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                           moe_stream_t stream, void* const* events, int n_events,
                                           int* n_launches) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    if (events && n_events < MOE_W4A8_N_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{events, n_events, 0};
    const moe_w4a8_layer s = moe::shape_of(*layer);
    const int st = moe::forward_impl(&s, moe::experts_of(*layer), x_bf16, router_logits, T, k,
                                     out_bf16, ws, ws_bytes, stream, sm);
    if (n_launches) *n_launches = sm.launches;
    return st;
}

extern "C" int moe_hybrid_forward(const moe_hybrid_layer* layer, const uint16_t* x_bf16,
                                  const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                                  void* ws, size_t ws_bytes, moe_stream_t stream) {
    return moe_hybrid_forward_profiled(layer, x_bf16, router_logits, T, k, out_bf16, ws, ws_bytes, stream,
                                       nullptr, 0, nullptr);
}
