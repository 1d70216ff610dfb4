// forward.cuh — S5 SwiGLU + per-row FP8 requantization, S7 combine, the workspace plan and
// moe_w4a8_forward.
#pragma once
#include "common.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "gemm_simple.cuh"
#include "gemm_tc.cuh"
#include "gemm_ws.cuh"

namespace moe {

// S5 requantization of the SwiGLU activations h (fp32, one expert-sorted row per CTA, written
// by the gate/up GEMM together with max|h| per row): s_h = max|h| / 448, Hq = e4m3(h / s_h).
__global__ void __launch_bounds__(256) k_requant(const float* __restrict__ h, int N,
                                                 const unsigned* __restrict__ amax,
                                                 uint8_t* __restrict__ hq, float* __restrict__ s_h) {
    const int64_t r = blockIdx.x;
    const float s = __fdiv_rn(__uint_as_float(amax[r]), kFp8Max);
    const float4* src = reinterpret_cast<const float4*>(h + r * N);
    for (int c = threadIdx.x; c < (N >> 3); c += blockDim.x) {
        uint2 codes = make_uint2(0u, 0u);
        if (s != 0.0f) {
            const float4 a = src[2 * c], b = src[2 * c + 1];
            codes.x = static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s))) |
                      (static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(a.z, s), __fdiv_rn(a.w, s))) << 16);
            codes.y = static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(b.x, s), __fdiv_rn(b.y, s))) |
                      (static_cast<uint32_t>(f32x2_to_e4m3x2(__fdiv_rn(b.z, s), __fdiv_rn(b.w, s))) << 16);
        }
        reinterpret_cast<uint2*>(hq + r * N)[c] = codes;
    }
    if (threadIdx.x == 0) s_h[r] = s;
}

// out[t, m] = bf16( sum_j gate[t,j] * Y[row(t,j), m]  (+ shared[t, m]) ), j in selection
// order.  One thread per (token, 4 consecutive m): float4 loads of the k routed rows.
__global__ void __launch_bounds__(256) k_combine(const float* __restrict__ Y,
                                                 const float* __restrict__ gates,
                                                 const int32_t* __restrict__ rop, int k, int H,
                                                 int64_t T, const float* __restrict__ shared,
                                                 uint16_t* __restrict__ out) {
    const int q = H >> 2;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= T * q) return;
    const int64_t t = i / q;
    const int m4 = static_cast<int>(i % q);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float g = gates[t * k + j];
        const float4 y = reinterpret_cast<const float4*>(Y + (int64_t)rop[t * k + j] * H)[m4];
        o.x = __fadd_rn(o.x, __fmul_rn(g, y.x));
        o.y = __fadd_rn(o.y, __fmul_rn(g, y.y));
        o.z = __fadd_rn(o.z, __fmul_rn(g, y.z));
        o.w = __fadd_rn(o.w, __fmul_rn(g, y.w));
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

// s_out[t, n] = silu(g[t, n]) * u[t, n]   (shared-expert activation, fp32)
__global__ void k_swiglu_f32(const float* __restrict__ g, const float* __restrict__ u,
                             float* __restrict__ a, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        a[i] = __fmul_rn(silu(g[i]), u[i]);
}

// ------------------------------------------------------------------------------------------
// workspace
// ------------------------------------------------------------------------------------------
struct WsPlan {
    size_t topk_ids, topk_w, offsets, sorted, rop, route_ws;
    size_t x_sorted, s_x_sorted, h, amax, hq, s_h, y;
    size_t sh_g, sh_u, sh_a, sh_y;
    size_t total;
};

inline WsPlan plan_workspace(const moe_w4a8_layer& L, int64_t T, int k) {
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
    p.x_sorted = take((size_t)P * L.H);
    p.s_x_sorted = take(P * 4);
    p.h = take((size_t)P * L.N * 4);
    p.amax = take(P * 4);
    p.hq = take((size_t)P * L.N);
    p.s_h = take(P * 4);
    p.y = take((size_t)P * L.H * 4);
    if (L.n_shared > 0) {
        p.sh_g = take((size_t)T * L.shared_N * 4);
        p.sh_u = take((size_t)T * L.shared_N * 4);
        p.sh_a = take((size_t)T * L.shared_N * 4);
        p.sh_y = take((size_t)T * L.H * 4);
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
    out->x_sorted = p.x_sorted;
    out->s_x_sorted = p.s_x_sorted;
    out->hq = p.hq;
    out->s_h = p.s_h;
    out->total = p.total;
    return MOE_OK;
}

namespace moe {

// Records stage-boundary events when profiling; counts kernel launches.
struct StageMarks {
    void* const* ev;
    int n;
    int launches;
    void mark(int i, cudaStream_t s) const {
        if (ev && i < n && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
    }
};

int forward_impl(const moe_w4a8_layer* layer, const uint16_t* x_bf16, const float* router_logits,
                 int64_t T, int k, uint16_t* out_bf16, void* ws, size_t ws_bytes,
                 cudaStream_t stream, StageMarks& sm);

}  // namespace moe

extern "C" int moe_w4a8_forward(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                                const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe::StageMarks sm{nullptr, 0, 0};
    return moe::forward_impl(layer, x_bf16, router_logits, T, k, out_bf16, ws, ws_bytes, stream, sm);
}

extern "C" int moe_w4a8_forward_profiled(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                                         const float* router_logits, int64_t T, int k,
                                         uint16_t* out_bf16, void* ws, size_t ws_bytes,
                                         moe_stream_t stream, void* const* events, int n_events,
                                         int* n_launches) {
    if (events && n_events < MOE_W4A8_N_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    moe::StageMarks sm{events, n_events, 0};
    const int st =
        moe::forward_impl(layer, x_bf16, router_logits, T, k, out_bf16, ws, ws_bytes, stream, sm);
    if (n_launches) *n_launches = sm.launches;
    return st;
}

int moe::forward_impl(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                      const float* router_logits, int64_t T, int k, uint16_t* out_bf16, void* ws,
                      size_t ws_bytes, cudaStream_t stream, StageMarks& sm) {
    using namespace moe;
    int st = layer_args_ok(layer, T, k);
    if (st != MOE_OK) return st;
    const moe_w4a8_layer& L = *layer;
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !router_logits || !out_bf16 || !L.gate_packed || !L.up_packed ||
        !L.down_packed || !L.gate_scales || !L.up_scales || !L.down_scales)
        return MOE_ERR_INVALID_ARG;
    if (L.n_shared > 0 && (!L.sh_gate || !L.sh_up || !L.sh_down)) return MOE_ERR_INVALID_ARG;
    const WsPlan p = plan_workspace(L, T, k);
    if (!ws || ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(x_bf16, 16) || !aligned(out_bf16, 16) ||
        !aligned(router_logits, 4) || !aligned(L.gate_packed, 16) || !aligned(L.up_packed, 16) ||
        !aligned(L.down_packed, 16) || !aligned(L.gate_scales, 2) || !aligned(L.up_scales, 2) ||
        !aligned(L.down_scales, 2))
        return MOE_ERR_MISALIGNED;

    char* w = static_cast<char*>(ws);
    auto at = [&](size_t off) { return static_cast<void*>(w + off); };
    int32_t* ids = (int32_t*)at(p.topk_ids);
    float* gates = (float*)at(p.topk_w);
    int32_t* offsets = (int32_t*)at(p.offsets);
    int32_t* sorted = (int32_t*)at(p.sorted);
    int32_t* rop = (int32_t*)at(p.rop);
    uint8_t* xs = (uint8_t*)at(p.x_sorted);
    float* sxs = (float*)at(p.s_x_sorted);
    float* h = (float*)at(p.h);
    unsigned* amax = (unsigned*)at(p.amax);
    uint8_t* hq = (uint8_t*)at(p.hq);
    float* sh = (float*)at(p.s_h);
    float* y = (float*)at(p.y);
    const int64_t P = T * k;

    sm.mark(0, stream);
    // S2 + S3
    if ((st = launch_topk(router_logits, T, L.E, k, ids, gates, stream))) return st;
    if ((st = launch_permute(ids, T, L.E, k, offsets, sorted, rop, (int32_t*)at(p.route_ws), stream)))
        return st;
    sm.launches += 1 + (P <= kSinglePassMaxP ? 1 : 3);
    sm.mark(1, stream);
    // S1, written straight into the expert-sorted rows
    if ((st = launch_quant_tokens(x_bf16, T, L.H, xs, sxs, rop, k, stream))) return st;
    if (cudaMemsetAsync(amax, 0, P * sizeof(unsigned), stream) != cudaSuccess) return MOE_ERR_CUDA;
    sm.launches += 1;
    sm.mark(2, stream);
    // S4 + SwiGLU: h = silu(G) * U, max|h| per row
    {
        WsGemmArgs a{sxs, L.gate_scales, L.up_scales, offsets, L.E, L.N, L.H, (int)P, h, L.N, amax};
        if ((st = launch_gemm_ws<true>(a, xs, L.gate_packed, L.up_packed, stream))) return st;
    }
    sm.launches += 1;
    sm.mark(3, stream);
    // S5
    k_requant<<<static_cast<unsigned>(P), 256, 0, stream>>>(h, L.N, amax, hq, sh);
    if ((st = launch_status())) return st;
    sm.launches += 1;
    sm.mark(4, stream);
    // S6
    {
        WsGemmArgs a{sh, L.down_scales, nullptr, offsets, L.E, L.H, L.N, (int)P, y, L.H, nullptr};
        if ((st = launch_gemm_ws<false>(a, hq, L.down_packed, nullptr, stream))) return st;
    }
    sm.launches += 1;
    sm.mark(5, stream);
    // S8
    float* shared = nullptr;
    if (L.n_shared > 0) {
        const int Ns = L.shared_N;
        float* sg = (float*)at(p.sh_g);
        float* su = (float*)at(p.sh_u);
        float* sa = (float*)at(p.sh_a);
        shared = (float*)at(p.sh_y);
        for (int s = 0; s < L.n_shared; ++s) {
            const uint16_t* wg = L.sh_gate + (int64_t)s * Ns * L.H;
            const uint16_t* wu = L.sh_up + (int64_t)s * Ns * L.H;
            const uint16_t* wd = L.sh_down + (int64_t)s * L.H * Ns;
            if ((st = launch_gemm_bf16_simple<uint16_t>(x_bf16, wg, (int)T, Ns, L.H, sg, Ns, false, stream)))
                return st;
            if ((st = launch_gemm_bf16_simple<uint16_t>(x_bf16, wu, (int)T, Ns, L.H, su, Ns, false, stream)))
                return st;
            const int64_t n = T * Ns;
            k_swiglu_f32<<<static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 148 * 32)), 256, 0,
                           stream>>>(sg, su, sa, n);
            if ((st = launch_status())) return st;
            if ((st = launch_gemm_bf16_simple<float>(sa, wd, (int)T, L.H, Ns, shared, L.H, s > 0, stream)))
                return st;
            sm.launches += 4;
        }
    }
    sm.mark(6, stream);
    // S7
    {
        const int64_t n = T * (L.H / 4);
        k_combine<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(y, gates, rop, k, L.H, T,
                                                                            shared, out_bf16);
    }
    if ((st = launch_status())) return st;
    sm.launches += 1;
    sm.mark(7, stream);
    return MOE_OK;
}
