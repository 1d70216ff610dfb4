// ep.cuh — expert parallelism: the E routed experts of a layer held by n_ranks GPUs in
// contiguous ranges of E / n_ranks experts.  The pages serve the layer tensor-parallel over four
// or eight GPUs (Inkling-512k-NVFP4-AQLM-hybrid card, "Serving"; Inkling 2 Small FP8 for AMD
// MI300X card, its launch command); splitting the independent experts instead is the plainest
// multi-GPU form of the same computation, and it moves FP8 token rows rather than activations.
// Each GPU, per layer:
//   moe_ep_dispatch         S2, S3 and S1 on its own tokens: one record per routed pair (the
//                           token's FP8 codes, its scale, the expert's index on its owner),
//                           ordered by expert and so by owner, and the number for each owner;
//   moe_ep_experts_forward  S4-S6 on the records it received: fp32 output rows in record order;
//   moe_ep_combine          S8 and S7 on its own tokens from the rows returned to it.
// The caller moves the records to their owners and the rows back (two all-to-all exchanges).
#pragma once
#include "common.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "forward.cuh"

namespace moe {

constexpr int kEpMeta = 16;   // record bytes after the codes: scale f32, expert i32, 8 zero bytes

__host__ __device__ __forceinline__ int64_t ep_record_bytes(int64_t H) { return H + kEpMeta; }

// S1 for token t (one CTA, the arithmetic of k_quant_tokens) written into the record of each of
// its k pairs, slot rop[t k + j], with the scale and the expert's index within its owner's range.
// CTA 0 also writes the record count of every owner from the expert offsets.
__global__ void __launch_bounds__(256) k_ep_pack(const uint16_t* __restrict__ x, int H, int k,
                                                 const int32_t* __restrict__ ids,
                                                 const int32_t* __restrict__ rop, int E_local,
                                                 const int32_t* __restrict__ offsets, int n_ranks,
                                                 int32_t* __restrict__ send_counts,
                                                 uint8_t* __restrict__ rec) {
    pdl_enter();
    __shared__ float red[32];
    const int64_t t = blockIdx.x;
    const int64_t stride = ep_record_bytes(H);
    if (t == 0)
        for (int r = threadIdx.x; r < n_ranks; r += blockDim.x)
            send_counts[r] = offsets[(r + 1) * E_local] - offsets[r * E_local];
    const uint4* row = reinterpret_cast<const uint4*>(x + t * H);
    const int chunks = H >> 3;
    float a = 0.0f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) a = fmaxf(a, amax8(__ldg(row + c)));
    a = block_max(a, red);
    const float s = __fdiv_rn(a, kFp8Max);
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        const uint2 codes = quant8(__ldg(row + c), s);
        for (int j = 0; j < k; ++j)
            reinterpret_cast<uint2*>(rec + rop[t * k + j] * stride)[c] = codes;
    }
    if (threadIdx.x < k) {
        const int j = threadIdx.x;
        const int e = ids[t * k + j];
        uint8_t* meta = rec + rop[t * k + j] * stride + H;
        *reinterpret_cast<float*>(meta) = s;
        *reinterpret_cast<int32_t*>(meta + 4) = e - (e / E_local) * E_local;
        *reinterpret_cast<uint2*>(meta + 8) = make_uint2(0u, 0u);
    }
}

// The local expert of a received record; an index outside [0, E_local) (a record not written by
// moe_ep_dispatch with this expert split) sets kStatusBadRecord and yields -1.
__device__ __forceinline__ int ep_record_expert(const uint8_t* meta, int E_local) {
    const int e = *reinterpret_cast<const int32_t*>(meta + 4);
    if (e < 0 || e >= E_local) {
        atomicOr(&g_device_status, kStatusBadRecord);
        return -1;
    }
    return e;
}

// ids[r] = the checked local expert of record r (a bad one becomes expert 0; its row is zeroed
// by k_ep_unpack).
__global__ void __launch_bounds__(256) k_ep_ids(const uint8_t* __restrict__ rec, int64_t R, int H,
                                                int E_local, int32_t* __restrict__ ids) {
    pdl_enter();
    const int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (r >= R) return;
    const int e = ep_record_expert(rec + r * ep_record_bytes(H) + H, E_local);
    ids[r] = e < 0 ? 0 : e;
}

// One CTA per received record r: its codes to row dst of q_out (dst = r when rop is null, the
// narrow tiles' per-row gather, in their K order when perm; else rop[r], the expert-sorted row),
// its scale to s_out[dst], and with qsum non-null the per-128-column sums of the FP8 values the
// unsigned widening needs.  With `offsets` non-null (expert-sorted rows of a layer that runs its
// short segments on narrow tiles) perm and qsum apply only to rows of segments of at most
// kShortRows rows.  With ids non-null the checked local expert goes to ids[r].  A record with a
// bad expert index gives a zero row with scale 0 under expert 0.
__global__ void __launch_bounds__(256) k_ep_unpack(const uint8_t* __restrict__ rec, int H, int E_local,
                                                   const int32_t* __restrict__ rop,
                                                   int32_t* __restrict__ ids, uint8_t* __restrict__ q_out,
                                                   float* __restrict__ s_out, float* __restrict__ qsum,
                                                   bool perm, const int32_t* __restrict__ offsets) {
    pdl_enter();
    const int64_t r = blockIdx.x;
    const uint8_t* src = rec + r * ep_record_bytes(H);
    const uint8_t* meta = src + H;
    const int e = *reinterpret_cast<const int32_t*>(meta + 4);
    const bool bad = e < 0 || e >= E_local;
    const int64_t dst = rop ? rop[r] : r;
    if (offsets) {   // uniform over the CTA
        const int ee = bad ? 0 : e;
        perm = offsets[ee + 1] - offsets[ee] <= kShortRows;
        if (!perm) qsum = nullptr;
    }
    const int chunks = H >> 3;
    const int G = H / kGroup;
    for (int base = 0; base < chunks; base += blockDim.x) {   // blockDim = 256: whole half-warps
        const int c = base + threadIdx.x;
        const bool live = c < chunks;
        const uint2 codes = (live && !bad) ? reinterpret_cast<const uint2*>(src)[c] : make_uint2(0u, 0u);
        if (live) reinterpret_cast<uint2*>(q_out + dst * H)[c] = perm ? perm8(codes) : codes;
        if (qsum) {
            const float gs = halfwarp_sum(e4m3x8_sum(codes));
            if (live && (threadIdx.x & 15) == 0) qsum[dst * G + c / 16] = gs;
        }
    }
    if (threadIdx.x == 0) {
        s_out[dst] = bad ? 0.0f : *reinterpret_cast<const float*>(meta);
        if (ids) ids[r] = bad ? 0 : e;
        if (bad) atomicOr(&g_device_status, kStatusBadRecord);
    }
}

// out[r] = y[rop[r]]: the down GEMM's expert-sorted fp32 rows back in record order.
__global__ void __launch_bounds__(256) k_ep_unsort(const float* __restrict__ y,
                                                   const int32_t* __restrict__ rop, int64_t R, int H,
                                                   float* __restrict__ out) {
    pdl_enter();
    const int q = H >> 2;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= R * q) return;
    const int64_t r = i / q;
    const int m4 = static_cast<int>(i % q);
    reinterpret_cast<float4*>(out)[r * q + m4] = reinterpret_cast<const float4*>(y)[(int64_t)rop[r] * q + m4];
}

// The dispatching GPU's workspace, kept from moe_ep_dispatch to moe_ep_combine.
struct EpSendPlan {
    size_t ids, gates, offsets, sorted, rop, route_ws, sh_a, sh_y, sh_wd, total;
};

inline EpSendPlan plan_ep_send(const moe_w4a8_layer& L, int64_t T, int k) {
    EpSendPlan p{};
    const int64_t P = T * k;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + (bytes ? bytes : 1), 256);
        return at;
    };
    p.ids = take(P * 4);
    p.gates = take(P * 4);
    p.offsets = take((L.E + 1) * 4);
    p.sorted = take(P * 4);
    p.rop = take(P * 4);
    p.route_ws = take(route_ws_bytes(T, L.E, k));
    if (L.n_shared > 0) {
        p.sh_a = take((size_t)T * L.n_shared * L.shared_N * 2);
        p.sh_y = take((size_t)T * L.H * 4);
        p.sh_wd = take((size_t)L.n_shared * L.H * L.shared_N * 2);
    }
    p.total = off;
    return p;
}

inline int ep_args_ok(const moe_w4a8_layer* L, int64_t T, int k, int n_ranks) {
    const int st = layer_args_ok(L, T, k);
    if (st != MOE_OK) return st;
    if (n_ranks < 1 || n_ranks > L->E) return MOE_ERR_INVALID_ARG;
    if (L->E % n_ranks) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

}  // namespace moe

extern "C" size_t moe_ep_dispatch_workspace_bytes(const moe_w4a8_layer* layer, int64_t T, int k) {
    if (moe::layer_args_ok(layer, T, k) != MOE_OK) return 0;
    return moe::plan_ep_send(*layer, T, k).total;
}

extern "C" int moe_ep_dispatch(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                               const float* router_logits, int64_t T, int k, int n_ranks,
                               int32_t* send_counts, uint8_t* send_records, void* ws, size_t ws_bytes,
                               moe_stream_t stream) {
    using namespace moe;
    int st = ep_args_ok(layer, T, k, n_ranks);
    if (st != MOE_OK) return st;
    if (!send_counts) return MOE_ERR_INVALID_ARG;
    if (!aligned(send_counts, 4)) return MOE_ERR_MISALIGNED;
    if (T == 0)
        return cudaMemsetAsync(send_counts, 0, n_ranks * sizeof(int32_t), stream) == cudaSuccess ? MOE_OK
                                                                                                 : MOE_ERR_CUDA;
    const moe_w4a8_layer& L = *layer;
    if (!x_bf16 || !router_logits || !send_records) return MOE_ERR_INVALID_ARG;
    const EpSendPlan p = plan_ep_send(L, T, k);
    if (!ws || ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(x_bf16, 16) || !aligned(router_logits, 4) || !aligned(send_records, 16))
        return MOE_ERR_MISALIGNED;
    char* w = static_cast<char*>(ws);
    int32_t* ids = reinterpret_cast<int32_t*>(w + p.ids);
    float* gates = reinterpret_cast<float*>(w + p.gates);
    int32_t* offsets = reinterpret_cast<int32_t*>(w + p.offsets);
    int32_t* rop = reinterpret_cast<int32_t*>(w + p.rop);
    // S2, then S3 over all E experts: owners hold contiguous expert ranges, so the expert-sorted
    // pair order is also owner-sorted and rop[p] is pair p's record slot
    if ((st = launch_topk(router_logits, T, L.E, k, ids, gates, stream))) return st;
    if ((st = launch_permute(ids, T, L.E, k, offsets, reinterpret_cast<int32_t*>(w + p.sorted), rop,
                             reinterpret_cast<int32_t*>(w + p.route_ws), stream)))
        return st;
    return launch_pdl(k_ep_pack, dim3(static_cast<unsigned>(T)), dim3(256), 0, stream, x_bf16, L.H, k,
                      (const int32_t*)ids, (const int32_t*)rop, L.E / n_ranks, (const int32_t*)offsets, n_ranks,
                      send_counts, send_records);
}

extern "C" size_t moe_ep_experts_workspace_bytes(const moe_w4a8_layer* local_layer, int64_t R) {
    if (moe::layer_args_ok(local_layer, R, 1) != MOE_OK) return 0;
    return moe::plan_workspace(*local_layer, R, 1).total;
}

extern "C" int moe_ep_experts_forward(const moe_w4a8_layer* local_layer, const uint8_t* records, int64_t R,
                                      float* y_rows, void* ws, size_t ws_bytes, moe_stream_t stream) {
    using namespace moe;
    int st = layer_args_ok(local_layer, R, 1);
    if (st != MOE_OK) return st;
    if (R == 0) return MOE_OK;
    const moe_w4a8_layer& L = *local_layer;
    if (!records || !y_rows || !L.gate_packed || !L.up_packed || !L.down_packed || !L.gate_scales ||
        !L.up_scales || !L.down_scales)
        return MOE_ERR_INVALID_ARG;
    const WsPlan p = plan_workspace(L, R, 1);
    if (!ws || ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(records, 16) || !aligned(y_rows, 16) || !aligned(L.gate_packed, 16) ||
        !aligned(L.up_packed, 16) || !aligned(L.down_packed, 16) || !aligned(L.gate_scales, 2) ||
        !aligned(L.up_scales, 2) || !aligned(L.down_scales, 2))
        return MOE_ERR_MISALIGNED;
    char* w = static_cast<char*>(ws);
    auto at = [&](size_t off) { return static_cast<void*>(w + off); };
    int32_t* ids = (int32_t*)at(p.topk_ids);
    int32_t* offsets = (int32_t*)at(p.offsets);
    int32_t* sorted = (int32_t*)at(p.sorted);
    int32_t* rop = (int32_t*)at(p.rop);
    uint8_t* xq = (uint8_t*)at(p.xq);
    float* sx = (float*)at(p.s_x);
    uint8_t* xs = (uint8_t*)at(p.x_sorted);
    float* sxs = (float*)at(p.s_x_sorted);
    float* qs_x = (float*)at(p.qs_x);
    unsigned* zero = (unsigned*)at(p.zero);
    // the forward's choice of token tile for R rows over this GPU's E_local experts; narrow W4A8
    // tiles gather the rows in their K order with their group sums, wide ones read expert-sorted
    // copies
    const bool gather = ws_narrow(tc_tile_rows(R, L.E));
    const bool split = ws_split(R, L.E, L.H, L.N);
    float* qs_xr = (float*)at(p.qs_xr);
    const unsigned grid = static_cast<unsigned>(R);
    if (gather) {
        if ((st = launch_pdl(k_ep_unpack, dim3(grid), dim3(256), 0, stream, records, L.H, L.E,
                             (const int32_t*)nullptr, ids, xq, sx, qs_x, true, (const int32_t*)nullptr)))
            return st;
        if ((st = launch_permute(ids, R, L.E, 1, offsets, sorted, rop, (int32_t*)at(p.route_ws), stream, zero,
                                 p.n_zero)))
            return st;
    } else {
        if ((st = launch_pdl(k_ep_ids, dim3((grid + 255) / 256), dim3(256), 0, stream, records, R, L.H, L.E, ids)))
            return st;
        if ((st = launch_permute(ids, R, L.E, 1, offsets, sorted, rop, (int32_t*)at(p.route_ws), stream, zero,
                                 p.n_zero)))
            return st;
        // the forward's split of a layer on 128-row tiles: rows of short segments in the narrow
        // tiles' K order with their group sums
        if ((st = launch_pdl(k_ep_unpack, dim3(grid), dim3(256), 0, stream, records, L.H, L.E, (const int32_t*)rop,
                             (int32_t*)nullptr, xs, sxs, split ? qs_xr : (float*)nullptr, false,
                             split ? (const int32_t*)offsets : (const int32_t*)nullptr)))
            return st;
    }
    StageMarks sm{nullptr, 0, 0};
    RoutedRows rr{offsets, sorted, R, R, 1, gather, gather, xq, sx, xs, sxs, qs_x, split, qs_xr};
    if ((st = run_experts(L, experts_of(L), p, w, rr, nullptr, stream, sm))) return st;
    const int64_t n = R * (L.H / 4);
    return launch_pdl(k_ep_unsort, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, stream,
                      (const float*)at(p.y), (const int32_t*)rop, R, L.H, y_rows);
}

extern "C" int moe_ep_combine(const moe_w4a8_layer* layer, const uint16_t* x_bf16, const float* y_back,
                              int64_t T, int k, uint16_t* out_bf16, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
    using namespace moe;
    int st = layer_args_ok(layer, T, k);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    const moe_w4a8_layer& L = *layer;
    if (!y_back || !out_bf16 || (L.n_shared > 0 && !x_bf16)) return MOE_ERR_INVALID_ARG;
    if (L.n_shared > 0 && (!L.sh_gate || !L.sh_up || !L.sh_down)) return MOE_ERR_INVALID_ARG;
    const EpSendPlan p = plan_ep_send(L, T, k);
    if (!ws || ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(x_bf16, 16) || !aligned(y_back, 16) || !aligned(out_bf16, 16) ||
        !aligned(L.sh_gate, 16) || !aligned(L.sh_up, 16) || !aligned(L.sh_down, 16))
        return MOE_ERR_MISALIGNED;
    char* w = static_cast<char*>(ws);
    StageMarks sm{nullptr, 0, 0};
    float* shared = nullptr;
    if ((st = run_shared(L, reinterpret_cast<uint16_t*>(w + p.sh_a), reinterpret_cast<uint16_t*>(w + p.sh_wd),
                         reinterpret_cast<float*>(w + p.sh_y), x_bf16, T, stream, sm, &shared)))
        return st;
    const int64_t n = T * (L.H / 4);
    return launch_pdl(k_combine, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, stream, y_back,
                      (const float*)(w + p.gates), (const int32_t*)(w + p.rop), k, L.H, T,
                      (const float*)shared, out_bf16);
}
