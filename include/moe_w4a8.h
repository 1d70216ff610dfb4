/*
 * moe_w4a8.h — C ABI of the B200 (sm_100a) W4A8-FP8 routed mixture-of-experts layer.
 *
 * The layer is the routed MoE block of an Inkling-class model whose experts are stored as
 * symmetric INT4 weights in K-groups of 128 and run on FP8 E4M3 activations quantized per
 * token ("Inkling-Small: GPTQ W4A8-FP8 creation and INT4 export recovery" model card,
 * section 1 "What is being created?": its table gives symmetric INT4 weights with 128-wide
 * groups and dynamic FP8 input activations with a per-token scale, and the text defines
 * W4A8-FP8 as 4-bit integer weights with 8-bit floating-point input activations).  256 routed experts with 6 active per token and the gate|up / down expert
 * projections come from the "Inkling-512k-NVFP4-AQLM-hybrid" model card (opening paragraph
 * and "On-disk tensor format").
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers owned by the caller (for example PyTorch
 *     tensors).  The library never allocates, frees or synchronises inside a call, and keeps
 *     no per-call host state, so calls can be captured in a CUDA graph.
 *   - Work is enqueued on `stream` (NULL = legacy default stream) and runs asynchronously.
 *     The return value reports argument validation and launch errors only; faults detected
 *     on the device are reported by moe_last_device_status().
 *   - bf16 values are passed as their 16-bit patterns (uint16_t), FP8 as E4M3 bytes
 *     (uint8_t, OCP E4M3FN: bias 7, max 448, no infinities).
 *   - Matrices are row-major with the last index contiguous.  Pointers to bf16 / fp8 /
 *     int32 matrices must be 16-byte aligned; other pointers need their type's alignment.
 *   - Calls on different streams are independent; a call does not touch memory it was not
 *     given, except the library's sticky device-status word (see moe_last_device_status).
 */
#ifndef MOE_W4A8_H
#define MOE_W4A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same type as cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,       /* null pointer, negative size, k outside [1, min(E, 8)] */
    MOE_ERR_UNSUPPORTED_SHAPE = -2, /* a dimension the kernels do not cover (see each call) */
    MOE_ERR_MISALIGNED = -3,        /* a pointer below its required alignment */
    MOE_ERR_WORKSPACE = -4,         /* workspace missing or smaller than required */
    MOE_ERR_CUDA = -5,              /* a CUDA runtime error at launch */
    MOE_ERR_TIMEOUT = -6,           /* a bounded device-side wait gave up (device status) */
    MOE_ERR_NO_DEVICE = -7          /* no sm_100 device current */
} moe_status;

/* ---------------------------------------------------------------------------------------
 * S0. Offline weight quantization to pack-quantized INT4.
 *
 * Defined by the "Inkling-Small ... model card", section 1 (symmetric INT4 in 128-wide
 * groups) and section 7 "Recover and physically pack INT4" (codes in [-8,7] stored as the nibble
 * code+8; eight consecutive codes along the last dimension in one little-endian I32 word,
 * the first code in the least significant nibble; `.weight_packed` I32 of shape
 * [rows, K/8]).  Scales are stored as bf16 [rows, K/group] (the export's non-I8 payload is
 * BF16, section 5).  Per group of `group` consecutive K:
 *     amax = max |w|,  scale = bf16_rn(amax / 7),  code = clamp(rint(w / scale), -8, 7)
 * (round half to even; an all-zero group gets scale 0 and codes 0).
 *
 *   w_bf16      [rows, K] bf16 weights (out-features x in-features), 16-byte aligned
 *   rows, K     rows >= 0; K a positive multiple of `group`
 *   group       must be 128
 *   packed      [rows, K/8] int32 output, 16-byte aligned
 *   scales_bf16 [rows, K/group] bf16 output
 * Returns MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_MISALIGNED or
 * MOE_ERR_CUDA.  rows == 0 is a no-op.
 * --------------------------------------------------------------------------------------- */
int w4a8_pack_weights(const uint16_t* w_bf16, int64_t rows, int64_t K, int group,
                      int32_t* packed, uint16_t* scales_bf16, moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * S1. Dynamic per-token FP8 quantization (section 1 of the Inkling-Small card: FP8 input
 * activations, scaled per token at run time).  For each row t:
 *     amax = max |x[t,:]|,  scale[t] = amax / 448,  q[t,h] = e4m3_rn_satfinite(x[t,h] / scale[t])
 * with IEEE fp32 division; a row with amax == 0 gets scale 0 and all-zero codes.
 *
 *   x_bf16  [T, H] bf16, 16-byte aligned;  H a positive multiple of 8, at most 65536
 *   q_e4m3  [T, H] E4M3 output, 16-byte aligned
 *   scale   [T] fp32 output
 * T == 0 is a no-op.
 * --------------------------------------------------------------------------------------- */
int fp8_quant_tokens(const uint16_t* x_bf16, int64_t T, int64_t H, uint8_t* q_e4m3,
                     float* scale, moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Router logits: the step upstream of S2.
 *
 * logits[t][e] = sum over k of x[t][k] * wr[e][k], with the router weight kept in its source
 * bf16 precision (the "Inkling-Small-Mixed-Quant-GGUF" card, "Precision differences": router
 * tensors stay native; the "Inkling-512k-NVFP4-AQLM-hybrid" card, "Layout summary": the gate
 * is copied verbatim).  Products of two bf16 values are exact in fp32; the sum is fp32 in an
 * order of the kernel's choosing (so not bit-identical to a sequential sum); no bias.
 *
 *   x_bf16   [T, H] bf16, 16-byte aligned;  H a positive multiple of 8, at most 16384
 *   wr_bf16  [E, H] bf16, 16-byte aligned;  E in [1, 1024]
 *   logits   [T, E] fp32 output, 4-byte aligned (feeds moe_route_topk / moe_w4a8_forward)
 * T == 0 is a no-op.  Small T runs on the CUDA cores (each weight row read once); T >= 256
 * with E a multiple of 128 and H of 64 runs on the tensor cores.
 * --------------------------------------------------------------------------------------- */
int moe_router_logits(const uint16_t* x_bf16, const uint16_t* wr_bf16, int64_t T, int H, int E,
                      float* logits, moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * Router logits fused with S2 (top-k and softmax gate).
 *
 * logits as moe_router_logits, and from them topk_ids / topk_w exactly as moe_route_topk's S2
 * (ranking by logit descending then index ascending, softmax over the selected logits).  For
 * T < 256 (or E not a multiple of 128) the top-k runs inside the router kernel: the CTA that
 * completes a block of tokens ranks those tokens' logits, so routing is one launch; for larger
 * T the tensor-core router is followed by the top-k kernel.
 *
 *   x_bf16, wr_bf16, T, H, E   as moe_router_logits;  k in [1, min(E, 8)]
 *   logits     [T, E] fp32 output (the logits the top-k ranked)
 *   topk_ids   [T, k] int32 out      topk_w [T, k] fp32 out
 *   ws, ws_bytes   device scratch of at least moe_router_topk_workspace_bytes(T, E, k) bytes,
 *                  256-byte aligned (completion counters; contents on entry are ignored)
 * T == 0 is a no-op.
 * --------------------------------------------------------------------------------------- */
size_t moe_router_topk_workspace_bytes(int64_t T, int E, int k);
int moe_router_topk(const uint16_t* x_bf16, const uint16_t* wr_bf16, int64_t T, int H, int E, int k,
                    float* logits, int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes,
                    moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * S2 + S3. Top-k routing and the stable token permutation.
 *
 * Top-k of each row of the router logits (the Inkling-512k card's opening paragraph: 256
 * routed experts per layer, 6 of them active per token): experts are ranked by (logit descending, index ascending); the first
 * k are the selection, in that order.  Gates are a softmax over the selected logits:
 *     gate_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)   (fp32, i, j < k).
 * The routed pairs p = t*k + j are then grouped by expert into one contiguous segment per
 * expert, segments in expert order, pairs ascending in p inside a segment:
 *     expert_offsets[e] = number of pairs routed to experts < e   (expert_offsets[E] = T*k)
 *     sorted_pairs[r]   = the pair at sorted row r;  row_of_pair[p] = its row.
 *
 *   logits          [T, E] fp32;  E in [1, 1024];  k in [1, min(E, 8)]
 *   topk_ids        [T, k] int32 out      topk_w [T, k] fp32 out
 *   expert_offsets  [E + 1] int32 out
 *   sorted_pairs    [T*k] int32 out       row_of_pair [T*k] int32 out
 *   ws, ws_bytes    device scratch of at least moe_route_workspace_bytes(T, E, k) bytes,
 *                   256-byte aligned; contents on entry are ignored
 * --------------------------------------------------------------------------------------- */
size_t moe_route_workspace_bytes(int64_t T, int E, int k);
int moe_route_topk(const float* logits, int64_t T, int E, int k, int32_t* topk_ids,
                   float* topk_w, int32_t* expert_offsets, int32_t* sorted_pairs,
                   int32_t* row_of_pair, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * S4..S8. The layer.
 *
 * Weights of the routed experts in the pack-quantized layout of w4a8_pack_weights, gate and
 * up as separate projections (Inkling-Small card, section 6: the recovered checkpoint keeps
 * separate gate/up projections), stacked over experts:
 *   gate_packed, up_packed  [E, N, H/8] int32     gate_scales, up_scales  [E, N, H/128] bf16
 *   down_packed             [E, H, N/8] int32     down_scales             [E, H, N/128] bf16
 * Shared experts (always on, kept in bf16 — Inkling-Small card section 1: the shared-expert
 * parameters are among those left in BF16), n_shared may be 0 and the pointers NULL:
 *   sh_gate, sh_up          [n_shared, shared_N, H] bf16
 *   sh_down                 [n_shared, H, shared_N] bf16
 * --------------------------------------------------------------------------------------- */
typedef struct {
    int E, H, N, group;
    const int32_t *gate_packed, *up_packed, *down_packed;
    const uint16_t *gate_scales, *up_scales, *down_scales;
    int n_shared, shared_N;
    const uint16_t *sh_gate, *sh_up, *sh_down;
} moe_w4a8_layer;

/* Bytes of device workspace moe_w4a8_forward needs for T tokens and top-k (0 on bad args). */
size_t moe_w4a8_workspace_bytes(const moe_w4a8_layer* layer, int64_t T, int k);

/* Byte offsets, inside the forward workspace, of the intermediates a caller may inspect
 * after the forward completes (all in expert-sorted row order r, P = T*k rows):
 *   topk_ids [T,k] i32, topk_w [T,k] f32, expert_offsets [E+1] i32, sorted_pairs [P] i32,
 *   row_of_pair [P] i32, xq [T,H] e4m3 and s_x [T] f32 (the S1 codes and scales of every
 *   token), hq [P,N] e4m3 and s_h [P] f32 (requantized SwiGLU activations, sorted rows).
 * act_order: 0 when xq and hq hold their codes in column order; 1 when, within every block of
 * 8 columns, they hold columns 0,2,4,6,1,3,5,7 (the order in which the W4A8 GEMM's 16- and
 * 32-row token tiles split a packed word into its even and odd nibbles; used for W4A8 and
 * hybrid layers whose tiles are that narrow); 2 when xq is in column order and the hq rows of
 * experts whose segment has at most 32 rows are in that K order, the other rows in column order
 * (a W4A8 layer on 128-row tiles with H and N of at least 2048, which runs its short segments on
 * 32-row tiles). */
typedef struct {
    size_t topk_ids, topk_w, expert_offsets, sorted_pairs, row_of_pair;
    size_t xq, s_x, hq, s_h;
    size_t total;
    size_t act_order;
} moe_w4a8_ws_layout;
int moe_w4a8_workspace_layout(const moe_w4a8_layer* layer, int64_t T, int k,
                              moe_w4a8_ws_layout* out);

/*
 * out[t,:] = bf16_rn( sum_{j<k} gate[t,j] * Y[(t,j),:]  +  sum_s shared_s(x[t,:]) ) with, for
 * the pair (t,j) routed to expert e:
 *   G[n] = s_x[t] * sum_g s_gate[e,n,g] * sum_{k in g} Xq[t,k] * Cgate[e,n,k]   (likewise U)
 *   h    = silu(G) * U;   s_h = max|h| / 448;   Hq = e4m3(h / s_h)
 *   Y[m] = s_h * sum_g s_down[e,m,g] * sum_{k in g} Hq[k] * Cdown[e,m,k]
 * (Xq, s_x from S1; the routing and permutation of S2/S3).
 *
 *   x_bf16         [T, H] bf16 hidden states        router_logits [T, E] fp32
 *   out_bf16       [T, H] bf16 output
 *   ws, ws_bytes   device scratch, >= moe_w4a8_workspace_bytes(layer, T, k), 256-byte aligned
 * Supported shapes: H and N multiples of 128 (H <= 16384, N <= 8192), group 128, E <= 1024,
 * 1 <= k <= min(E, 8), shared_N a multiple of 128.  T == 0 is a no-op.
 */
int moe_w4a8_forward(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                     const float* router_logits, int64_t T, int k, uint16_t* out_bf16, void* ws,
                     size_t ws_bytes, moe_stream_t stream);

/* Profiling variant of moe_w4a8_forward: the same work, plus `events[i]` (caller-created
 * cudaEvent_t handles, n_events >= MOE_W4A8_N_STAGE_EVENTS) recorded on `stream` at the stage
 * boundaries below, and the number of kernels the call launched in *n_launches (may be NULL).
 *   0 start  1 routed (top-k + permutation)  2 tokens quantized  3 shared experts done
 *   4 gate/up GEMM done  5 SwiGLU requant done  6 down GEMM done  7 combined (end).
 * Stages that a call fuses into a neighbour (the decode path quantizes the tokens in the
 * routing kernel) show as zero-length intervals. */
#define MOE_W4A8_N_STAGE_EVENTS 8
int moe_w4a8_forward_profiled(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                              const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                              void* ws, size_t ws_bytes, moe_stream_t stream,
                              void* const* events, int n_events, int* n_launches);

/* ---------------------------------------------------------------------------------------
 * Row-scaled FP8 (W8A8) experts: a second weight format on the same layer.
 *
 * The "Inkling 2 Small FP8 for AMD MI300X" card ("Precision and files") stores the expert
 * projections as FP8 with one fp32 scale per expert output channel, computed as the row's
 * max |w| over the largest FP8 value, and runs them on per-token FP8 activations.  The card's
 * FP8 is AMD's E4M3FNUZ (largest value 240); this library keeps the one FP8 format it uses
 * everywhere, OCP E4M3FN (448), so a weight row is quantized exactly like a token row of
 * fp8_quant_tokens:
 *     scale[r] = max_k |w[r,k]| / 448,   q[r,k] = e4m3_rn_satfinite(w[r,k] / scale[r])
 *
 *   w_bf16     [rows, K] bf16 weights, 16-byte aligned;  K a positive multiple of 8, <= 65536
 *   q_e4m3     [rows, K] E4M3 output, 16-byte aligned
 *   row_scale  [rows] fp32 output
 * rows == 0 is a no-op.
 * --------------------------------------------------------------------------------------- */
int w8a8_quant_weights(const uint16_t* w_bf16, int64_t rows, int64_t K, uint8_t* q_e4m3,
                       float* row_scale, moe_stream_t stream);

/* The layer with row-scaled FP8 routed experts, gate and up as separate projections:
 *   gate_w8, up_w8  [E, N, H] E4M3      gate_rs, up_rs  [E, N] fp32 row scales
 *   down_w8         [E, H, N] E4M3      down_rs         [E, H] fp32 row scales
 * (E4M3 pointers 16-byte aligned, scales 4-byte aligned); shared experts as in moe_w4a8_layer. */
typedef struct {
    int E, H, N;
    const uint8_t *gate_w8, *up_w8, *down_w8;
    const float *gate_rs, *up_rs, *down_rs;
    int n_shared, shared_N;
    const uint16_t *sh_gate, *sh_up, *sh_down;
} moe_w8a8_layer;

/* Workspace size and layout of moe_w8a8_forward: the same plan (and the same offsets) as the
 * W4A8 layer of equal shape. */
size_t moe_w8a8_workspace_bytes(const moe_w8a8_layer* layer, int64_t T, int k);
int moe_w8a8_workspace_layout(const moe_w8a8_layer* layer, int64_t T, int k,
                              moe_w4a8_ws_layout* out);

/*
 * The layer of moe_w4a8_forward with each projection computed on row-scaled FP8 weights:
 *   G[n] = (sum_k Xq[t,k] * Wgate[e,n,k]) * s_gate[e,n] * s_x[t]      (likewise U)
 *   h    = silu(G) * U;   s_h = max|h| / 448;   Hq = e4m3(h / s_h)
 *   Y[m] = (sum_n Hq[n] * Wdown[e,m,n]) * s_down[e,m] * s_h
 * with the same routing, permutation, requantization, shared experts and combine.  Same
 * shape limits and return codes as moe_w4a8_forward.
 */
int moe_w8a8_forward(const moe_w8a8_layer* layer, const uint16_t* x_bf16,
                     const float* router_logits, int64_t T, int k, uint16_t* out_bf16, void* ws,
                     size_t ws_bytes, moe_stream_t stream);

/* Profiling variant of moe_w8a8_forward, with the stage events of moe_w4a8_forward_profiled. */
int moe_w8a8_forward_profiled(const moe_w8a8_layer* layer, const uint16_t* x_bf16,
                              const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                              void* ws, size_t ws_bytes, moe_stream_t stream,
                              void* const* events, int n_events, int* n_launches);

/* ---------------------------------------------------------------------------------------
 * NVFP4 experts: a third weight format on the same layer.
 *
 * Storage as the "Inkling-512k-NVFP4-AQLM-hybrid" card specifies for its hot experts ("On-disk
 * tensor format", "Dequant math"): two E2M1 (FP4) codes per byte, the first weight of a pair in
 * the low nibble; one E4M3 scale per block of 16 input weights; one fp32 scale2 per expert
 * projection; W = LUT[code] * scale * scale2 with LUT = 0, .5, 1, 1.5, 2, 3, 4, 6 for codes
 * 0..7 and their negatives for 8..15.
 *
 * nvfp4_quant_weights quantizes `experts` bf16 projections [experts, rows, K] (the card's slabs
 * come from an NVFP4 base; this is the usual two-level recipe):
 *     scale2[e] = max |w_e| / (6 * 448)
 *     scale[e, r, b] = e4m3_rn_satfinite(max_{block b} |w| / (6 * scale2[e]))
 *     code = nearest E2M1 value of w / (dec(scale) * scale2[e]), ties to the even code,
 *            at most +-6, the sign kept (a zero scale gives codes 0)
 *   codes    [experts, rows, K/2] uint8 out, 8-byte aligned
 *   scales   [experts, rows, K/16] E4M3 out
 *   scale2   [experts] fp32 out (also used as scratch during the call)
 * K must be a multiple of 16.  Returns as w4a8_pack_weights.
 * --------------------------------------------------------------------------------------- */
int nvfp4_quant_weights(const uint16_t* w_bf16, int64_t experts, int64_t rows, int64_t K,
                        uint8_t* codes, uint8_t* scales, float* scale2, moe_stream_t stream);

/* The layer with NVFP4 routed experts (gate and up separate):
 *   gate_f4, up_f4  [E, N, H/2]    gate_bs, up_bs  [E, N, H/16] E4M3    gate_s2, up_s2  [E] fp32
 *   down_f4         [E, H, N/2]    down_bs         [E, H, N/16] E4M3    down_s2         [E] fp32
 * (codes 16-byte aligned, block scales 8-byte aligned); shared experts as in moe_w4a8_layer. */
typedef struct {
    int E, H, N;
    const uint8_t *gate_f4, *up_f4, *down_f4;
    const uint8_t *gate_bs, *up_bs, *down_bs;
    const float *gate_s2, *up_s2, *down_s2;
    int n_shared, shared_N;
    const uint16_t *sh_gate, *sh_up, *sh_down;
} moe_nvfp4_layer;

/* Workspace of moe_nvfp4_forward: the W4A8 plan plus f16 copies of the GEMM inputs
 * (T*k * max(H, N) * 2 bytes); the layout offsets are the W4A8 layer's. */
size_t moe_nvfp4_workspace_bytes(const moe_nvfp4_layer* layer, int64_t T, int k);
int moe_nvfp4_workspace_layout(const moe_nvfp4_layer* layer, int64_t T, int k,
                               moe_w4a8_ws_layout* out);

/*
 * The layer of moe_w4a8_forward with each projection on NVFP4 weights and the same per-token
 * FP8 activations:
 *   G[n] = (sum_k Xq[t,k] * W_gate[e,n,k]) * s_x[t]        (likewise U), W as dequantized above
 *   h = silu(G) * U;   s_h = max|h| / 448;   Hq = e4m3(h / s_h)
 *   Y[m] = (sum_n Hq[n] * W_down[e,m,n]) * s_h
 * The GPU computes each sum as (sum_k f16(LUT[code] * scale) * f16(dec Xq)) * scale2 (exact
 * products, fp32 accumulation in the tensor core's order).  Same shapes and return codes as
 * moe_w4a8_forward; the profiled variant records the same stage events.
 */
int moe_nvfp4_forward(const moe_nvfp4_layer* layer, const uint16_t* x_bf16,
                      const float* router_logits, int64_t T, int k, uint16_t* out_bf16, void* ws,
                      size_t ws_bytes, moe_stream_t stream);
int moe_nvfp4_forward_profiled(const moe_nvfp4_layer* layer, const uint16_t* x_bf16,
                               const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                               void* ws, size_t ws_bytes, moe_stream_t stream,
                               void* const* events, int n_events, int* n_launches);

/* ---------------------------------------------------------------------------------------
 * Hybrid layers: hot experts in NVFP4, the others in W4A8, dispatched by expert.
 *
 * The "Inkling-512k-NVFP4-AQLM-hybrid" card ("On-disk tensor format") splits each layer's routed
 * experts into a small hot set kept in NVFP4 and a cold set in another format, with hot_ids /
 * cold_ids giving the routed expert of each slab (together a partition of 0..E-1).  Here the
 * cold format is W4A8.  Each routed pair runs the projections of its expert's format; the two
 * formats' grouped GEMMs share the routing, the permutation, the requantization and the
 * combine.
 *   hot_ids  [n_hot] int32, cold_ids [n_cold] int32: must partition 0..E-1 (ids outside [0, E)
 *            are ignored; an expert in neither list contributes nothing)
 *   hot_*    NVFP4 slabs as in moe_nvfp4_layer with n_hot slabs
 *   cold_*   W4A8 slabs as in moe_w4a8_layer with n_cold slabs
 * Workspace, shapes and return codes as moe_nvfp4_forward.
 * --------------------------------------------------------------------------------------- */
typedef struct {
    int E, H, N;
    int n_hot, n_cold;
    const int32_t *hot_ids, *cold_ids;
    const uint8_t *hot_gate_f4, *hot_up_f4, *hot_down_f4;
    const uint8_t *hot_gate_bs, *hot_up_bs, *hot_down_bs;
    const float *hot_gate_s2, *hot_up_s2, *hot_down_s2;
    const int32_t *cold_gate_packed, *cold_up_packed, *cold_down_packed;
    const uint16_t *cold_gate_scales, *cold_up_scales, *cold_down_scales;
    int n_shared, shared_N;
    const uint16_t *sh_gate, *sh_up, *sh_down;
} moe_hybrid_layer;

size_t moe_hybrid_workspace_bytes(const moe_hybrid_layer* layer, int64_t T, int k);
int moe_hybrid_workspace_layout(const moe_hybrid_layer* layer, int64_t T, int k,
                                moe_w4a8_ws_layout* out);
int moe_hybrid_forward(const moe_hybrid_layer* layer, const uint16_t* x_bf16,
                       const float* router_logits, int64_t T, int k, uint16_t* out_bf16, void* ws,
                       size_t ws_bytes, moe_stream_t stream);
int moe_hybrid_forward_profiled(const moe_hybrid_layer* layer, const uint16_t* x_bf16,
                                const float* router_logits, int64_t T, int k, uint16_t* out_bf16,
                                void* ws, size_t ws_bytes, moe_stream_t stream,
                                void* const* events, int n_events, int* n_launches);

/* The layer fed by the router weight instead of precomputed logits: the router logits
 * (moe_router_logits' definition, written into the workspace), then the layer of
 * moe_w4a8_forward / moe_w8a8_forward on them.  At decode sizes (T <= 16) the router, the
 * per-token FP8 quantization (S1) and the top-k (S2) are one kernel.
 *   wr_bf16   [E, H] bf16 router weight, 16-byte aligned
 * Everything else as moe_w4a8_forward / moe_w8a8_forward (same workspace size). */
int moe_w4a8_forward_router(const moe_w4a8_layer* layer, const uint16_t* x_bf16,
                            const uint16_t* wr_bf16, int64_t T, int k, uint16_t* out_bf16,
                            void* ws, size_t ws_bytes, moe_stream_t stream);
int moe_w8a8_forward_router(const moe_w8a8_layer* layer, const uint16_t* x_bf16,
                            const uint16_t* wr_bf16, int64_t T, int k, uint16_t* out_bf16,
                            void* ws, size_t ws_bytes, moe_stream_t stream);
int moe_nvfp4_forward_router(const moe_nvfp4_layer* layer, const uint16_t* x_bf16,
                             const uint16_t* wr_bf16, int64_t T, int k, uint16_t* out_bf16,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/* Waits for `stream`, then returns and clears the library's sticky device-status word for
 * the current device: MOE_OK; MOE_ERR_TIMEOUT when a bounded device-side wait gave up (its
 * kernel then skipped the rest of its work and returned); MOE_ERR_INVALID_ARG when
 * moe_ep_experts_forward met a record naming an expert outside its range (that row was computed
 * as zero); MOE_ERR_CUDA when the stream itself reports an error. */
int moe_last_device_status(moe_stream_t stream);

/* Diagnostic for the failure-detection path: launches one CTA that waits, with the same
 * bounded wait the GEMM kernels use but a limit of `limit_ns` nanoseconds (1 us .. 1 s), on an
 * mbarrier that nothing ever arrives on.  The wait gives up, the kernel sets the sticky
 * device-status word and returns; moe_last_device_status() then reports MOE_ERR_TIMEOUT and the
 * context stays usable.  No page describes this; it exists so the timeout path can be tested
 * without hanging a GPU. */
int moe_selftest_bounded_wait(int64_t limit_ns, moe_stream_t stream);

/* Allocation-free variant of moe_route_topk, for callers that cannot allocate device memory
 * (an engine whose own allocator has reserved all of the GPU's memory up front, so a further
 * allocation fails; a C caller with no device allocator to link).  There is no counterpart on
 * the pages: it is moe_route_topk with the permutation scratch taken from a fixed array inside
 * the library (moe_route_noalloc_max_scratch_bytes() bytes, held by every GPU that loads the
 * library until the process exits) instead of a caller buffer; all outputs are still the
 * caller's.  It supports shapes with moe_route_workspace_bytes(T, E, k) <= that size (for
 * E = 256, up to 262,144 routed pairs) and returns MOE_ERR_UNSUPPORTED_SHAPE beyond it.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress), so
 * make that first call before any stream capture; the address is kept per device (safe when
 * several host threads make their first calls at once) and does not survive a cudaDeviceReset()
 * of that device.  All calls share the one array: calls that
 * overlap on the GPU (issued on streams with no ordering between them) race and must be
 * serialised by the caller.  Every scratch word a call reads is written earlier in the same
 * call, so stale contents from a previous call do not matter.  Never allocates or frees. */
size_t moe_route_noalloc_max_scratch_bytes(void);
int moe_route_topk_noalloc(const float* logits, int64_t T, int E, int k, int32_t* topk_ids,
                           float* topk_w, int32_t* expert_offsets, int32_t* sorted_pairs,
                           int32_t* row_of_pair, moe_stream_t stream);

/* ---- Expert parallelism ---------------------------------------------------------------------
 * The layer's E routed experts held by n_ranks GPUs (E % n_ranks == 0), GPU r owning experts
 * [r E_l, (r + 1) E_l), E_l = E / n_ranks, as a W4A8 layer of E_l experts (its expert e is
 * the full layer's expert r E_l + e).  The pages serve the layer tensor-parallel (TP4 on the
 * Inkling-512k-NVFP4-AQLM-hybrid card, "Serving"; TP8 in the Inkling 2 Small FP8 for AMD MI300X
 * card's launch command); splitting the experts is the plainest multi-GPU form of the same
 * layer, with FP8 rows on the wire.  Per layer, every GPU:
 *   1. moe_ep_dispatch on its T tokens: records and the count for each owner;
 *   2. sends counts[r] records to GPU r and receives R records in total (all-to-all);
 *   3. moe_ep_experts_forward on the R received records: R fp32 rows;
 *   4. returns each received row to its sender, in the order received (all-to-all), so that
 *      it gets back T k rows in the order of its own records;
 *   5. moe_ep_combine on its T tokens.
 * The result equals moe_w4a8_forward of the full layer on the same tokens bit for bit when
 * n_ranks = 1; with more GPUs each owner picks the forward's token tile for its own R rows
 * over E_l experts, and the output keeps that forward's accuracy.
 *
 * Record: MOE_EP_RECORD_BYTES(H) bytes, 16-byte aligned in an array: the token's E4M3 codes
 * [H] (S1, column order), its fp32 scale s_x, the int32 expert index within the owner's range,
 * and 8 zero bytes. */
#define MOE_EP_RECORD_BYTES(H) ((size_t)(H) + 16)

/* Workspace of moe_ep_dispatch, which moe_ep_combine reads back (0 on invalid arguments). */
size_t moe_ep_dispatch_workspace_bytes(const moe_w4a8_layer* layer, int64_t T, int k);

/* S2 (top-k), S3 (stable permutation by expert, hence by owner) and S1 (per-token FP8) on this
 * GPU's tokens.  layer: the full layer's shapes (E, H, N, group; its weight pointers are not
 * read).  x_bf16 [T, H] and router_logits fp32 [T, E] as in moe_w4a8_forward.
 *   send_counts   device int32 [n_ranks]: records for each owner
 *   send_records  device [T k] records, those of owner 0 first, then owner 1, ...; within an
 *                 owner by (expert, pair t k + j)
 * ws (256-byte aligned, moe_ep_dispatch_workspace_bytes) keeps the gates and each pair's
 * record slot for moe_ep_combine: leave it untouched in between.  T == 0 zeroes send_counts.
 * Returns MOE_ERR_UNSUPPORTED_SHAPE when E % n_ranks != 0, MOE_ERR_INVALID_ARG when n_ranks is
 * outside [1, E], else as moe_w4a8_forward. */
int moe_ep_dispatch(const moe_w4a8_layer* layer, const uint16_t* x_bf16, const float* router_logits,
                    int64_t T, int k, int n_ranks, int32_t* send_counts, uint8_t* send_records,
                    void* ws, size_t ws_bytes, moe_stream_t stream);

/* Workspace of moe_ep_experts_forward for R records (0 on invalid arguments). */
size_t moe_ep_experts_workspace_bytes(const moe_w4a8_layer* local_layer, int64_t R);

/* S4-S6 on R received records: y_rows fp32 [R, H] (16-byte aligned), row i for record i.
 * local_layer: this GPU's E_l experts (shared-expert fields are not read).  A record whose
 * expert index is outside [0, E_l) gives a zero row and sets the device-status word
 * (moe_last_device_status).  R == 0 is a no-op. */
int moe_ep_experts_forward(const moe_w4a8_layer* local_layer, const uint8_t* records, int64_t R,
                           float* y_rows, void* ws, size_t ws_bytes, moe_stream_t stream);

/* S8 and S7 on this GPU's tokens: out_bf16 [T, H] = bf16( sum_j gate[t,j] y_back[slot(t,j)]
 * + shared experts(x_t) ), j in selection order, exactly the forward's combine.  y_back fp32
 * [T k, H]: the rows returned for this GPU's records, in record order.  layer, x_bf16, T, k
 * and ws as given to moe_ep_dispatch (layer's shared experts are used; x_bf16 may be null
 * without them). */
int moe_ep_combine(const moe_w4a8_layer* layer, const uint16_t* x_bf16, const float* y_back,
                   int64_t T, int k, uint16_t* out_bf16, void* ws, size_t ws_bytes,
                   moe_stream_t stream);

/* Static description of a status code. */
const char* moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_W4A8_H */
