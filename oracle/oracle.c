/*
 * oracle.c — plain, slow, CPU reference of the W4A8-FP8 routed MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library; the two only read
 * the same seeded inputs.
 *
 * Arithmetic is IEEE fp32 throughout (the layer's stated precision), compiled
 * with -ffp-contract=off and without fast-math, so every expression rounds
 * exactly as written.  Loops follow the definitions step by step; the only
 * freedom taken is loop order across *independent* outputs (and OpenMP over
 * independent experts/tokens), which never changes a value: every sum below
 * is accumulated in the order the definition states.
 *
 * Sources (web pages; the section named is where the fact is stated):
 *  [P1] "Inkling-Small: GPTQ W4A8-FP8 creation and INT4 export recovery"
 *       (wstewart3/Inkling-Small-W4A8-G128 model card):
 *       §1 "What is being created?" — symmetric INT4 weights in groups of 128,
 *       dynamic per-token FP8 activations, W4A8-FP8 = INT4 weights + FP8
 *       input activations; §5 — scales are stored next to I8 codes with a BF16
 *       payload (no F32 payload); §7 "Recover and physically pack INT4" —
 *       codes in [-8,7], nibble = code+8, eight codes along the last dim per
 *       little-endian I32, first code in the least significant nibble.
 *  [P2] "Inkling-512k-NVFP4-AQLM-hybrid" model card: 256 routed experts, 6
 *       active; "On-disk tensor format" — w13 = fused gate|up, w2 = down.
 *  [P5] "Inkling 2 Small FP8 for AMD MI300X", "Precision and files": expert
 *       projections in FP8 with one fp32 scale per expert output channel,
 *       scale = max|row| / (largest FP8 value), per-token FP8 activations.
 *  [P2] also, "On-disk tensor format" / "Dequant math": NVFP4 hot experts —
 *       two E2M1 codes per byte (low nibble first), one E4M3 scale per block of
 *       16 input weights, one fp32 scale2 per expert; W = LUT[code] * scale *
 *       scale2 with LUT = 0 .5 1 1.5 2 3 4 6 and their negatives (codes 8..15).
 *  Readings where the pages are silent (listed with each function):
 *   R1 symmetric RTN scale = amax/7 stored as BF16 (round to nearest even),
 *      codes = clamp(rint(w/scale), -8, 7), all-zero group -> scale 0, codes 0;
 *   R2 per-token FP8 = OCP E4M3FN (max 448), scale = amax/448, q = E4M3(x/s)
 *      with round-to-nearest-even and saturation; zero row -> s = 0, q = 0;
 *   R3 gate = softmax over the k selected logits; ties -> lower expert index;
 *   R4 expert MLP = down(silu(gate(x)) * up(x)); the SwiGLU output is
 *      requantized to FP8 per routed (token, expert) row like R2;
 *   R5 group partial sums in increasing k, promoted with the group scale in
 *      increasing g, token scale applied last; combine sums the k routed
 *      outputs in selection order, adds the shared experts, rounds once to
 *      bf16;
 *   R6 router logits = x . wr over the bf16 router weight, no bias, fp32
 *      accumulation in increasing k;
 *   R7 row-scaled FP8 experts ([P5]) use the OCP E4M3FN format of R2, so the
 *      row scale is amax/448 (the page's 240 is the largest E4M3FNUZ value),
 *      codes = E4M3(w/scale) exactly as R2 does for a token row; a projection
 *      output is (sum_k dec(q_k) dec(w_k), k increasing) * s_w[n] * s_x.
 *   R8 NVFP4 quantization (the page's hot slabs come from an NVFP4 base this
 *      build does not have): per expert projection scale2 = amax / (6*448);
 *      per block of 16 scale = E4M3(amax_block / (6*scale2)) as in R2; code =
 *      nearest E2M1 value of w / (dec(scale)*scale2), ties to the even code,
 *      saturating at +-6, sign kept (-0 -> code 8); a zero scale gives codes 0.
 *   R9 NVFP4 experts run on the same per-token FP8 activations (S1): a
 *      projection output is (sum_k dec(q_k) * W[n,k], k increasing) * s_x with
 *      W dequantized by the page's formula in fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

/* Threads of the OpenMP loops below, for timing the oracle at a chosen core count; results never
 * depend on it (every parallel loop runs over independent experts or tokens). */
void or_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
int or_max_threads(void) { return omp_get_max_threads(); }

/* ------------------------------------------------------------------------------------------ */
/* bf16                                                                                        */
/* ------------------------------------------------------------------------------------------ */

typedef union { float f; uint32_t u; } fbits;

float or_bf16_to_f32(uint16_t h) {
    fbits b;
    b.u = (uint32_t)h << 16;
    return b.f;
}

/* Round a finite fp32 to the nearest bf16, ties to even. */
uint16_t or_f32_to_bf16(float f) {
    fbits b;
    b.f = f;
    uint32_t lsb = (b.u >> 16) & 1u;
    return (uint16_t)((b.u + 0x7FFFu + lsb) >> 16);
}

/* ------------------------------------------------------------------------------------------ */
/* OCP FP8 E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities; S.1111.111 is   */
/* NaN; largest finite 448; subnormals m * 2^-9.                                                */
/* ------------------------------------------------------------------------------------------ */

float or_e4m3_decode(uint8_t c) {
    int s = c >> 7, E = (c >> 3) & 15, M = c & 7;
    float v;
    if (E == 15 && M == 7) return NAN;
    if (E == 0) v = ldexpf((float)M, -9);
    else v = ldexpf(1.0f + (float)M / 8.0f, E - 7);
    return s ? -v : v;
}

/* Nearest E4M3 value to finite x, ties to even mantissa, saturating to +-448. */
uint8_t or_e4m3_encode(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    float a = fabsf(x);
    if (a >= 448.0f) return sign | 0x7E;
    /* spacing of E4M3 values around a: 2^-9 below 2^-6 (subnormals), else 2^(floor(log2 a)-3) */
    int q_exp;
    if (a < ldexpf(1.0f, -6)) {
        q_exp = -9;
    } else {
        int e2;
        frexpf(a, &e2);          /* a = f * 2^e2, f in [0.5,1) -> floor(log2 a) = e2-1 */
        q_exp = (e2 - 1) - 3;
    }
    float n = rintf(ldexpf(a, -q_exp));  /* exact scaling; rintf rounds half to even */
    float v = ldexpf(n, q_exp);          /* the rounded magnitude */
    if (v >= 448.0f) return sign | 0x7E; /* cannot exceed: a < 448 rounds to <= 448 */
    if (v < ldexpf(1.0f, -6)) return sign | (uint8_t)n; /* subnormal (n = 8 is 2^-6 = 0x08) */
    int e2;
    float f = frexpf(v, &e2);            /* v = f * 2^e2, f in [0.5,1) */
    int E = (e2 - 1) + 7;
    int M = (int)(f * 16.0f) - 8;        /* f*16 in [8,16) exactly */
    return sign | (uint8_t)((E << 3) | M);
}

/* ------------------------------------------------------------------------------------------ */
/* S0: symmetric RTN INT4 in K-groups, pack-quantized storage ([P1] §1, §7; readings R1).        */
/* ------------------------------------------------------------------------------------------ */

/* One group: amax = max |w|; s = bf16(amax / 7); code = clamp(rint(w / s), -8, 7). */
static void rtn_group(const uint16_t* w, int n, int8_t* codes, uint16_t* scale_bf16) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(or_bf16_to_f32(w[i]));
        if (a > amax) amax = a;
    }
    uint16_t sb = or_f32_to_bf16(amax / 7.0f);
    float s = or_bf16_to_f32(sb);
    for (int i = 0; i < n; ++i) {
        if (s == 0.0f) { codes[i] = 0; continue; }
        float r = rintf(or_bf16_to_f32(w[i]) / s);
        if (r < -8.0f) r = -8.0f;
        if (r > 7.0f) r = 7.0f;
        codes[i] = (int8_t)r;
    }
    *scale_bf16 = sb;
}

/* Pack eight codes along K into one little-endian word, first code in the low nibble,
 * nibble = code + 8 ([P1] §7). Returns -1 if a code is outside [-8, 7]. */
static int pack_word(const int8_t* c, int32_t* out) {
    uint32_t w = 0;
    for (int i = 0; i < 8; ++i) {
        if (c[i] < -8 || c[i] > 7) return -1;
        w |= (uint32_t)(c[i] + 8) << (4 * i);
    }
    memcpy(out, &w, 4);
    return 0;
}

/* W bf16 [rows, K] (K innermost) -> packed int32 [rows, K/8], scales bf16 [rows, K/group].
 * Also returns the unpacked codes when `codes` is non-NULL. Returns 0, or -1 on bad shape. */
int or_rtn_pack(const uint16_t* w, int64_t rows, int64_t K, int group, int32_t* packed,
                uint16_t* scales, int8_t* codes_out) {
    if (group <= 0 || K % group != 0 || group % 8 != 0) return -1;
    int64_t G = K / group;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t r = 0; r < rows; ++r) {
        int8_t* codes = (int8_t*)malloc((size_t)K);
        for (int64_t g = 0; g < G; ++g)
            rtn_group(w + r * K + g * group, group, codes + g * group, scales + r * G + g);
        for (int64_t j = 0; j < K / 8; ++j) bad |= pack_word(codes + 8 * j, packed + r * (K / 8) + j);
        if (codes_out) memcpy(codes_out + r * K, codes, (size_t)K);
        free(codes);
    }
    return bad ? -1 : 0;
}

/* Inverse of the packing: code of K-index 8j+i is nibble i of word j minus 8. */
void or_unpack(const int32_t* packed, int64_t rows, int64_t K, int8_t* codes) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < K / 8; ++j) {
            uint32_t w;
            memcpy(&w, packed + r * (K / 8) + j, 4);
            for (int i = 0; i < 8; ++i) codes[r * K + 8 * j + i] = (int8_t)((int)((w >> (4 * i)) & 15u) - 8);
        }
}

/* ------------------------------------------------------------------------------------------ */
/* S1: dynamic per-token FP8 ([P1] §1: FP8 activations with a per-token scale; reading R2).   */
/* ------------------------------------------------------------------------------------------ */

static void quant_row_f32(const float* x, int64_t n, uint8_t* q, float* s_out) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    for (int64_t i = 0; i < n; ++i) q[i] = (s == 0.0f) ? 0 : or_e4m3_encode(x[i] / s);
    *s_out = s;
}

void or_quant_tokens(const uint16_t* x, int64_t T, int64_t H, uint8_t* q, float* s) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float* row = (float*)malloc((size_t)H * sizeof(float));
        for (int64_t i = 0; i < H; ++i) row[i] = or_bf16_to_f32(x[t * H + i]);
        quant_row_f32(row, H, q + t * H, s + t);
        free(row);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* NVFP4 ([P2] "Dequant math", reading R8)                                                      */
/* ------------------------------------------------------------------------------------------ */

static const float kE2M1[16] = {0.0f,  0.5f,  1.0f,  1.5f,  2.0f,  3.0f,  4.0f,  6.0f,
                                -0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};

float or_e2m1_decode(uint8_t c) { return kE2M1[c & 15]; }

/* Nearest E2M1 value by exhaustive comparison with the eight magnitudes; on a tie the even
 * code (lower code bit clear); above 6 the largest; the sign goes to code bit 3. */
uint8_t or_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 8 : 0;
    float a = fabsf(x);
    int best = 0;
    for (int i = 1; i < 8; ++i) {
        float di = fabsf(a - kE2M1[i]), db = fabsf(a - kE2M1[best]);
        if (di < db || (di == db && (i & 1) == 0)) best = i;
    }
    return (uint8_t)(sign | best);
}

/* NVFP4 quantization of one projection [rows, K] (reading R8): codes [rows, K/2] (element 2j
 * in the low nibble of byte j), E4M3 block scales [rows, K/16], fp32 scale2.  -1 on K % 16. */
int or_nvfp4_quant(const uint16_t* w, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales,
                   float* scale2) {
    if (K % 16) return -1;
    float amax = 0.0f;
    for (int64_t i = 0; i < rows * K; ++i) {
        float a = fabsf(or_bf16_to_f32(w[i]));
        if (a > amax) amax = a;
    }
    const float s2 = amax / 2688.0f;    /* 6 * 448 */
    *scale2 = s2;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < K / 16; ++b) {
            const uint16_t* wb = w + r * K + b * 16;
            float ab = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(or_bf16_to_f32(wb[i]));
                if (a > ab) ab = a;
            }
            uint8_t sc = (s2 == 0.0f) ? 0 : or_e4m3_encode(ab / (6.0f * s2));
            scales[r * (K / 16) + b] = sc;
            float d = or_e4m3_decode(sc) * s2;
            for (int i = 0; i < 16; ++i) {
                uint8_t c = (d == 0.0f) ? 0 : or_e2m1_encode(or_bf16_to_f32(wb[i]) / d);
                int64_t k = b * 16 + i;
                uint8_t* byte = codes + r * (K / 2) + k / 2;
                if ((k & 1) == 0) *byte = c;
                else *byte = (uint8_t)(*byte | (c << 4));
            }
        }
    }
    return 0;
}

/* Row-scaled FP8 weights ([P5], reading R7): one scale per row, same rule as a token row. */
void or_quant_rows(const uint16_t* w, int64_t rows, int64_t K, uint8_t* q, float* s) {
    or_quant_tokens(w, rows, K, q, s);
}

/* ------------------------------------------------------------------------------------------ */
/* Router (the step upstream of S2): logits[t][e] = sum over k of x[t][k] * wr[e][k] with the  */
/* router weight kept in its source bf16 precision ("Baekpica/Inkling-Small-Mixed-Quant-GGUF"  */
/* card, "Precision differences": router tensors stay native; [P2] "Layout summary": the gate */
/* is copied verbatim).  Reading R6: no bias, fp32 accumulation in increasing k; each product */
/* of two bf16 values is exact in fp32, so only the running sum rounds.                       */
/* ------------------------------------------------------------------------------------------ */

void or_router_logits(const uint16_t* x, const uint16_t* wr, int64_t T, int64_t H, int E,
                      float* logits) {
    for (int64_t t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int64_t k = 0; k < H; ++k)
                acc += or_bf16_to_f32(x[t * H + k]) * or_bf16_to_f32(wr[(int64_t)e * H + k]);
            logits[t * E + e] = acc;
        }
}

/* ------------------------------------------------------------------------------------------ */
/* S2: top-k routing with a softmax over the selected logits ([P2]: 256 experts, 6 active;      */
/* reading R3).                                                                                 */
/* ------------------------------------------------------------------------------------------ */

void or_route_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* gates) {
    char* taken = (char*)malloc((size_t)E);
    float* ex = (float*)malloc((size_t)k * sizeof(float));
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {          /* j-th largest; strict '>' keeps the lower index */
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
            taken[best] = 1;
            ids[t * k + j] = best;
        }
        float lmax = l[ids[t * k]];
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) {
            ex[j] = expf(l[ids[t * k + j]] - lmax);
            sum += ex[j];
        }
        for (int j = 0; j < k; ++j) gates[t * k + j] = ex[j] / sum;
    }
    free(taken);
    free(ex);
}

/* ------------------------------------------------------------------------------------------ */
/* S3: stable permutation of routed pairs p = t*k + j into per-expert segments.                 */
/* offsets = exclusive prefix sum of per-expert counts; within a segment pairs ascend in p.     */
/* ------------------------------------------------------------------------------------------ */

void or_permute(const int32_t* ids, int64_t T, int k, int E, int32_t* offsets,
                int32_t* sorted_pairs, int32_t* row_of_pair) {
    int64_t P = T * k;
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t p = 0; p < P; ++p) offsets[ids[p] + 1] += 1;
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    for (int64_t p = 0; p < P; ++p) {
        int e = ids[p];
        int32_t r = offsets[e] + fill[e]++;
        sorted_pairs[r] = (int32_t)p;
        row_of_pair[p] = r;
    }
    free(fill);
}

/* ------------------------------------------------------------------------------------------ */
/* S4..S8: the layer.                                                                           */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    int E, H, N, group;
    const int32_t *gate_packed, *up_packed, *down_packed;   /* [E,N,H/8], [E,N,H/8], [E,H,N/8] */
    const uint16_t *gate_scales, *up_scales, *down_scales;  /* bf16 [E,N,H/g], [E,N,H/g], [E,H,N/g] */
    int n_shared, shared_N;
    const uint16_t *sh_gate, *sh_up, *sh_down;              /* bf16 [S,Ns,H], [S,Ns,H], [S,H,Ns] */
    /* fmt 1 = row-scaled FP8 experts (reading R7): E4M3 codes and one fp32 scale per output row */
    int fmt;
    const uint8_t *gate_w8, *up_w8, *down_w8;               /* [E,N,H], [E,N,H], [E,H,N] */
    const float *gate_rs, *up_rs, *down_rs;                  /* [E,N], [E,N], [E,H] */
    /* fmt 2 = NVFP4 experts (readings R8, R9) */
    const uint8_t *gate_f4, *up_f4, *down_f4;               /* [E,N,H/2], [E,N,H/2], [E,H,N/2] */
    const uint8_t *gate_bs, *up_bs, *down_bs;               /* [E,N,H/16], [E,N,H/16], [E,H,N/16] */
    const float *gate_s2, *up_s2, *down_s2;                  /* [E] */
    /* fmt 3 = hybrid ([P2] "On-disk tensor format": hot experts NVFP4, the rest another format;
     * hot_ids / cold_ids give the routed expert of each slab and partition 0..E-1): hot slab i
     * is NVFP4 slab i of the fmt-2 arrays, cold slab j is W4A8 slab j of the fmt-0 arrays. */
    const int32_t *hot_ids, *cold_ids;
    int n_hot, n_cold;
} or_layer;

/* Format and slab of routed expert e: the layer's format with slab e, or for a hybrid layer
 * NVFP4 (2) with its hot slab or W4A8 (0) with its cold slab; -1 if e is in neither list. */
static int expert_fmt(const or_layer* L, int64_t e, int64_t* slab) {
    if (L->fmt != 3) {
        *slab = e;
        return L->fmt;
    }
    for (int i = 0; i < L->n_hot; ++i)
        if (L->hot_ids[i] == e) { *slab = i; return 2; }
    for (int j = 0; j < L->n_cold; ++j)
        if (L->cold_ids[j] == e) { *slab = j; return 0; }
    return -1;
}

/* Unpacked codes of one projection as floats, transposed to [K][rows] so that the
 * inner loop runs over independent outputs. */
static void codes_T(const int32_t* packed, int64_t rows, int64_t K, float* cT) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < K / 8; ++j) {
            uint32_t w;
            memcpy(&w, packed + r * (K / 8) + j, 4);
            for (int i = 0; i < 8; ++i)
                cT[(8 * j + i) * rows + r] = (float)((int)((w >> (4 * i)) & 15u) - 8);
        }
}

/* W4A8 projection of one FP8 row: for every output n,
 *   acc_n = sum_g scale[n,g] * ( sum_{k in g} dec(q_k) * code[n,k] ),   out_n = acc_n * s_x
 * (reading R5: k increasing inside a group, g increasing). */
static void w4a8_proj(const uint8_t* q, float s_x, const float* cT, const uint16_t* scales,
                      int64_t rows, int64_t K, int group, float* out, float* part, float* acc) {
    int64_t G = K / group;
    for (int64_t n = 0; n < rows; ++n) acc[n] = 0.0f;
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t n = 0; n < rows; ++n) part[n] = 0.0f;
        for (int64_t kk = g * group; kk < (g + 1) * group; ++kk) {
            float a = or_e4m3_decode(q[kk]);
            const float* c = cT + kk * rows;
            for (int64_t n = 0; n < rows; ++n) part[n] += a * c[n];
        }
        for (int64_t n = 0; n < rows; ++n) acc[n] += part[n] * or_bf16_to_f32(scales[n * G + g]);
    }
    for (int64_t n = 0; n < rows; ++n) out[n] = acc[n] * s_x;
}

/* Decoded E4M3 codes of one projection, transposed to [K][rows]. */
static void w8_T(const uint8_t* codes, int64_t rows, int64_t K, float* cT) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t kk = 0; kk < K; ++kk) cT[kk * rows + r] = or_e4m3_decode(codes[r * K + kk]);
}

/* Row-scaled FP8 projection of one FP8 row (reading R7): for every output n,
 *   acc_n = sum_k dec(q_k) * dec(w[n,k])  (k increasing),   out_n = acc_n * s_w[n] * s_x. */
static void w8a8_proj(const uint8_t* q, float s_x, const float* cT, const float* rs, int64_t rows,
                      int64_t K, float* out, float* acc) {
    for (int64_t n = 0; n < rows; ++n) acc[n] = 0.0f;
    for (int64_t kk = 0; kk < K; ++kk) {
        float a = or_e4m3_decode(q[kk]);
        const float* c = cT + kk * rows;
        for (int64_t n = 0; n < rows; ++n) acc[n] += a * c[n];
    }
    for (int64_t n = 0; n < rows; ++n) out[n] = acc[n] * rs[n] * s_x;
}

/* NVFP4 weights dequantized by the page's formula ([P2] "Dequant math"), transposed to [K][rows]:
 * W[r,k] = LUT[code] * dec(scale[r, k/16]) * scale2. */
static void f4_T(const uint8_t* codes, const uint8_t* scales, float s2, int64_t rows, int64_t K,
                 float* cT) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t kk = 0; kk < K; ++kk) {
            uint8_t c = (codes[r * (K / 2) + kk / 2] >> (4 * (kk & 1))) & 15;
            cT[kk * rows + r] = kE2M1[c] * or_e4m3_decode(scales[r * (K / 16) + kk / 16]) * s2;
        }
}

/* Projection of one FP8 row on dequantized weights (reading R9): for every output n,
 *   acc_n = sum_k dec(q_k) * W[n,k]  (k increasing),   out_n = acc_n * s_x. */
static void f4_proj(const uint8_t* q, float s_x, const float* cT, int64_t rows, int64_t K,
                    float* out, float* acc) {
    for (int64_t n = 0; n < rows; ++n) acc[n] = 0.0f;
    for (int64_t kk = 0; kk < K; ++kk) {
        float a = or_e4m3_decode(q[kk]);
        const float* c = cT + kk * rows;
        for (int64_t n = 0; n < rows; ++n) acc[n] += a * c[n];
    }
    for (int64_t n = 0; n < rows; ++n) out[n] = acc[n] * s_x;
}

static float silu_f32(float g) { return g * (1.0f / (1.0f + expf(-g))); }

/*
 * One routed row: token row q/s_x through expert weights (already unpacked), giving the
 * FP8 SwiGLU activations (hq, s_h) and the down-projection output y[H].  With given_h set
 * (or_moe_forward_given_h only) hq/s_h already hold the row's requantized SwiGLU activations
 * and only the down projection runs.
 */
static void expert_row(const uint8_t* q, float s_x, const float* cg, const float* cu,
                       const float* cd, const uint16_t* sg, const uint16_t* su, const uint16_t* sd,
                       int64_t H, int64_t N, int group, uint8_t* hq, float* s_h, float* y,
                       float* scratch, int given_h) {
    float* G = scratch;               /* N */
    float* U = G + N;                 /* N */
    float* h = U + N;                 /* N */
    float* part = h + N;              /* max(N,H) */
    float* acc = part + (H > N ? H : N);
    if (!given_h) {
        w4a8_proj(q, s_x, cg, sg, N, H, group, G, part, acc);
        w4a8_proj(q, s_x, cu, su, N, H, group, U, part, acc);
        for (int64_t n = 0; n < N; ++n) h[n] = silu_f32(G[n]) * U[n];
        quant_row_f32(h, N, hq, s_h);
    }
    w4a8_proj(hq, *s_h, cd, sd, H, N, group, y, part, acc);
}

/* expert_row for row-scaled FP8 experts (same steps, w8a8_proj for the three projections). */
static void expert_row_w8(const uint8_t* q, float s_x, const float* cg, const float* cu,
                          const float* cd, const float* rg, const float* ru, const float* rd,
                          int64_t H, int64_t N, uint8_t* hq, float* s_h, float* y, float* scratch,
                          int given_h) {
    float* G = scratch;
    float* U = G + N;
    float* h = U + N;
    float* acc = h + N;
    if (!given_h) {
        w8a8_proj(q, s_x, cg, rg, N, H, G, acc);
        w8a8_proj(q, s_x, cu, ru, N, H, U, acc);
        for (int64_t n = 0; n < N; ++n) h[n] = silu_f32(G[n]) * U[n];
        quant_row_f32(h, N, hq, s_h);
    }
    w8a8_proj(hq, *s_h, cd, rd, H, N, y, acc);
}

/* expert_row for NVFP4 experts (same steps, f4_proj for the three projections). */
static void expert_row_f4(const uint8_t* q, float s_x, const float* cg, const float* cu,
                          const float* cd, int64_t H, int64_t N, uint8_t* hq, float* s_h, float* y,
                          float* scratch, int given_h) {
    float* G = scratch;
    float* U = G + N;
    float* h = U + N;
    float* acc = h + N;
    if (!given_h) {
        f4_proj(q, s_x, cg, N, H, G, acc);
        f4_proj(q, s_x, cu, N, H, U, acc);
        for (int64_t n = 0; n < N; ++n) h[n] = silu_f32(G[n]) * U[n];
        quant_row_f32(h, N, hq, s_h);
    }
    f4_proj(hq, *s_h, cd, H, N, y, acc);
}

/* Shared expert in bf16 weights / fp32 arithmetic on the unquantized token row:
 * y += down( silu(Wg x) * (Wu x) ).  Sums run over the reduction index in increasing order. */
static void shared_expert_add(const float* x, const uint16_t* wg, const uint16_t* wu,
                              const uint16_t* wd, int64_t H, int64_t Ns, float* y, float* scratch) {
    float* a = scratch;
    for (int64_t n = 0; n < Ns; ++n) {
        float g = 0.0f, u = 0.0f;
        for (int64_t kk = 0; kk < H; ++kk) {
            g += x[kk] * or_bf16_to_f32(wg[n * H + kk]);
            u += x[kk] * or_bf16_to_f32(wu[n * H + kk]);
        }
        a[n] = silu_f32(g) * u;
    }
    for (int64_t m = 0; m < H; ++m) {
        float s = 0.0f;
        for (int64_t n = 0; n < Ns; ++n) s += a[n] * or_bf16_to_f32(wd[m * Ns + n]);
        y[m] = s;
    }
}

/*
 * S4..S6 for n routed rows of expert e: row i reads the FP8 codes q[i] (H of them) with scale
 * s_x[i], writes its requantized SwiGLU activations to hq[i N ..] / s_h[i] and its
 * down-projection output to y[i][0 .. H).  With given_h, hq / s_h are inputs.
 */
static void expert_segment(const or_layer* L, int64_t e, int64_t n, const uint8_t* const* q,
                           const float* s_x, uint8_t* hq, float* s_h, float* const* y, int given_h) {
    const int64_t H = L->H, N = L->N;
    const int group = L->group;
    const int64_t G_h = H / group, G_n = N / group;
    float* cg = (float*)malloc((size_t)N * H * 4);
    float* cu = (float*)malloc((size_t)N * H * 4);
    float* cd = (float*)malloc((size_t)H * N * 4);
    float* scratch = (float*)malloc((size_t)(3 * N + 2 * (H > N ? H : N)) * 4);
    int64_t b;                           /* the expert's slab in its format's arrays */
    const int f = expert_fmt(L, e, &b);
    if (f == 1) {
        w8_T(L->gate_w8 + b * N * H, N, H, cg);
        w8_T(L->up_w8 + b * N * H, N, H, cu);
        w8_T(L->down_w8 + b * H * N, H, N, cd);
    } else if (f == 2) {
        f4_T(L->gate_f4 + b * N * (H / 2), L->gate_bs + b * N * (H / 16), L->gate_s2[b], N, H, cg);
        f4_T(L->up_f4 + b * N * (H / 2), L->up_bs + b * N * (H / 16), L->up_s2[b], N, H, cu);
        f4_T(L->down_f4 + b * H * (N / 2), L->down_bs + b * H * (N / 16), L->down_s2[b], H, N, cd);
    } else {
        codes_T(L->gate_packed + b * N * (H / 8), N, H, cg);
        codes_T(L->up_packed + b * N * (H / 8), N, H, cu);
        codes_T(L->down_packed + b * H * (N / 8), H, N, cd);
    }
    for (int64_t i = 0; i < n; ++i) {
        if (f == 1)
            expert_row_w8(q[i], s_x[i], cg, cu, cd, L->gate_rs + b * N, L->up_rs + b * N,
                          L->down_rs + b * H, H, N, hq + i * N, s_h + i, y[i], scratch, given_h);
        else if (f == 2)
            expert_row_f4(q[i], s_x[i], cg, cu, cd, H, N, hq + i * N, s_h + i, y[i], scratch,
                          given_h);
        else
            expert_row(q[i], s_x[i], cg, cu, cd, L->gate_scales + b * N * G_h,
                       L->up_scales + b * N * G_h, L->down_scales + b * H * G_n, H, N, group,
                       hq + i * N, s_h + i, y[i], scratch, given_h);
    }
    free(cg); free(cu); free(cd); free(scratch);
}

/*
 * S7 (+ S8) for token t: out[t] = bf16( sum_j gate_j * y_j  +  sum_s shared_s(x_t) ), j in
 * selection order, y_j = yr[j] the output row of the token's j-th routed pair, accumulated in
 * fp32 in that order; the shared experts' sum is added last.
 */
static void combine_token(const or_layer* L, const uint16_t* x, int64_t t, int k,
                          const float* gates_t, const float* const* yr, uint16_t* out,
                          float* out_f32) {
    const int64_t H = L->H;
    float* o = (float*)malloc((size_t)H * 4);
    for (int64_t m = 0; m < H; ++m) o[m] = 0.0f;
    for (int j = 0; j < k; ++j) {
        float gj = gates_t[j];
        for (int64_t m = 0; m < H; ++m) o[m] += gj * yr[j][m];
    }
    if (L->n_shared > 0) {
        int64_t Ns = L->shared_N;
        float* xf = (float*)malloc((size_t)H * 4);
        float* ys = (float*)malloc((size_t)H * 4);
        float* a = (float*)malloc((size_t)Ns * 4);
        float* shsum = (float*)calloc((size_t)H, 4);
        for (int64_t i = 0; i < H; ++i) xf[i] = or_bf16_to_f32(x[t * H + i]);
        for (int s = 0; s < L->n_shared; ++s) {
            shared_expert_add(xf, L->sh_gate + s * Ns * H, L->sh_up + s * Ns * H,
                              L->sh_down + s * H * Ns, H, Ns, ys, a);
            for (int64_t m = 0; m < H; ++m) shsum[m] += ys[m];
        }
        for (int64_t m = 0; m < H; ++m) o[m] += shsum[m];
        free(xf); free(ys); free(a); free(shsum);
    }
    for (int64_t m = 0; m < H; ++m) {
        out[t * H + m] = or_f32_to_bf16(o[m]);
        if (out_f32) out_f32[t * H + m] = o[m];
    }
    free(o);
}

/*
 * The layer.  x bf16 [T,H], logits fp32 [T,E] -> out bf16 [T,H].
 * Optional intermediates (NULL to skip), all in expert-sorted row order r:
 *   ids/gates [T,k], offsets [E+1], sorted_pairs/row_of_pair [P], xq [T,H], s_x [T],
 *   hq [P,N], s_h [P], y [P,H] fp32, out_f32 [T,H] (sum before the bf16 rounding).
 * Returns 0, or -1 on a bad shape.
 */
static int moe_forward_impl(const or_layer* L, const uint16_t* x, const float* logits, int64_t T,
                            int k, uint16_t* out, int32_t* ids_o, float* gates_o, int32_t* offsets_o,
                            int32_t* sorted_o, int32_t* rop_o, uint8_t* xq_o, float* sx_o,
                            uint8_t* hq_o, float* sh_o, float* y_o, float* out_f32_o,
                            const uint8_t* hq_pairs, const float* sh_pairs);

int or_moe_forward(const or_layer* L, const uint16_t* x, const float* logits, int64_t T, int k,
                   uint16_t* out, int32_t* ids_o, float* gates_o, int32_t* offsets_o,
                   int32_t* sorted_o, int32_t* rop_o, uint8_t* xq_o, float* sx_o, uint8_t* hq_o,
                   float* sh_o, float* y_o, float* out_f32_o) {
    return moe_forward_impl(L, x, logits, T, k, out, ids_o, gates_o, offsets_o, sorted_o, rop_o, xq_o,
                            sx_o, hq_o, sh_o, y_o, out_f32_o, NULL, NULL);
}

/*
 * The layer with the requantized SwiGLU activations given (test infrastructure for the parity
 * rules): hq_pairs [T*k, N] and sh_pairs [T*k] in pair order p = t*k + j replace S5's result,
 * and the down projection (S6) and combine (S7, S8) run on them.  Lets a test evaluate the
 * oracle's output on another implementation's requantized codes, so that an output difference
 * caused by a permitted FP8 code difference can be told from one that is not.
 */
int or_moe_forward_given_h(const or_layer* L, const uint16_t* x, const float* logits, int64_t T,
                           int k, const uint8_t* hq_pairs, const float* sh_pairs, uint16_t* out,
                           float* out_f32_o) {
    if (!hq_pairs || !sh_pairs) return -1;
    return moe_forward_impl(L, x, logits, T, k, out, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                            NULL, NULL, NULL, out_f32_o, hq_pairs, sh_pairs);
}

/*
 * Expert parallelism, receive side: S4..S6 for R routed rows given as FP8 codes q [R,H] with
 * scales s_x [R] and experts expert [R] (indices into L) -> y [R,H] fp32.  The per-row
 * arithmetic of the layer (each expert is independent of the others), rows taken expert by
 * expert in increasing row order.  Returns -1 on a bad shape or an expert outside [0, E).
 */
int or_expert_rows(const or_layer* L, const uint8_t* q, const float* s_x, const int32_t* expert,
                   int64_t R, float* y) {
    const int64_t H = L->H, N = L->N, E = L->E;
    if (H % L->group || N % L->group) return -1;
    for (int64_t i = 0; i < R; ++i)
        if (expert[i] < 0 || expert[i] >= E) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < E; ++e) {
        int64_t n = 0;
        for (int64_t i = 0; i < R; ++i) n += expert[i] == e;
        if (n == 0) continue;
        const uint8_t** qr = (const uint8_t**)malloc((size_t)n * sizeof(void*));
        float* sr = (float*)malloc((size_t)n * 4);
        float** yr = (float**)malloc((size_t)n * sizeof(void*));
        uint8_t* hq = (uint8_t*)malloc((size_t)n * N);
        float* sh = (float*)malloc((size_t)n * 4);
        int64_t c = 0;
        for (int64_t i = 0; i < R; ++i) {
            if (expert[i] != e) continue;
            qr[c] = q + i * H;
            sr[c] = s_x[i];
            yr[c] = y + i * H;
            ++c;
        }
        expert_segment(L, e, n, qr, sr, hq, sh, yr, 0);
        free(qr); free(sr); free(yr); free(hq); free(sh);
    }
    return 0;
}

/*
 * S7 (+ S8) alone: out bf16 [T,H] from the routed rows y_pairs [T*k, H] fp32 in pair order
 * p = t*k + j, the gates [T,k] and (for the shared experts) x bf16 [T,H].  Same arithmetic as
 * the layer's combine.
 */
int or_combine(const or_layer* L, const uint16_t* x, const float* gates, const float* y_pairs,
               int64_t T, int k, uint16_t* out) {
    if (k < 1) return -1;
    const int64_t H = L->H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        const float** yr = (const float**)malloc((size_t)k * sizeof(void*));
        for (int j = 0; j < k; ++j) yr[j] = y_pairs + (t * k + j) * H;
        combine_token(L, x, t, k, gates + t * k, yr, out, NULL);
        free(yr);
    }
    return 0;
}

static int moe_forward_impl(const or_layer* L, const uint16_t* x, const float* logits, int64_t T,
                            int k, uint16_t* out, int32_t* ids_o, float* gates_o, int32_t* offsets_o,
                            int32_t* sorted_o, int32_t* rop_o, uint8_t* xq_o, float* sx_o,
                            uint8_t* hq_o, float* sh_o, float* y_o, float* out_f32_o,
                            const uint8_t* hq_pairs, const float* sh_pairs) {
    const int64_t H = L->H, N = L->N, E = L->E;
    const int group = L->group;
    if (H % group || N % group || k < 1 || k > E) return -1;
    if (L->fmt == 3)                     /* the hot and cold lists must cover every expert */
        for (int64_t e = 0; e < E; ++e) {
            int64_t b;
            if (expert_fmt(L, e, &b) < 0) return -1;
        }
    const int64_t P = T * k;
    const int given_h = hq_pairs != NULL;   /* S5's results given: only S6..S8 run */

    int32_t* ids = (int32_t*)malloc((size_t)(P > 0 ? P : 1) * 4);
    float* gates = (float*)malloc((size_t)(P > 0 ? P : 1) * 4);
    int32_t* offsets = (int32_t*)malloc((size_t)(E + 1) * 4);
    int32_t* sorted = (int32_t*)malloc((size_t)(P > 0 ? P : 1) * 4);
    int32_t* rop = (int32_t*)malloc((size_t)(P > 0 ? P : 1) * 4);
    uint8_t* xq = (uint8_t*)malloc((size_t)(T > 0 ? T : 1) * H);
    float* sx = (float*)malloc((size_t)(T > 0 ? T : 1) * 4);
    uint8_t* hq = (uint8_t*)malloc((size_t)(P > 0 ? P : 1) * N);
    float* sh = (float*)malloc((size_t)(P > 0 ? P : 1) * 4);
    float* y = (float*)malloc((size_t)(P > 0 ? P : 1) * H * 4);

    /* S1, S2, S3 */
    or_quant_tokens(x, T, H, xq, sx);
    or_route_topk(logits, T, (int)E, k, ids, gates);
    or_permute(ids, T, k, (int)E, offsets, sorted, rop);
    if (hq_pairs) {                      /* S5's result given, pair order -> sorted rows */
        for (int64_t pp = 0; pp < P; ++pp) {
            memcpy(hq + (int64_t)rop[pp] * N, hq_pairs + pp * N, (size_t)N);
            sh[rop[pp]] = sh_pairs[pp];
        }
    }

    /* S4..S6, one expert segment at a time (experts are independent) */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < E; ++e) {
        int32_t r0 = offsets[e], r1 = offsets[e + 1];
        if (r0 == r1) continue;
        const uint8_t** qr = (const uint8_t**)malloc((size_t)(r1 - r0) * sizeof(void*));
        float* sr = (float*)malloc((size_t)(r1 - r0) * 4);
        float** yr = (float**)malloc((size_t)(r1 - r0) * sizeof(void*));
        for (int32_t r = r0; r < r1; ++r) {
            int64_t t = sorted[r] / k;
            qr[r - r0] = xq + t * H;
            sr[r - r0] = sx[t];
            yr[r - r0] = y + (int64_t)r * H;
        }
        expert_segment(L, e, r1 - r0, qr, sr, hq + (int64_t)r0 * N, sh + r0, yr, given_h);
        free(qr); free(sr); free(yr);
    }

    /* S7 (+ S8) */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        const float** yr = (const float**)malloc((size_t)k * sizeof(void*));
        for (int j = 0; j < k; ++j) yr[j] = y + (int64_t)rop[t * k + j] * H;
        combine_token(L, x, t, k, gates + t * k, yr, out, out_f32_o);
        free(yr);
    }

    if (ids_o) memcpy(ids_o, ids, (size_t)P * 4);
    if (gates_o) memcpy(gates_o, gates, (size_t)P * 4);
    if (offsets_o) memcpy(offsets_o, offsets, (size_t)(E + 1) * 4);
    if (sorted_o) memcpy(sorted_o, sorted, (size_t)P * 4);
    if (rop_o) memcpy(rop_o, rop, (size_t)P * 4);
    if (xq_o) memcpy(xq_o, xq, (size_t)T * H);
    if (sx_o) memcpy(sx_o, sx, (size_t)T * 4);
    if (hq_o) memcpy(hq_o, hq, (size_t)P * N);
    if (sh_o) memcpy(sh_o, sh, (size_t)P * 4);
    if (y_o) memcpy(y_o, y, (size_t)P * H * 4);
    free(ids); free(gates); free(offsets); free(sorted); free(rop);
    free(xq); free(sx); free(hq); free(sh); free(y);
    return 0;
}

/*
 * Dense brute force of the same layer that never builds the permutation: every token runs
 * through every expert, and the expert outputs are combined with a dense gate vector that is
 * zero off the top-k, visiting the selected experts in selection order.  Per-(token, expert)
 * arithmetic is the same as above, so out/out_f32 must equal or_moe_forward bit for bit.
 * y_dense [T,E,H] and hq_dense [T,E,N] / sh_dense [T,E] receive every (token, expert) row.
 * Shared experts are left out here (they do not depend on routing).
 */
int or_moe_forward_dense(const or_layer* L, const uint16_t* x, const float* logits, int64_t T,
                         int k, uint16_t* out, float* out_f32, uint8_t* hq_dense,
                         float* sh_dense, float* y_dense) {
    const int64_t H = L->H, N = L->N, E = L->E;
    const int group = L->group;
    if (H % group || N % group || k < 1 || k > E) return -1;
    if (L->fmt == 3)                     /* the hot and cold lists must cover every expert */
        for (int64_t e = 0; e < E; ++e) {
            int64_t b;
            if (expert_fmt(L, e, &b) < 0) return -1;
        }
    uint8_t* xq = (uint8_t*)malloc((size_t)(T > 0 ? T : 1) * H);
    float* sx = (float*)malloc((size_t)(T > 0 ? T : 1) * 4);
    int32_t* ids = (int32_t*)malloc((size_t)(T * k > 0 ? T * k : 1) * 4);
    float* gates = (float*)malloc((size_t)(T * k > 0 ? T * k : 1) * 4);
    or_quant_tokens(x, T, H, xq, sx);
    or_route_topk(logits, T, (int)E, k, ids, gates);
    const int64_t G_h = H / group, G_n = N / group;
    float* cg = (float*)malloc((size_t)N * H * 4);
    float* cu = (float*)malloc((size_t)N * H * 4);
    float* cd = (float*)malloc((size_t)H * N * 4);
    float* scratch = (float*)malloc((size_t)(3 * N + 2 * (H > N ? H : N)) * 4);
    for (int64_t e = 0; e < E; ++e) {
        int64_t b;                       /* the expert's slab in its format's arrays */
        const int f = expert_fmt(L, e, &b);
        if (f == 1) {
            w8_T(L->gate_w8 + b * N * H, N, H, cg);
            w8_T(L->up_w8 + b * N * H, N, H, cu);
            w8_T(L->down_w8 + b * H * N, H, N, cd);
        } else if (f == 2) {
            f4_T(L->gate_f4 + b * N * (H / 2), L->gate_bs + b * N * (H / 16), L->gate_s2[b], N, H, cg);
            f4_T(L->up_f4 + b * N * (H / 2), L->up_bs + b * N * (H / 16), L->up_s2[b], N, H, cu);
            f4_T(L->down_f4 + b * H * (N / 2), L->down_bs + b * H * (N / 16), L->down_s2[b], H, N, cd);
        } else {
            codes_T(L->gate_packed + b * N * (H / 8), N, H, cg);
            codes_T(L->up_packed + b * N * (H / 8), N, H, cu);
            codes_T(L->down_packed + b * H * (N / 8), H, N, cd);
        }
        for (int64_t t = 0; t < T; ++t) {
            if (f == 1)
                expert_row_w8(xq + t * H, sx[t], cg, cu, cd, L->gate_rs + b * N, L->up_rs + b * N,
                              L->down_rs + b * H, H, N, hq_dense + (t * E + e) * N,
                              sh_dense + t * E + e, y_dense + (t * E + e) * H, scratch, 0);
            else if (f == 2)
                expert_row_f4(xq + t * H, sx[t], cg, cu, cd, H, N, hq_dense + (t * E + e) * N,
                              sh_dense + t * E + e, y_dense + (t * E + e) * H, scratch, 0);
            else
                expert_row(xq + t * H, sx[t], cg, cu, cd, L->gate_scales + b * N * G_h,
                           L->up_scales + b * N * G_h, L->down_scales + b * H * G_n, H, N, group,
                           hq_dense + (t * E + e) * N, sh_dense + t * E + e,
                           y_dense + (t * E + e) * H, scratch, 0);
        }
    }
    float* dense_gate = (float*)malloc((size_t)E * 4);
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) dense_gate[e] = 0.0f;
        for (int j = 0; j < k; ++j) dense_gate[ids[t * k + j]] = gates[t * k + j];
        for (int64_t m = 0; m < H; ++m) {
            float o = 0.0f;
            for (int j = 0; j < k; ++j) {
                int64_t e = ids[t * k + j];
                o += dense_gate[e] * y_dense[(t * E + e) * H + m];
            }
            out_f32[t * H + m] = o;
            out[t * H + m] = or_f32_to_bf16(o);
        }
    }
    free(dense_gate); free(xq); free(sx); free(ids); free(gates);
    free(cg); free(cu); free(cd); free(scratch);
    return 0;
}
