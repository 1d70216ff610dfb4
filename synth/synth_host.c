/*
 * synth_host.c — host filler for the seeded workload generator (see
 * synth_core.h for the definition of every value).  Built with
 * -ffp-contract=off so that its doubles match the device filler bit for bit.
 * OpenMP splits the element range; every element is a pure function of its
 * index, so the thread count never changes a value.
 */
#include <stdint.h>
#include <stddef.h>
#include "synth_core.h"

/* out[j] = bf16(fp32(sigma * z(start + j))), j < n. */
void syn_fill_normal_bf16(uint64_t seed, uint64_t stream, int64_t start, int64_t n,
                          double sigma, uint16_t* out) {
    uint64_t key = syn_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = syn_f32_to_bf16((float)(sigma * syn_normal(key, (uint64_t)(start + j))));
}

/* out[j] = fp32(sigma * z(start + j)), j < n. */
void syn_fill_normal_f32(uint64_t seed, uint64_t stream, int64_t start, int64_t n,
                         double sigma, float* out) {
    uint64_t key = syn_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (float)(sigma * syn_normal(key, (uint64_t)(start + j)));
}

/* Hidden states, rows [t0, t0+nt) of a [T, H] tensor: element (t, h) is
 * z(t*H + h), multiplied by `gain` on channels with mask[h] != 0 (mask may be
 * NULL), rounded to fp32 then bf16. */
void syn_fill_tokens_bf16(uint64_t seed, uint64_t stream, int64_t t0, int64_t nt, int64_t H,
                          const uint8_t* mask, double gain, uint16_t* out) {
    uint64_t key = syn_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nt * H; ++j) {
        int64_t h = j % H;
        double z = syn_normal(key, (uint64_t)(t0 * H + j));
        if (mask && mask[h]) z = z * gain;
        out[j] = syn_f32_to_bf16((float)z);
    }
}

/* Router logits, rows [t0, t0+nt) of a [T, E] tensor: element (t, e) is
 * fp32(z(t*E + e) + bias[e]) (bias may be NULL). */
void syn_fill_logits(uint64_t seed, uint64_t stream, int64_t t0, int64_t nt, int64_t E,
                     const double* bias, float* out) {
    uint64_t key = syn_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nt * E; ++j) {
        double z = syn_normal(key, (uint64_t)(t0 * E + j));
        if (bias) z = z + bias[j % E];
        out[j] = (float)z;
    }
}

/* Seeded Fisher–Yates shuffle of 0..n-1: for i = n-1 down to 1, swap
 * perm[i] with perm[draw(n-1-i) mod (i+1)]. */
void syn_permutation(uint64_t seed, uint64_t stream, int64_t n, int32_t* perm) {
    uint64_t key = syn_stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) perm[i] = (int32_t)i;
    for (int64_t i = n - 1; i >= 1; --i) {
        uint64_t d = syn_draw(key, (uint64_t)(n - 1 - i));
        int64_t j = (int64_t)(d % (uint64_t)(i + 1));
        int32_t tmp = perm[i];
        perm[i] = perm[j];
        perm[j] = tmp;
    }
}

/* Zipf prior on expert popularity: bias[e] = -s * ln(rank[e]), rank in 1..E. */
void syn_zipf_bias(const int32_t* rank, int64_t E, double s, double* bias) {
    for (int64_t e = 0; e < E; ++e) bias[e] = -s * syn_log((double)rank[e]);
}

/* Single values, for tests of the generator itself. */
double syn_normal_at(uint64_t seed, uint64_t stream, uint64_t i) {
    return syn_normal(syn_stream_key(seed, stream), i);
}
double syn_log_at(double x) { return syn_log(x); }
void syn_cossin_at(double u, double* c, double* s) { syn_cossin_2pi(u, c, s); }
