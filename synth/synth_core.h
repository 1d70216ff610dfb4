/*
 * synth_core.h — seeded, counter-based input generator for the W4A8 MoE
 * layer workloads.  Shared by the host filler (synth_host.c, used by the CPU
 * oracle, tests and bench) and the device filler (synth_dev.cu, used to build
 * full-size inputs in HBM).  It holds none of the layer's arithmetic: only
 * random draws, their transform to normals, and the rounding of a draw to the
 * storage type of the tensor it fills.
 *
 * Definition (every value is a pure function of (seed, stream, index)):
 *   - SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): the i-th 64-bit draw of
 *     stream `key` is mix64(key + (i + 1) * 0x9E3779B97F4A7C15).
 *   - key(seed, stream) = mix64(seed * 0x9E3779B97F4A7C15
 *                               + mix64(stream + 0x632BE59BD9B4E019)).
 *   - Box–Muller (1958): element 2j and 2j+1 of a normal stream come from draws
 *     2j and 2j+1: u1 = ((d0 >> 11) + 1) * 2^-53 in (0,1], u2 = (d1 >> 11) *
 *     2^-53 in [0,1), r = sqrt(-2 ln u1), z_{2j} = r cos(2 pi u2),
 *     z_{2j+1} = r sin(2 pi u2).
 *   - ln, cos and sin are evaluated here with argument reduction and truncated
 *     series in IEEE double using only +, -, *, / and sqrt (each correctly
 *     rounded), so the host build (gcc -ffp-contract=off) and the device build
 *     (nvcc -fmad=false) produce bit-identical values.  Their accuracy (~1e-15
 *     relative) only shapes the distribution; exactness to the true ln/cos is
 *     not needed.
 *   - A value is scaled in double, rounded once to fp32 (round to nearest
 *     even), and, for bf16 tensors, rounded from fp32 to bf16 (nearest even).
 */
#ifndef MOE_SYNTH_CORE_H
#define MOE_SYNTH_CORE_H

#include <stdint.h>
#include <math.h>

#ifdef __CUDACC__
#define SYN_FN __host__ __device__ static inline
#else
#define SYN_FN static inline
#endif

#define SYN_GAMMA 0x9E3779B97F4A7C15ULL

SYN_FN uint64_t syn_mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

SYN_FN uint64_t syn_stream_key(uint64_t seed, uint64_t stream) {
    return syn_mix64(seed * SYN_GAMMA + syn_mix64(stream + 0x632BE59BD9B4E019ULL));
}

SYN_FN uint64_t syn_draw(uint64_t key, uint64_t i) {
    return syn_mix64(key + (i + 1) * SYN_GAMMA);
}

typedef union { double d; uint64_t u; } syn_dbits;
typedef union { float f; uint32_t u; } syn_fbits;

/* Natural log of a positive, finite, normal double. */
SYN_FN double syn_log(double x) {
    syn_dbits b;
    b.d = x;
    int64_t e = (int64_t)((b.u >> 52) & 0x7FF) - 1023;
    b.u = (b.u & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL; /* m in [1,2) */
    double m = b.d;
    if (m > 1.4142135623730951) { m = m * 0.5; e += 1; }         /* m in [0.707,1.414] */
    double s = (m - 1.0) / (m + 1.0);
    double s2 = s * s;
    /* ln m = 2 atanh(s) = 2 (s + s^3/3 + s^5/5 + ...), |s| < 0.1716 */
    double p = 1.0 / 23.0;
    p = p * s2 + 1.0 / 21.0;
    p = p * s2 + 1.0 / 19.0;
    p = p * s2 + 1.0 / 17.0;
    p = p * s2 + 1.0 / 15.0;
    p = p * s2 + 1.0 / 13.0;
    p = p * s2 + 1.0 / 11.0;
    p = p * s2 + 1.0 / 9.0;
    p = p * s2 + 1.0 / 7.0;
    p = p * s2 + 1.0 / 5.0;
    p = p * s2 + 1.0 / 3.0;
    p = p * s2 + 1.0;
    double lnm = 2.0 * s * p;
    return (double)e * 0.69314718055994530942 + lnm;
}

/* cos and sin of 2*pi*u for u in [0,1). */
SYN_FN void syn_cossin_2pi(double u, double* c, double* s) {
    double v = 4.0 * u;              /* quarter turns, exact */
    int q = (int)(v + 0.5);          /* nearest quadrant 0..4 */
    double f = v - (double)q;        /* in [-0.5, 0.5] */
    double a = f * 1.5707963267948966;
    double a2 = a * a;
    /* Taylor series on |a| <= pi/4 */
    double sp = -1.0 / 1307674368000.0;          /* -1/15! */
    sp = sp * a2 + 1.0 / 6227020800.0;           /*  1/13! */
    sp = sp * a2 - 1.0 / 39916800.0;             /* -1/11! */
    sp = sp * a2 + 1.0 / 362880.0;               /*  1/9!  */
    sp = sp * a2 - 1.0 / 5040.0;                 /* -1/7!  */
    sp = sp * a2 + 1.0 / 120.0;                  /*  1/5!  */
    sp = sp * a2 - 1.0 / 6.0;                    /* -1/3!  */
    double sa = a + a * a2 * sp;
    double cp = 1.0 / 20922789888000.0;          /*  1/16! */
    cp = cp * a2 - 1.0 / 87178291200.0;          /* -1/14! */
    cp = cp * a2 + 1.0 / 479001600.0;            /*  1/12! */
    cp = cp * a2 - 1.0 / 3628800.0;              /* -1/10! */
    cp = cp * a2 + 1.0 / 40320.0;                /*  1/8!  */
    cp = cp * a2 - 1.0 / 720.0;                  /* -1/6!  */
    cp = cp * a2 + 1.0 / 24.0;                   /*  1/4!  */
    cp = cp * a2 - 0.5;                          /* -1/2!  */
    double ca = 1.0 + a2 * cp;
    switch (q & 3) {
        case 0: *c = ca;  *s = sa;  break;
        case 1: *c = -sa; *s = ca;  break;
        case 2: *c = -ca; *s = -sa; break;
        default: *c = sa; *s = -ca; break;
    }
}

/* Element i of the standard-normal stream `key`. */
SYN_FN double syn_normal(uint64_t key, uint64_t i) {
    uint64_t j = i >> 1;
    uint64_t d0 = syn_draw(key, 2 * j);
    uint64_t d1 = syn_draw(key, 2 * j + 1);
    double u1 = ((double)(d0 >> 11) + 1.0) * 1.1102230246251565e-16; /* 2^-53 */
    double u2 = (double)(d1 >> 11) * 1.1102230246251565e-16;
    double r = sqrt(-2.0 * syn_log(u1));
    double c, s;
    syn_cossin_2pi(u2, &c, &s);
    return (i & 1) ? r * s : r * c;
}

/* fp32 -> bf16, round to nearest even; the generator makes no NaN or inf. */
SYN_FN uint16_t syn_f32_to_bf16(float f) {
    syn_fbits b;
    b.f = f;
    uint32_t lsb = (b.u >> 16) & 1u;
    return (uint16_t)((b.u + 0x7FFFu + lsb) >> 16);
}

#endif /* MOE_SYNTH_CORE_H */
