/*
 * Counter-based normal generator shared by the host (synth.c) and device
 * (synth_dev.cu) input generators.  Input generation only: nothing here
 * quantises, packs or multiplies.
 *
 *   mix(z)      SplitMix64 output function (Steele, Lea & Flood, "Fast splittable
 *               pseudorandom number generators", OOPSLA 2014).
 *   key(s, t)   mix(mix(s * PHI + 1) ^ (t * 0xD1B54A32D192ED03)),  PHI = 0x9E3779B97F4A7C15
 *   draw(k, i)  mix(k + (i + 1) * PHI)
 *   normal(k,i) Box-Muller (Box & Muller, 1958) on u1 = ((draw(k,2i) >> 11) + 1) 2^-53 in (0,1]
 *               and u2 = (draw(k,2i+1) >> 11) 2^-53 in [0,1):
 *               sqrt(-2 ln u1) * cos(2 pi u2)
 *
 * ln and cos are evaluated with fixed-order series using only IEEE-754
 * +, -, *, / and sqrt in binary64, so both compilers produce the same bits as
 * long as no multiply-add is fused (host: -ffp-contract=off; device:
 * -fmad=false).  Coefficients are written as hexadecimal literals.
 */
#ifndef SYNTH_CORE_H
#define SYNTH_CORE_H
#include <math.h>
#include <stdint.h>

#if defined(__CUDACC__)
#define SYN_FN static __host__ __device__ __forceinline__
#else
#define SYN_FN static inline
#endif

#define SYN_PHI 0x9E3779B97F4A7C15ull

SYN_FN uint64_t syn_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

SYN_FN uint64_t syn_key(uint64_t seed, uint64_t tag) {
    return syn_mix(syn_mix(seed * SYN_PHI + 1ull) ^ (tag * 0xD1B54A32D192ED03ull));
}

SYN_FN uint64_t syn_draw(uint64_t key, uint64_t i) { return syn_mix(key + (i + 1ull) * SYN_PHI); }

SYN_FN double syn_bits_to_double(uint64_t b) {
    union { uint64_t u; double d; } v;
    v.u = b;
    return v.d;
}

SYN_FN uint64_t syn_double_to_bits(double d) {
    union { uint64_t u; double d; } v;
    v.d = d;
    return v.u;
}

/* ln u for u a positive normal double: u = m 2^e, m in [sqrt(1/2), sqrt(2)],
 * ln m = 2 atanh t with t = (m - 1)/(m + 1), |t| <= 0.1716; the atanh series
 * is cut after t^21 (remainder below 2^-55 relative). */
SYN_FN double syn_ln(double u) {
    uint64_t b = syn_double_to_bits(u);
    int e = (int)((b >> 52) & 0x7FF) - 1023;
    double m = syn_bits_to_double((b & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull);
    if (m > 0x1.6a09e667f3bcdp+0) { m = m * 0.5; e += 1; }
    double t = (m - 1.0) / (m + 1.0);
    double t2 = t * t;
    double p = 0x1.8618618618618p-5;       /* 1/21 */
    p = p * t2 + 0x1.af286bca1af28p-5;     /* 1/19 */
    p = p * t2 + 0x1.e1e1e1e1e1e1ep-5;     /* 1/17 */
    p = p * t2 + 0x1.1111111111111p-4;     /* 1/15 */
    p = p * t2 + 0x1.3b13b13b13b14p-4;     /* 1/13 */
    p = p * t2 + 0x1.745d1745d1746p-4;     /* 1/11 */
    p = p * t2 + 0x1.c71c71c71c71cp-4;     /* 1/9 */
    p = p * t2 + 0x1.2492492492492p-3;     /* 1/7 */
    p = p * t2 + 0x1.999999999999ap-3;     /* 1/5 */
    p = p * t2 + 0x1.5555555555555p-2;     /* 1/3 */
    p = p * t2 + 1.0;
    return 2.0 * t * p + (double)e * 0x1.62e42fefa39efp-1; /* + e ln 2 */
}

/* sin and cos of th in [0, pi/4] by Taylor series to th^17 / th^18. */
SYN_FN void syn_sincos_small(double th, double* s, double* c) {
    double t2 = th * th;
    /* sin th = th - th t2 (1/3! - t2/5! + t2^2/7! - ... - t2^7/17!) */
    double ps = -0x1.952c77030ad4ap-49;    /* -1/17! */
    ps = ps * t2 + 0x1.ae7f3e733b81fp-41;  /* 1/15! */
    ps = ps * t2 - 0x1.6124613a86d09p-33;  /* 1/13! */
    ps = ps * t2 + 0x1.ae64567f544e4p-26;  /* 1/11! */
    ps = ps * t2 - 0x1.71de3a556c734p-19;  /* 1/9! */
    ps = ps * t2 + 0x1.a01a01a01a01ap-13;  /* 1/7! */
    ps = ps * t2 - 0x1.1111111111111p-7;   /* 1/5! */
    ps = ps * t2 + 0x1.5555555555555p-3;   /* 1/3! */
    /* cos th = 1 - t2 (1/2! - t2/4! + t2^2/6! - ... + t2^8/18!) */
    double pc = 0x1.6827863b97d97p-53;     /* 1/18! */
    pc = pc * t2 - 0x1.ae7f3e733b81fp-45;  /* 1/16! */
    pc = pc * t2 + 0x1.93974a8c07c9dp-37;  /* 1/14! */
    pc = pc * t2 - 0x1.1eed8eff8d898p-29;  /* 1/12! */
    pc = pc * t2 + 0x1.27e4fb7789f5cp-22;  /* 1/10! */
    pc = pc * t2 - 0x1.a01a01a01a01ap-16;  /* 1/8! */
    pc = pc * t2 + 0x1.6c16c16c16c17p-10;  /* 1/6! */
    pc = pc * t2 - 0x1.5555555555555p-5;   /* 1/4! */
    pc = pc * t2 + 0.5;                    /* 1/2! */
    *s = th - th * t2 * ps;
    *c = 1.0 - t2 * pc;
}

/* cos(2 pi u), u in [0, 1): quadrant from 4u (exact), reflection into [0, pi/4]. */
SYN_FN double syn_cos2pi(double u) {
    double v = u * 4.0;
    int q = (int)v;
    double f = v - (double)q;
    double s, c;
    if (f > 0.5) {
        double s2, c2;
        syn_sincos_small((1.0 - f) * 0x1.921fb54442d18p+0, &s2, &c2);
        s = c2;
        c = s2;
    } else {
        syn_sincos_small(f * 0x1.921fb54442d18p+0, &s, &c);
    }
    switch (q & 3) {
        case 0: return c;
        case 1: return -s;
        case 2: return -c;
        default: return s;
    }
}

/* One standard normal per counter i (the cosine branch of Box-Muller). */
SYN_FN double syn_normal(uint64_t key, uint64_t i) {
    uint64_t d1 = syn_draw(key, 2ull * i);
    uint64_t d2 = syn_draw(key, 2ull * i + 1ull);
    double u1 = (double)((d1 >> 11) + 1ull) * 0x1.0p-53;
    double u2 = (double)(d2 >> 11) * 0x1.0p-53;
    return sqrt(-2.0 * syn_ln(u1)) * syn_cos2pi(u2);
}

#endif /* SYNTH_CORE_H */
