/*
 * FP64 CPU oracle for the W4A16 weight-only linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library; the product path (the
 * CUDA library and its Python binding) never calls it and shares no code with
 * it.  It is deliberately plain and slow: one straightforward loop per step of
 * the method, every floating-point decision in binary64, rows spread over
 * OpenMP threads and nothing else.
 *
 * What it computes (source pages, by title and section):
 *  - "Axe Corsa 28B" model card, "How the Compression Works": asymmetric INT4,
 *    each group of 128 consecutive weights has its own scale and zero point,
 *    all 16 levels used; dequantisation w_hat = (q - z_g) * s_g with s_g a
 *    BF16 scale and z_g an INT32 zero point ("What the Tensor Types Tell You");
 *    activations stay BF16 and the dequantised weights feed the multiply.
 *  - "Quantization I: int8, int4, the basics", Concept: round to a scale, a
 *    zero point shifts the grid, clipping maps extremes to the boundary; the
 *    products accumulate in higher precision.
 *
 * The forward quantisation formula did not survive in the pages' text; the
 * reading implemented here is the plainest one the prose supports (min/max
 * affine):
 *   lo = min w, hi = max w over the group (FP32 compares)
 *   s  = bf16_rne((hi - lo) / 15)                (difference and quotient in binary64)
 *        if s == 0: s = bf16_rne(max(|lo|, |hi|)); if still 0: s = 1
 *   z  = rint(-lo / s)                            (ties to even, not clamped)
 *   q  = clamp(rint(w / s) + z, 0, 15)
 * using the stored BF16 scale for z and q so the stored parameters reproduce
 * the codes.  The symmetric variant (orc_quantize_pack_sym), the AWQ
 * equivalence transform (orc_awq_scale_*) and the INT8 per-channel weights of
 * W8A16 (orc_w8_*) are documented at their definitions.  Codes are packed 8 per uint32 word, lowest K index in the lowest
 * nibble.  Group index runs along K, per output row n.
 *
 * Parity status: quantise/pack/unpack/dequant (both variants) are pinned by
 * hand-worked groups, tie cases, grid round trips, brute force and invariants; the matmul by a library
 * FP64 matmul of the dequantised weights and one-hot/constant inputs; the
 * row renormalisation by its closed form (unit RMS) on tiny inputs; the AWQ
 * transform by exact power-of-two equivalence, the rounding bounds of its one
 * rounding per element, and the error reduction the pages claim for salient
 * channels.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_G 128 /* the format's group size; the _g entry points take 32, 64 or 128 */

enum {
    ORC_OK = 0,
    ORC_ERR_ARG = 1,
    ORC_ERR_SHAPE = 3,
    ORC_ERR_NONFINITE = 7,
    ORC_ERR_ZERO_RANGE = 8,
};

int orc_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* BF16 bit pattern -> value (exact). */
double orc_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Binary64 -> nearest BF16 (8 significant bits, exponent range of binary32,
 * ties to even), written from the definition: find the spacing of BF16 values
 * around |x|, round |x| / spacing to an integer, scale back. */
uint16_t orc_bf16_round(double x) {
    if (isnan(x)) return 0x7FC0;
    double a = fabs(x);
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    frexp(a, &e);              /* a = f 2^e, f in [0.5, 1): 2^(e-1) <= a < 2^e */
    int lead = e - 1;          /* exponent of the leading bit */
    if (lead < -126) lead = -126; /* below the normal range the spacing stays 2^-133 */
    double spacing = ldexp(1.0, lead - 7);
    double r = nearbyint(a / spacing) * spacing; /* a / spacing is exact (power of two) */
    if (r > 0x1.FEp127) return (uint16_t)(sign | 0x7F80); /* overflow past the largest BF16 */
    float rf = (float)r;       /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, 4);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFF));
}

/* Quantise one group of G weights (steps above).  Returns a status code. */
static int orc_quantize_group(const float* w, int64_t G, uint16_t* s_out, int32_t* z_out, uint8_t* q_out,
                              uint8_t* clipped) {
    float lo = w[0], hi = w[0];
    for (int64_t i = 0; i < G; ++i) {
        if (!isfinite(w[i])) return ORC_ERR_NONFINITE;
        if (w[i] < lo) lo = w[i];
        if (w[i] > hi) hi = w[i];
    }
    uint16_t sb = orc_bf16_round(((double)hi - (double)lo) / 15.0);
    if (orc_bf16_value(sb) == 0.0) {
        double m = fabs((double)lo) > fabs((double)hi) ? fabs((double)lo) : fabs((double)hi);
        sb = orc_bf16_round(m);
        if (orc_bf16_value(sb) == 0.0) sb = 0x3F80; /* 1.0 */
    }
    double s = orc_bf16_value(sb);
    double z = nearbyint(-(double)lo / s);
    if (z > 2147483647.0 || z < -2147483648.0) return ORC_ERR_ZERO_RANGE;
    for (int64_t i = 0; i < G; ++i) {
        double t = nearbyint((double)w[i] / s) + z;
        int clip = (t < 0.0) || (t > 15.0);
        if (t < 0.0) t = 0.0;
        if (t > 15.0) t = 15.0;
        q_out[i] = (uint8_t)t;
        if (clipped) clipped[i] = (uint8_t)clip;
    }
    *s_out = sb;
    *z_out = (int32_t)z;
    return ORC_OK;
}

/* Pack codes[N][K] (values 0..15) into qweight[N][K/8]: nibble i of word j
 * holds the code of k = 8j + i. */
void orc_pack_codes(const uint8_t* codes, int64_t N, int64_t K, uint32_t* qweight) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 8; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) word |= ((uint32_t)(codes[n * K + 8 * j + i] & 15u)) << (4 * i);
            qweight[n * (K / 8) + j] = word;
        }
}

/* Symmetric INT4 ("Quantization I: int8, int4, the basics", Concept: a real
 * value becomes an integer code through a scale alone; a zero point is what
 * the affine variants add).  The formula did not survive in the page's text;
 * the reading implemented is the plainest one for signed 4-bit codes:
 *   m = max |w| over the group; s = bf16_rne(m / 7)
 *       (if s == 0: s = bf16_rne(m); if still 0: s = 1)
 *   q = clamp(rint(w / s), -8, 7)
 * In the packed container the signed code q is the nibble q + 8 with the zero
 * point 8, so (nibble - z) * s = q * s and every consumer of the affine format
 * reads a symmetric weight unchanged. */
static int orc_quantize_group_sym(const float* w, int64_t G, uint16_t* s_out, int32_t* z_out, uint8_t* q_out,
                                  uint8_t* clipped) {
    double m = 0.0;
    for (int64_t i = 0; i < G; ++i) {
        if (!isfinite(w[i])) return ORC_ERR_NONFINITE;
        if (fabs((double)w[i]) > m) m = fabs((double)w[i]);
    }
    uint16_t sb = orc_bf16_round(m / 7.0);
    if (orc_bf16_value(sb) == 0.0) {
        sb = orc_bf16_round(m);
        if (orc_bf16_value(sb) == 0.0) sb = 0x3F80; /* 1.0 */
    }
    double s = orc_bf16_value(sb);
    for (int64_t i = 0; i < G; ++i) {
        double q = nearbyint((double)w[i] / s);
        int clip = (q < -8.0) || (q > 7.0);
        if (q < -8.0) q = -8.0;
        if (q > 7.0) q = 7.0;
        q_out[i] = (uint8_t)(q + 8.0);
        if (clipped) clipped[i] = (uint8_t)clip;
    }
    *s_out = sb;
    *z_out = 8;
    return ORC_OK;
}

typedef int (*orc_group_quantiser)(const float*, int64_t, uint16_t*, int32_t*, uint8_t*, uint8_t*);

/* Quantise every group of G consecutive weights of W with `quantise_group` and
 * pack the codes.  G = 128 is the format of the model card; 32 and 64 are the
 * smaller groups of "Quantization I: int8, int4, the basics", Concept (groups
 * of 32-128 values) and "Weight-Only Quantization and Mixed Precision",
 * section 8 (32/64/128), with the same per-group rule. */
static int orc_quantize_pack_groups(orc_group_quantiser quantise_group, const float* W, int64_t N, int64_t K,
                                    int64_t G, uint32_t* qweight, uint16_t* scales, int32_t* zeros,
                                    uint8_t* clipped) {
    if (!W || !qweight || !scales || !zeros || N < 1 || K < 1) return ORC_ERR_ARG;
    if (G != 32 && G != 64 && G != 128) return ORC_ERR_ARG;
    if (K % G) return ORC_ERR_SHAPE;
    const int64_t ng = K / G;
    int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t n = 0; n < N; ++n) {
        uint8_t q[ORC_G];
        for (int64_t g = 0; g < ng; ++g) {
            const float* w = W + n * K + g * G;
            uint8_t* cl = clipped ? clipped + n * K + g * G : NULL;
            int st = quantise_group(w, G, &scales[n * ng + g], &zeros[n * ng + g], q, cl);
            if (st != ORC_OK) {
#pragma omp critical
                { if (status == ORC_OK) status = st; }
                memset(q, 0, sizeof q);
                scales[n * ng + g] = 0;
                zeros[n * ng + g] = 0;
            }
            for (int j = 0; j < G / 8; ++j) {
                uint32_t word = 0;
                for (int i = 0; i < 8; ++i) word |= ((uint32_t)q[8 * j + i]) << (4 * i);
                qweight[n * (K / 8) + g * (G / 8) + j] = word;
            }
        }
    }
    return status;
}

/* W fp32 [N][K] -> qweight u32 [N][K/8], scales bf16 [N][K/128], zeros i32 [N][K/128].
 * clipped (nullable) u8 [N][K]: 1 where rint(w/s)+z fell outside [0, 15]. */
int orc_quantize_pack(const float* W, int64_t N, int64_t K, uint32_t* qweight, uint16_t* scales,
                      int32_t* zeros, uint8_t* clipped) {
    return orc_quantize_pack_groups(orc_quantize_group, W, N, K, ORC_G, qweight, scales, zeros, clipped);
}

/* Symmetric variant, same outputs; every zero point is 8.
 * clipped (nullable) u8 [N][K]: 1 where rint(w/s) fell outside [-8, 7]. */
int orc_quantize_pack_sym(const float* W, int64_t N, int64_t K, uint32_t* qweight, uint16_t* scales,
                          int32_t* zeros, uint8_t* clipped) {
    return orc_quantize_pack_groups(orc_quantize_group_sym, W, N, K, ORC_G, qweight, scales, zeros, clipped);
}

/* Either quantiser with groups of G in {32, 64, 128}; scales and zeros [N][K/G]. */
int orc_quantize_pack_g(const float* W, int64_t N, int64_t K, int64_t G, int symmetric, uint32_t* qweight,
                        uint16_t* scales, int32_t* zeros, uint8_t* clipped) {
    return orc_quantize_pack_groups(symmetric ? orc_quantize_group_sym : orc_quantize_group, W, N, K, G, qweight,
                                    scales, zeros, clipped);
}

/* AWQ equivalence transform ("Axe Corsa 28B" model card, "How the Compression
 * Works", Stage 1; "Weight-Only Quantization and Mixed Precision", section 3):
 * input channel k of the weight matrix is multiplied by s_k and the same
 * channel of the activations by s_k^-1, which leaves X W^T unchanged in exact
 * arithmetic while moving the salient channels onto a finer part of the
 * quantisation grid.  The scales are inputs here (the calibration that picks
 * them is not part of this layer).
 * W'[n][k] = w[n][k] * s[k], the exact binary64 product rounded once to binary32. */
void orc_awq_scale_weights(const float* W, const float* s, int64_t N, int64_t K, float* W_out) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) W_out[n * K + k] = (float)((double)W[n * K + k] * (double)s[k]);
}

/* X'[m][k] = x[m][k] * r[k] rounded once to BF16 (nearest, ties to even), with
 * r[k] the inverse scale as the caller stores it (binary32): the exact product
 * of a BF16 and a binary32 value fits binary64. */
void orc_awq_scale_activations(const uint16_t* X, const float* r, int64_t M, int64_t K, uint16_t* X_out) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) X_out[m * K + k] = orc_bf16_round(orc_bf16_value(X[m * K + k]) * (double)r[k]);
}

/* W8A16: INT8 weights against BF16 activations ("Weight-Only Quantization and
 * Mixed Precision", section 5, the INT8-weight / 16-bit-activation row of the
 * selection matrix, and section 8: INT8 needs no grouping; "Weight-Only
 * Quantisation", Notes: weights stored in INT8 or INT4, activations and
 * accumulation in higher precision).  The pages give no INT8 formula; the
 * reading implemented is symmetric per output channel ("Quantization I: int8,
 * int4, the basics", Concept: a scale and no zero point), per row n:
 *   m = max_k |w[n][k]|; s = bf16_rne(m / 127)
 *       (if s == 0: s = bf16_rne(m); if still 0: s = 1)
 *   q = clamp(rint(w / s), -127, 127)
 * and w_hat = q s.  clipped (nullable) u8 [N][K]: 1 where rint(w / s) fell
 * outside [-127, 127]. */
int orc_w8_quantize(const float* W, int64_t N, int64_t K, int8_t* q, uint16_t* scales, uint8_t* clipped) {
    if (!W || !q || !scales || N < 1 || K < 1) return ORC_ERR_ARG;
    int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        double m = 0.0;
        int finite = 1;
        for (int64_t k = 0; k < K; ++k) {
            if (!isfinite(w[k])) finite = 0;
            else if (fabs((double)w[k]) > m) m = fabs((double)w[k]);
        }
        if (!finite) {
#pragma omp critical
            { if (status == ORC_OK) status = ORC_ERR_NONFINITE; }
            memset(q + n * K, 0, (size_t)K);
            scales[n] = 0;
            continue;
        }
        uint16_t sb = orc_bf16_round(m / 127.0);
        if (orc_bf16_value(sb) == 0.0) {
            sb = orc_bf16_round(m);
            if (orc_bf16_value(sb) == 0.0) sb = 0x3F80; /* 1.0 */
        }
        const double sv = orc_bf16_value(sb);
        for (int64_t k = 0; k < K; ++k) {
            double t = nearbyint((double)w[k] / sv);
            int clip = (t < -127.0) || (t > 127.0);
            if (t < -127.0) t = -127.0;
            if (t > 127.0) t = 127.0;
            q[n * K + k] = (int8_t)t;
            if (clipped) clipped[n * K + k] = (uint8_t)clip;
        }
        scales[n] = sb;
    }
    return status;
}

/* Y[m][n] = sum_k x[m][k] * q[n][k] * s[n] in binary64 (unrounded); X is BF16
 * bits [M][K], q int8 [N][K], scales BF16 bits [N]. */
void orc_w8_linear(const uint16_t* X, int64_t M, int64_t K, const int8_t* q, const uint16_t* scales, int64_t N,
                   double* Y) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        const double sv = orc_bf16_value(scales[n]);
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += orc_bf16_value(X[m * K + k]) * ((double)q[n * K + k] * sv);
            Y[m * N + n] = acc;
        }
    }
}

/* qweight -> codes u8 [N][K]. */
void orc_unpack(const uint32_t* qweight, int64_t N, int64_t K, uint8_t* codes) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) codes[n * K + k] = (uint8_t)((qweight[n * (K / 8) + k / 8] >> (4 * (k % 8))) & 15u);
}

/* Exact dequantised weight of one element with groups of G: (q - z) * s, exact
 * in binary64. */
static double orc_w_hat_g(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t K,
                          int64_t G, int64_t n, int64_t k) {
    int64_t ng = K / G;
    uint32_t q = (qweight[n * (K / 8) + k / 8] >> (4 * (k % 8))) & 15u;
    int64_t g = k / G;
    return ((double)q - (double)zeros[n * ng + g]) * orc_bf16_value(scales[n * ng + g]);
}

static double orc_w_hat(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t K,
                        int64_t n, int64_t k) {
    return orc_w_hat_g(qweight, scales, zeros, K, ORC_G, n, k);
}

/* W_hat f64 [N][K]. */
void orc_dequant(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                 double* W_hat) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) W_hat[n * K + k] = orc_w_hat(qweight, scales, zeros, K, n, k);
}

/* W_hat f64 [N][K] with groups of G. */
void orc_dequant_g(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                   int64_t G, double* W_hat) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) W_hat[n * K + k] = orc_w_hat_g(qweight, scales, zeros, K, G, n, k);
}

/* Y_ref [M][N] in binary64 with groups of G: the sum of x * w_hat over k,
 * one group at a time. */
void orc_linear_g(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                  const int32_t* zeros, int64_t N, int64_t G, double* Y) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        double w[ORC_G];
        for (int64_t m = 0; m < M; ++m) Y[m * N + n] = 0.0;
        for (int64_t k0 = 0; k0 < K; k0 += G) {
            for (int64_t t = 0; t < G; ++t) w[t] = orc_w_hat_g(qweight, scales, zeros, K, G, n, k0 + t);
            for (int64_t m = 0; m < M; ++m) {
                const uint16_t* x = X + m * K + k0;
                double acc = 0.0;
                for (int64_t t = 0; t < G; ++t) acc += orc_bf16_value(x[t]) * w[t];
                Y[m * N + n] += acc;
            }
        }
    }
}

/* W_hat rounded to BF16 (nearest, ties to even) [N][K]. */
void orc_dequant_bf16(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t N,
                      int64_t K, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) out[n * K + k] = orc_bf16_round(orc_w_hat(qweight, scales, zeros, K, n, k));
}

/* Y_ref[i][j] = sum_k x[m_i][k] * w_hat[n_j][k] in binary64 (unrounded), for
 * the listed token rows m_i and output columns n_j.  X is BF16 bits [M][K]. */
void orc_linear_sampled(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                        const int32_t* zeros, int64_t N, const int64_t* m_idx, int64_t n_m, const int64_t* n_idx,
                        int64_t n_n, double* Y) {
    (void)M;
    (void)N;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t j = 0; j < n_n; ++j) {
        int64_t n = n_idx[j];
        double w[ORC_G];
        for (int64_t i = 0; i < n_m; ++i) Y[i * n_n + j] = 0.0;
        for (int64_t k0 = 0; k0 < K; k0 += ORC_G) {
            for (int64_t t = 0; t < ORC_G; ++t) w[t] = orc_w_hat(qweight, scales, zeros, K, n, k0 + t);
            for (int64_t i = 0; i < n_m; ++i) {
                const uint16_t* x = X + m_idx[i] * K + k0;
                double acc = 0.0;
                for (int64_t t = 0; t < ORC_G; ++t) acc += orc_bf16_value(x[t]) * w[t];
                Y[i * n_n + j] += acc;
            }
        }
    }
}

/* Full Y_ref [M][N] in binary64. */
void orc_linear(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                const int32_t* zeros, int64_t N, double* Y) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        double w[ORC_G];
        for (int64_t m = 0; m < M; ++m) Y[m * N + n] = 0.0;
        for (int64_t k0 = 0; k0 < K; k0 += ORC_G) {
            for (int64_t t = 0; t < ORC_G; ++t) w[t] = orc_w_hat(qweight, scales, zeros, K, n, k0 + t);
            for (int64_t m = 0; m < M; ++m) {
                const uint16_t* x = X + m * K + k0;
                double acc = 0.0;
                for (int64_t t = 0; t < ORC_G; ++t) acc += orc_bf16_value(x[t]) * w[t];
                Y[m * N + n] += acc;
            }
        }
    }
}

/* Row renormalisation between chained layers (the decode-stack workload):
 * out[m][:] = bf16_rne(y[m][:] / sqrt(mean_j y[m][j]^2)), y read as BF16
 * bits [M][N]; exact[m][j] (nullable) receives the unrounded quotient.
 * A zero row stays zero. */
void orc_renorm(const uint16_t* y, int64_t M, int64_t N, uint16_t* out, double* exact) {
    for (int64_t m = 0; m < M; ++m) {
        double ss = 0.0;
        for (int64_t j = 0; j < N; ++j) {
            double v = orc_bf16_value(y[m * N + j]);
            ss += v * v;
        }
        double rms = sqrt(ss / (double)N);
        for (int64_t j = 0; j < N; ++j) {
            double v = orc_bf16_value(y[m * N + j]);
            double r = rms > 0.0 ? v / rms : 0.0;
            if (exact) exact[m * N + j] = r;
            out[m * N + j] = orc_bf16_round(r);
        }
    }
}
