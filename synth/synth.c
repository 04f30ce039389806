/*
 * Seeded synthetic inputs for the W4A16 linear layer (host side).
 *
 * Draws the inputs only: FP32 weights W ~ N(0, sigma) and BF16 activations
 * X ~ N(0, 1) with a small set of salient input channels scaled up.  Nothing
 * here quantises, packs or multiplies; the CUDA library's tests and the FP64
 * oracle both consume what it produces.  The generator itself (counter-based
 * SplitMix64 + Box-Muller) is defined in synth_core.h, shared bit for bit with
 * the device filler in synth_dev.cu.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (a fused multiply-add
 * would change the bits).
 */
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include "synth_core.h"

uint64_t synth_key(uint64_t seed, uint64_t tag) { return syn_key(seed, tag); }
uint64_t synth_draw(uint64_t key, uint64_t i) { return syn_draw(key, i); }
double synth_ln(double u) { return syn_ln(u); }
double synth_cos2pi(double u) { return syn_cos2pi(u); }
double synth_normal(uint64_t key, uint64_t i) { return syn_normal(key, i); }

/* out[i] = (float)(sigma * normal(key(seed, tag), offset + i)), i in [0, count). */
void synth_fill_normal_f32(uint64_t seed, uint64_t tag, uint64_t offset, int64_t count, double sigma,
                           float* out) {
    uint64_t key = syn_key(seed, tag);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = (float)(sigma * syn_normal(key, offset + (uint64_t)i));
}

/* Selected rows of a row-major [*, cols] matrix drawn as above:
 * out[r][j] = (float)(sigma * normal(key, rows[r] * cols + j)). */
void synth_fill_normal_rows_f32(uint64_t seed, uint64_t tag, int64_t cols, const int64_t* rows,
                                int64_t n_rows, double sigma, float* out) {
    uint64_t key = syn_key(seed, tag);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int64_t j = 0; j < cols; ++j)
            out[r * cols + j] =
                (float)(sigma * syn_normal(key, (uint64_t)rows[r] * (uint64_t)cols + (uint64_t)j));
}

/* Binary64 value to BF16 bits, round to nearest, ties to even (formats the
 * activations; saturates to infinity past the largest finite BF16). */
uint16_t synth_bf16_bits(double x) {
    uint64_t b = syn_double_to_bits(x);
    uint64_t sign = b >> 63;
    uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
    uint16_t r;
    if (mag == 0) {
        r = 0;
    } else if (mag >= 0x7FF0000000000000ull) {
        r = (uint16_t)(mag > 0x7FF0000000000000ull ? 0x7FC0 : 0x7F80);
    } else if (syn_bits_to_double(mag) < 0x1.0p-126) {
        /* BF16 subnormals are the multiples of 2^-133 */
        r = (uint16_t)nearbyint(syn_bits_to_double(mag) * 0x1.0p133);
    } else {
        /* keep 8 significant bits: round the 52-bit fraction at bit 45 */
        uint64_t keep = mag >> 45;
        uint64_t rest = mag & ((1ull << 45) - 1ull);
        uint64_t half = 1ull << 44;
        if (rest > half || (rest == half && (keep & 1ull))) keep += 1ull;
        int64_t e16 = (int64_t)(keep >> 7) - 1023 + 127;
        r = (e16 >= 255) ? (uint16_t)0x7F80 : (uint16_t)(((uint64_t)e16 << 7) | (keep & 0x7Full));
    }
    return (uint16_t)((sign << 15) | r);
}

/* Salient input channels: a partial Fisher-Yates shuffle of [0, K) with draws
 * from key(seed, tag); channels[0..n_out) are the first n_out shuffled entries. */
void synth_outlier_channels(uint64_t seed, uint64_t tag, int64_t K, int64_t n_out, int64_t* channels,
                            int64_t* scratch_perm) {
    uint64_t key = syn_key(seed, tag);
    for (int64_t i = 0; i < K; ++i) scratch_perm[i] = i;
    for (int64_t i = 0; i < n_out; ++i) {
        uint64_t span = (uint64_t)(K - i);
        int64_t j = i + (int64_t)(syn_draw(key, (uint64_t)i) % span);
        int64_t t = scratch_perm[i];
        scratch_perm[i] = scratch_perm[j];
        scratch_perm[j] = t;
        channels[i] = scratch_perm[i];
    }
}

/* X[m][k] = bf16(normal(key(seed, tag), m K + k) * (k salient ? mult : 1)). */
void synth_fill_activations_bf16(uint64_t seed, uint64_t tag, int64_t M, int64_t K, const int64_t* channels,
                                 int64_t n_out, double mult, uint16_t* X, uint8_t* scratch_flags) {
    uint64_t key = syn_key(seed, tag);
    memset(scratch_flags, 0, (size_t)K);
    for (int64_t i = 0; i < n_out; ++i) scratch_flags[channels[i]] = 1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double z = syn_normal(key, (uint64_t)(m * K + k));
            X[m * K + k] = synth_bf16_bits(scratch_flags[k] ? z * mult : z);
        }
}

int synth_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
