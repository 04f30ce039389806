/*
 * w8a16 -- INT8 weight-only linear layer (W8A16) of the w4a16 library, sm_100a.
 *
 * Y[M,N] (bf16) = X[M,K] (bf16) . W_hat^T,  W_hat[n,k] = q[n,k] * s[n]
 *
 * Operation: "Weight-Only Quantization and Mixed Precision", section 5 (the
 * INT8-weight / 16-bit-activation combination: half the weight bytes of BF16)
 * and section 8 (INT8 needs no grouping); "Weight-Only Quantisation", Notes
 * (weights in INT8 or INT4, activations and accumulation in higher
 * precision).  The pages give no INT8 formula; the quantiser here is
 * symmetric with one scale per output channel ("Quantization I: int8, int4,
 * the basics", Concept: a scale and no zero point), per row n in binary64:
 *   m = max_k |w[n][k]|; s = bf16_rne(m / 127)
 *   (if s == 0: s = bf16_rne(m); if still 0: s = 1)
 *   q = clamp(rint(w / s), -127, 127)   (ties to even)
 *
 * Conventions (status codes, alignment, streams, ownership, no allocation,
 * host-side validation, the device fault word) are those of w4a16.h.
 * Layouts: W fp32 [N][K]; qweight int8 [N][K]; scales bf16 bits [N];
 * X bf16 [M][K]; Y bf16 [M][N].  The linear layer needs K a multiple of 128.
 */
#ifndef W8A16_H
#define W8A16_H

#include "w4a16.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Quantise W (offline step) with the formula above.
 *   W          device, fp32 [N][K]            (read; K >= 1)
 *   qweight    device, int8 [N][K]            (written)
 *   scales     device, bf16 bits [N]          (written)
 *   dev_status device, one int32: cleared on the stream, then set to
 *              W4A16_ERR_NONFINITE if a row holds a NaN or infinity (that
 *              row's outputs are zero).  Read it after the stream completes.
 * Returns a host-side status (argument, device or launch errors only).
 */
W4A16_API int w8a16_quantize(const float* W, int64_t N, int64_t K, int8_t* qweight, uint16_t* scales,
                             int32_t* dev_status, void* stream);

/* W_hat = q * s rounded to BF16 (nearest, ties to even; the product is exact in
 * FP32) into W_hat, device bf16 bits [N][K]. */
W4A16_API int w8a16_dequant(const int8_t* qweight, const uint16_t* scales, int64_t N, int64_t K, uint16_t* W_hat,
                            void* stream);

/* Bytes of device workspace w8a16_linear() needs (0 for an invalid shape).  The
 * layout starts with the same 256 KB counter area as the w4a16 workspace, with
 * the same rules: zero before first use, left zero by every completed call, so
 * one workspace can serve both layers' calls ordered on one stream. */
W4A16_API size_t w8a16_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * The W8A16 linear layer: persistent split-K kernel reading the INT8 codes once
 * (TMA), exact integer dot products against X in three signed base-256 digits
 * per 128-K block (mma.sync s8 x s8), folded in FP32 per block; the row scale
 * multiplies each output once; Y rounded to BF16 once.  Tokens are processed two
 * per launch (consecutive launches for M > 2: decode-sized M is the intended use).
 *   X, qweight, scales, Y device as above; workspace device,
 *   >= w8a16_workspace_bytes(M, N, K) bytes.
 */
W4A16_API int w8a16_linear(const uint16_t* X, int64_t M, int64_t K, const int8_t* qweight, const uint16_t* scales,
                           int64_t N, uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* W8A16_H */
