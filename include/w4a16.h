/*
 * w4a16 -- weight-only INT4 linear layer for NVIDIA B200 (sm_100a).
 *
 * Y[M,N] (bf16) = X[M,K] (bf16) . W_hat^T,  W_hat[n,k] = (q[n,k] - z[n,g]) * s[n,g],  g = k / 128
 *
 * Operation: "Axe Corsa 28B" model card, "How the Compression Works"
 * (asymmetric INT4, one scale and one zero point per group of 128
 * consecutive weights, dequantisation w_hat = (q - z_g) * s_g inside the
 * matrix multiply, BF16 activations never quantised) and "What the Tensor
 * Types Tell You" (BF16 scales, INT32 zero points, two codes per byte);
 * "Quantization I: int8, int4, the basics", Concept (dequantise tile by tile
 * inside the multiply so only the packed codes cross the memory bus;
 * accumulate in higher precision -- FP32 here).
 *
 * Conventions for every entry point
 *  - All tensors are row-major and contiguous.  Element types are given by
 *    the pointer types; BF16 values are passed as their 16-bit patterns
 *    (uint16_t).
 *  - Layouts: W fp32 [N][K]; qweight uint32 [N][K/8] with the code of
 *    k = 8j + i in bits 4i..4i+3 of word j (lowest K index in the lowest
 *    nibble); scales bf16 [N][K/128]; zeros int32 [N][K/128]; X bf16 [M][K];
 *    Y bf16 [M][N].  K must be a multiple of 128; M, N >= 1.
 *  - Pointers named "device" are CUDA device pointers owned by the caller;
 *    the library keeps no reference after the call returns and allocates no
 *    device memory.  Every base pointer must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    asynchronous on that stream; nothing synchronises the host.
 *  - Arguments are validated on the host before any launch; a failed check
 *    returns a status code and launches nothing.  Errors raised by the CUDA
 *    runtime at launch map to W4A16_ERR_CUDA.  The device must be sm_100
 *    (checked once per device, cached).
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4A16_GROUP 128

#if defined(__GNUC__)
#define W4A16_API __attribute__((visibility("default")))
#else
#define W4A16_API
#endif

typedef enum {
    W4A16_OK = 0,
    W4A16_ERR_ARG = 1,        /* null pointer, negative or zero size, unknown option */
    W4A16_ERR_ALIGN = 2,      /* a base pointer is not 16-byte aligned */
    W4A16_ERR_SHAPE = 3,      /* K not a multiple of 128, or a size beyond the supported range */
    W4A16_ERR_DEVICE = 4,     /* no CUDA device, or the current device is not sm_100 */
    W4A16_ERR_WORKSPACE = 5,  /* workspace missing or smaller than w4a16_workspace_bytes() */
    W4A16_ERR_CUDA = 6,       /* the CUDA runtime reported an error at launch */
    W4A16_ERR_NONFINITE = 7,  /* (device status word) a weight group holds NaN or Inf */
    W4A16_ERR_ZERO_RANGE = 8  /* (device status word) a zero point does not fit in int32 */
} w4a16_status;

/* Kernel family selection for w4a16_linear_path(). */
typedef enum {
    W4A16_PATH_AUTO = 0,    /* decode GEMV for small M, tensor-core GEMM for large M */
    W4A16_PATH_DECODE = 1,  /* split-K GEMVs, any M: integer mma.sync (codes x digit planes of X) for
                               M <= 16 when K / 128 is a multiple of 8, tcgen05 (8-bit, codes from tensor
                               memory) otherwise, in chunks of 32 tokens */
    W4A16_PATH_PREFILL = 2  /* TMA + tcgen05/TMEM GEMM on BF16 tiles dequantised in shared memory */
} w4a16_path;

/* Static, NUL-terminated description of a status code (never NULL). */
W4A16_API const char* w4a16_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
W4A16_API int w4a16_version(void);

/*
 * Quantise and pack (offline step; "Axe Corsa 28B" model card, "How the
 * Compression Works": each group of 128 consecutive weights along K gets a
 * scale and a zero point, asymmetric, all 16 levels used).  Per row n and
 * group g, in binary64:
 *   lo, hi = min, max of the group; s = bf16_rne((hi - lo) / 15)
 *   (if s == 0: s = bf16_rne(max(|lo|, |hi|)); if still 0: s = 1)
 *   z = rint(-lo / s) (ties to even, not clamped); q = clamp(rint(w / s) + z, 0, 15)
 * The stored BF16 scale is the one used for z and q.
 *   W          device, fp32 [N][K]                       (read)
 *   qweight    device, uint32 [N][K/8]                    (written)
 *   scales     device, bf16 bits [N][K/128]               (written)
 *   zeros      device, int32 [N][K/128]                   (written)
 *   dev_status device, one int32                          (written: cleared on the stream, then
 *              set to W4A16_ERR_NONFINITE / W4A16_ERR_ZERO_RANGE if a group fails; the failing
 *              group's outputs are unspecified).  Read it after the stream completes.
 * Returns a host-side status (argument, device or launch errors only).
 */
W4A16_API int w4a16_quantize_pack(const float* W, int64_t N, int64_t K, uint32_t* qweight, uint16_t* scales,
                        int32_t* zeros, int32_t* dev_status, void* stream);

/*
 * Symmetric INT4 quantise and pack ("Quantization I: int8, int4, the basics",
 * Concept: a real value maps to an integer code through a scale alone, with
 * no zero point).  The page's formula did not survive extraction; the reading
 * implemented, per row n and group g of 128 along K, in binary64:
 *   m = max |w| over the group; s = bf16_rne(m / 7)
 *   (if s == 0: s = bf16_rne(m); if still 0: s = 1)
 *   q = clamp(rint(w / s), -8, 7)   (ties to even; BF16 rounding of s keeps
 *                                    |w / s| < 7.5, so nothing clips)
 * The signed code is stored as the nibble q + 8 and every zero point is 8, so
 * the result is an ordinary packed weight: (nibble - z) * s = q * s, and
 * w4a16_linear, w4a16_dequant and the other consumers take it unchanged.
 * Arguments, layouts, ownership and errors as for w4a16_quantize_pack
 * (W4A16_ERR_ZERO_RANGE cannot occur).
 */
W4A16_API int w4a16_quantize_pack_sym(const float* W, int64_t N, int64_t K, uint32_t* qweight, uint16_t* scales,
                            int32_t* zeros, int32_t* dev_status, void* stream);

/*
 * Quantisation groups of 32 or 64 weights ("Quantization I: int8, int4, the
 * basics", Concept: groups of 32-128 values, finer fit for more metadata;
 * "Weight-Only Quantization and Mixed Precision", section 8: group size
 * 32/64/128).  The rule per group is the one above (symmetric != 0: the
 * symmetric rule of w4a16_quantize_pack_sym); codes are packed as for groups of
 * 128; scales and zeros are [N][K/group].  group = 128 is w4a16_quantize_pack /
 * w4a16_quantize_pack_sym.  K must be a multiple of 128; other arguments and
 * errors as w4a16_quantize_pack (W4A16_ERR_ARG for another group size).
 */
W4A16_API int w4a16_quantize_pack_g(const float* W, int64_t N, int64_t K, int group, int symmetric, uint32_t* qweight,
                          uint16_t* scales, int32_t* zeros, int32_t* dev_status, void* stream);

/* Workspace bytes of w4a16_linear_g (0 for an invalid shape or group). */
W4A16_API size_t w4a16_workspace_bytes_g(int64_t M, int64_t N, int64_t K, int group);

/*
 * The linear layer on weights packed with groups of `group` (32, 64 or 128;
 * 128 is w4a16_linear).  For 32 and 64, K a multiple of 512 (W4A16_ERR_SHAPE
 * otherwise): M = 1 runs the integer GEMV with the sub-groups of each 128-K
 * tile kept apart in the X operand (each digit plane split per sub-group);
 * M >= 2 runs the BF16 tensor-core GEMV with one FP32 accumulator per
 * quantisation group, in chunks of 32 tokens (also for M >= 64, where the
 * group-128 layer takes the GEMM).
 * Arguments, layouts and errors otherwise as w4a16_linear, with scales and
 * zeros [N][K/group] and workspace >= w4a16_workspace_bytes_g(M, N, K, group).
 */
W4A16_API int w4a16_linear_g(const uint16_t* X, int64_t M, int64_t K, int group, const uint32_t* qweight,
                   const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                   size_t workspace_bytes, void* stream);

/*
 * Bytes of device workspace w4a16_linear() needs for this shape (0 if none).
 * The workspace starts with a 256 KB area of split-K arrival counters, then
 * holds prepared activations and FP32 split-K partial sums.  The counter area
 * must be zero before its first use (w4a16_workspace_init); every completed
 * call leaves it zero again and no call writes anything else there, so one
 * workspace, sized for the largest shape, can be shared by calls of any
 * shapes that are ordered on one stream.  Exception: a decode call with
 * N > 8,388,480 (one token) or N > 8,388,608 (more) keeps counters beyond
 * that area and needs a workspace of its own.  Calls that may run
 * concurrently need separate workspaces.
 */
W4A16_API size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Zero a workspace (enqueues a memset of `bytes` on `stream`). */
W4A16_API int w4a16_workspace_init(void* workspace, size_t bytes, void* stream);

/*
 * The W4A16 linear layer (the hot path).  Dequantises each weight tile on
 * the fly -- codes unpacked and (q - z) formed in registers, the BF16 scale
 * applied per group to the FP32 partial sums -- so only packed codes and
 * per-group metadata are read from memory.  Accumulation is FP32; Y is
 * rounded to BF16 (nearest, ties to even) once at the end.
 *   X         device, bf16 bits [M][K]
 *   qweight   device, uint32 [N][K/8];  scales device, bf16 bits [N][K/128];
 *   zeros     device, int32 [N][K/128]
 *   Y         device, bf16 bits [M][N] (written; must not overlap the inputs)
 *   workspace device, >= w4a16_workspace_bytes(M, N, K) bytes (NULL allowed when that is 0)
 * Activations: the decode GEMVs take every finite BF16 value; the GEMM
 * (M >= 64) sums (q - c) x in FP32 before the scale and needs |x| < 2^113.
 * Results are the same bits on every run.
 */
W4A16_API int w4a16_linear(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                 const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace, size_t workspace_bytes,
                 void* stream);

/* As w4a16_linear() with an explicit kernel family (enum w4a16_path). */
W4A16_API int w4a16_linear_path(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                      const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace, size_t workspace_bytes,
                      int path, void* stream);

/*
 * AWQ equivalence transform ("Axe Corsa 28B" model card, "How the Compression
 * Works", Stage 1; "Weight-Only Quantization and Mixed Precision", section 3):
 * input channel k of the weight matrix is multiplied by s_k before
 * quantisation and the same channel of the activations by s_k^-1, so the
 * product is unchanged in exact arithmetic while the salient channels (large
 * activations, s_k > 1) land on a finer part of the 4-bit grid.  Choosing s
 * (calibration) is the caller's; both entries take it as data.
 *
 * w4a16_quantize_pack_awq: quantise and pack W'[n][k] = w[n][k] * s[k], the
 * product rounded once to FP32, exactly as w4a16_quantize_pack would quantise
 * a W' given directly (asymmetric, group 128).
 *   s     device, fp32 [K], 16-byte aligned (finite, positive)
 *   other arguments, errors: as w4a16_quantize_pack (a product that overflows
 *   to infinity reports W4A16_ERR_NONFINITE).
 */
W4A16_API int w4a16_quantize_pack_awq(const float* W, const float* s, int64_t N, int64_t K, uint32_t* qweight,
                            uint16_t* scales, int32_t* zeros, int32_t* dev_status, void* stream);

/*
 * w4a16_linear_awq: Y = X' W_hat'^T with X'[m][k] = bf16(x[m][k] * inv_s[k])
 * (the exact product rounded once to BF16, nearest, ties to even) formed
 * inside each kernel family's own preparation of X -- no separate pass over X
 * and no X' in memory -- and W_hat' the packed weights of
 * w4a16_quantize_pack_awq.  Where a preceding layer already produces X'
 * (the inverse folded into its weights), call w4a16_linear instead.
 *   inv_s device, fp32 [K], 16-byte aligned: the inverse scales as the caller
 *         rounded them (typically fp32(1 / s[k]))
 *   other arguments, errors: as w4a16_linear_path (path = enum w4a16_path).
 */
W4A16_API int w4a16_linear_awq(const uint16_t* X, const float* inv_s, int64_t M, int64_t K, const uint32_t* qweight,
                     const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                     size_t workspace_bytes, int path, void* stream);

/*
 * The linear layer on host buffers: one call enqueues, on `stream`, the copy
 * of X from host to device, w4a16_linear(), and the copy of Y back to the
 * host, so a caller that holds activations in host memory pays a single
 * library call per layer.  For one token (M = 1, K a multiple of 1024) with
 * host buffers mapped into the device's address space (cudaHostAlloc, or
 * cudaHostRegister with cudaHostRegisterMapped) the two transfers are done
 * by the library's kernels -- a copy kernel reads X_host, the split-K
 * reduction also stores Y into Y_host -- so that consecutive calls keep
 * overlapping on the stream; otherwise one cudaMemcpyAsync each way.
 *   X_host    host, bf16 bits [M][K]; page-locked (cudaHostAlloc or
 *             cudaHostRegister) for the copy to be asynchronous
 *   X_dev     device, bf16 bits [M][K], the staging buffer X is copied into
 *   Y_dev     device, bf16 bits [M][N], the layer's output
 *   Y_host    host, bf16 bits [M][N], page-locked; valid once the stream
 *             has reached the end of this call's work
 *   other arguments as w4a16_linear().  The buffers must not overlap.
 */
W4A16_API int w4a16_linear_host(const uint16_t* X_host, uint16_t* X_dev, int64_t M, int64_t K, const uint32_t* qweight,
                      const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y_dev, uint16_t* Y_host,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Unpack codes ("What the Tensor Types Tell You": two INT4 codes per byte;
 * the word layout above).  codes: device, uint8 [N][K], values 0..15.
 * Test and inspection use.
 */
W4A16_API int w4a16_unpack(const uint32_t* qweight, int64_t N, int64_t K, uint8_t* codes, void* stream);

/*
 * Materialise W_hat = (q - z) * s rounded to BF16 (nearest, ties to even):
 * W_hat device, bf16 bits [N][K].  This is the offline dequantisation the
 * pages call an anti-pattern for inference ("Quantization I", Concept);
 * provided for tests and for the unfused comparison only.
 */
W4A16_API int w4a16_dequant(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                  uint16_t* W_hat, void* stream);

/*
 * Materialise W_hat from unpacked codes (codes: device, uint8 [N][K], values
 * 0..15, as written by w4a16_unpack): the middle kernel of the unfused
 * three-kernel pipeline the fused kernel replaces ("Weight-Only Quantization
 * and Mixed Precision", section 7, "The Pain Point": read and unpack, then
 * dequantise, then multiply, each through HBM).  Same bits as w4a16_dequant.
 * Comparison use only.
 */
W4A16_API int w4a16_dequant_codes(const uint8_t* codes, const uint16_t* scales, const int32_t* zeros, int64_t N,
                        int64_t K, uint16_t* W_hat, void* stream);

/*
 * Row renormalisation used between chained layers of the decode-stack
 * workload (not part of the method): out[m][:] = bf16_rne(y[m][:] / rms(y[m][:]))
 * with the sum of squares in FP32; a zero row stays zero.
 *   y, out device, bf16 bits [M][N] (out may equal y).
 */
W4A16_API int w4a16_renorm_rows(const uint16_t* y, int64_t M, int64_t N, uint16_t* out, void* stream);

/*
 * The linear layer without a caller-provided workspace.  (The source pages
 * describe no such entry point; it exists for callers that cannot allocate.)
 * Some callers may not allocate device memory once they run -- a serving loop
 * that reserved all of HBM at start-up, a framework whose allocator owns the
 * device, code that cannot reach cudaMalloc where it calls this library.  This
 * variant of the decode path (split-K GEMV, any M in token tiles of 32) keeps
 * its scratch -- prepared X, split-K partial sums, arrival counters -- in one
 * file-scope device array of w4a16_noalloc_scratch_bytes() bytes (16 MiB) that
 * every process loading the library holds on each GPU it uses until exit.  It
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *  - Arguments and layouts are those of w4a16_linear().  It always runs the
 *    decode path, in tiles of 32 tokens for M > 32, with results identical
 *    bit for bit to w4a16_linear_path(..., W4A16_PATH_DECODE, ...); for
 *    M >= 64, where w4a16_linear would choose the GEMM, the results agree
 *    with it within the layer's tolerance but are not the same bits.
 *  - The limit is the decode path's own scratch (prepared X, split-K
 *    partial sums, counters), which grows with N and K and with M only up
 *    to 32 tokens; a problem whose decode scratch exceeds the array returns
 *    W4A16_ERR_WORKSPACE and launches nothing.  (w4a16_workspace_bytes()
 *    also counts the GEMM's needs and can be larger for M >= 64.)
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; each call clears the counters it needs before launching.
 *    Calls that may overlap on the GPU (different streams, concurrent host
 *    threads without ordering) race on the array: order them on one stream.
 */
W4A16_API int w4a16_linear_noalloc(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight,
                                   const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y,
                                   void* stream);

/* Size of the built-in scratch array w4a16_linear_noalloc() uses, in bytes. */
W4A16_API size_t w4a16_noalloc_scratch_bytes(void);

/*
 * Diagnostic: synchronise the current device, then read and clear its fault
 * word.  Returns 0 when no kernel gave up a bounded wait since the last
 * call, a positive site code when one did (its outputs are then invalid),
 * or -1 if the device could not be queried.  Kernels never trap or spin
 * forever: a pipeline wait that exceeds about two seconds records its site
 * here and the kernel returns.  Only the first site is kept until the word
 * is read.
 * After a non-zero result, zero every workspace the failed calls used
 * (w4a16_workspace_init) before its next use: a kernel that gave up may have
 * left split-K arrival counters non-zero.  (w4a16_linear_noalloc clears the
 * counters it needs on every call.)
 */
W4A16_API int w4a16_device_fault(void);

/* Site code that w4a16_selftest_wait() records. */
#define W4A16_SELFTEST_SITE 900
/* Largest wait limit w4a16_selftest_wait() accepts, in SM cycles (about one second). */
#define W4A16_SELFTEST_MAX_CYCLES 2000000000LL

/*
 * Test of the failure path (the pages have no counterpart; this checks the
 * library's own error reporting).  Launches one CTA of 32 threads that waits,
 * with the library's bounded mbarrier wait, on a barrier phase nothing will
 * complete -- no copy, MMA or other thread is attached to it -- and gives up
 * after `limit_cycles` SM cycles (1 .. W4A16_SELFTEST_MAX_CYCLES): it records
 * W4A16_SELFTEST_SITE in the fault word and returns, exactly as a pipeline
 * wait of the linear kernels does on a timeout.  The GPU context stays
 * usable; w4a16_device_fault() then returns W4A16_SELFTEST_SITE.
 * Returns W4A16_ERR_ARG for a limit out of range, W4A16_ERR_DEVICE if the
 * current device is not sm_100.  Asynchronous on `stream`.
 */
W4A16_API int w4a16_selftest_wait(int64_t limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
