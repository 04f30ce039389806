// Shared device/host helpers of the w4a16 CUDA library (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/w4a16.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "w4a16 targets sm_100a (Blackwell) only"
#endif

namespace w4a16 {

constexpr int kGroup = W4A16_GROUP;  // weights per quantisation group along K
constexpr int kWordsPerGroup = kGroup / 8;

// BF16 bit pattern -> float (exact).
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// float -> BF16 bits, round to nearest, ties to even (NaN kept quiet).
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// binary64 -> BF16 bits, one rounding (nearest, ties to even), by integer
// arithmetic on the binary64 encoding.
__device__ __forceinline__ uint16_t double_to_bf16_bits(double x) {
    uint64_t b = (uint64_t)__double_as_longlong(x);
    uint32_t sign = (uint32_t)(b >> 63) << 15;
    uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
    if (mag == 0) return (uint16_t)sign;
    if (mag >= 0x7FF0000000000000ull) return (uint16_t)(sign | (mag > 0x7FF0000000000000ull ? 0x7FC0u : 0x7F80u));
    uint32_t r;
    if (mag < 0x3810000000000000ull) {  // below 2^-126: BF16 subnormal spacing 2^-133
        double scaled = __longlong_as_double((long long)mag) * 0x1.0p133;
        r = (uint32_t)__double2ll_rn(scaled);  // <= 128; 128 is the smallest normal's encoding
    } else {
        uint64_t keep = mag >> 45;
        uint64_t rest = mag & ((1ull << 45) - 1ull);
        keep += (rest > (1ull << 44) || (rest == (1ull << 44) && (keep & 1ull))) ? 1ull : 0ull;
        int64_t e = (int64_t)(keep >> 7) - 1023 + 127;
        r = (e >= 255) ? 0x7F80u : (uint32_t)(((uint64_t)e << 7) | (keep & 0x7Full));
    }
    return (uint16_t)(sign | r);
}

// AWQ activation transform of one element: BF16 x times the binary32 inverse
// channel scale r, rounded once to BF16 (nearest, ties to even).  In FP32:
// p = fl(x r) and, by an FMA, the residual e = x r - p, which is exact while
// |p| >= 2^-100 (x r has at most 32 significant bits, so e has at most 9).
// Rounding p again to BF16 gives the rounding of x r except when p lies
// exactly halfway between two BF16 values; there the sign of e decides (e = 0
// is a true tie).  Below 2^-100 that case takes the exact binary64 product.
__device__ __forceinline__ uint32_t bf16_scaled(uint32_t xbits, float r) {
    const float x = __uint_as_float(xbits << 16);
    const float p = __fmul_rn(x, r);
    const float e = __fmaf_rn(x, r, -p);
    const uint32_t u = __float_as_uint(p);
    if ((u & 0x7FFFFFFFu) >= 0x7F800000u) return (u >> 16) | ((u & 0x7FFFFFFFu) > 0x7F800000u ? 0x40u : 0u);
    uint32_t hi = u >> 16;
    const uint32_t lo = u & 0xFFFFu;
    if (lo == 0x8000u) {
        if ((u & 0x7F800000u) < (27u << 23)) return double_to_bf16_bits((double)x * (double)r);
        hi += e != 0.f ? (((e > 0.f) == !(u >> 31)) ? 1u : 0u) : (hi & 1u);
    } else if (lo > 0x8000u) {
        hi += 1u;
    }
    return hi;
}
// The same for the two BF16 values of a 32-bit word (low half first along K).
__device__ __forceinline__ uint32_t bf16x2_scaled(uint32_t pair, float r_lo, float r_hi) {
    return bf16_scaled(pair & 0xFFFFu, r_lo) | (bf16_scaled(pair >> 16, r_hi) << 16);
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace w4a16

// Host-side launch helpers (defined in api.cu).
namespace w4a16 {
// Identity of the current CUDA context (0 while none is current).  Kernel attributes, occupancy
// and the device addresses of file-scope symbols belong to a context: they differ between devices
// and do not survive cudaDeviceReset, so the library's caches of them are keyed by it (runtime.cu).
uint64_t context_key();

// A value computed once per context: get(make) returns the value cached for the current device if
// it was made in the current context, else calls make() (a zero result is not cached).
template <class T>
class PerContext {
  public:
    template <class F>
    T get(F&& make) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) {
            cudaGetLastError();
            return T{};
        }
        std::lock_guard<std::mutex> lk(mu_);
        const uint64_t key = context_key();
        if (key != 0 && key_[dev] == key) return val_[dev];
        const T v = make();
        const uint64_t after = context_key();  // make() may have created the context
        if (v != T{} && after != 0) {
            key_[dev] = after;
            val_[dev] = v;
        }
        return v;
    }

  private:
    static constexpr int kDevices = 64;
    std::mutex mu_;
    uint64_t key_[kDevices] = {};
    T val_[kDevices] = {};
};

// The current device is sm_100: W4A16_OK (its SM count cached), else W4A16_ERR_DEVICE (api.cu).
int check_device();
int launch_quantize_pack(const float* W, const float* col_scale, int64_t N, int64_t K, uint32_t* qweight,
                         uint16_t* scales, int32_t* zeros, int32_t* dev_status, bool symmetric, cudaStream_t stream);
int launch_unpack(const uint32_t* qweight, int64_t N, int64_t K, uint8_t* codes, cudaStream_t stream);
int launch_dequant(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                   uint16_t* out, cudaStream_t stream);
int launch_dequant_codes(const uint8_t* codes, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                         uint16_t* out, cudaStream_t stream);
int launch_renorm(const uint16_t* y, int64_t M, int64_t N, uint16_t* out, cudaStream_t stream);

// Every workspace starts with the decode path's split-K arrival counters, at
// the same place for every shape: each call leaves its counters zero and no
// call writes anything else below kCounterBytes, so calls of any shapes and
// paths ordered on one stream can share one workspace (row tiles up to
// kSharedCounterTiles, i.e. N up to 8,388,608; the one-token kernel keeps one
// more counter after its row tiles', so N up to 8,388,480 there).
constexpr int64_t kSharedCounterTiles = 65536;
constexpr size_t kCounterBytes = (size_t)kSharedCounterTiles * 4;  // 256 KB

struct DecodePlan {
    int cc_tokens;    // > 0: the integer CUDA-core kernel for this many tokens (M <= 2)
    bool mt;          // the integer GEMV for 2-16 tokens per launch (gemv_mt.cu), in chunks of 16 tokens
    bool bf;          // the BF16 tensor-core GEMV (gemv_bf.cu), in chunks of 32 tokens
    int nt;           // tensor-core kernel: MMA N (16 or 32 tokens per launch); 1 with cc_tokens
    int row_tiles;    // 128-row tiles along N
    int unit_groups;  // units per row tile (a unit: 128 rows x one or two quantisation groups)
    int grid;         // persistent CTAs
    int units_base;   // each CTA streams units_base (+1 for the first units_rem CTAs) units
    int units_rem;
    int max_slots;    // partial-sum slots per row tile
    int cc_units;     // one-token kernel: units (quantisation groups) per chunk, 2 or 4
    int cc_cpt;       // one-token kernel: chunks per row tile (quantisation groups / cc_units)
    int cc_tiles_a;   // one-token kernel: row tiles in chunks of cc_units; the rest in chunks of 2
    int cc_chunks_a;  // one-token kernel: chunks of the first cc_tiles_a row tiles
    int cc_chunks;    // one-token kernel: chunks in all
    // workspace layout: [counters][Xp][xs][partials]
    size_t ws_counter_bytes, ws_xp_bytes, ws_xs_bytes, ws_partial_bytes;
    size_t workspace_bytes() const;
};
DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int num_sms);
// xscale (nullable, [K] FP32): the AWQ activation transform, x -> bf16(x * xscale[k]), applied
// where each path prepares X.
// X_host, Y_host (nullable, one-token plans only): device addresses of mapped page-locked host buffers; X is
// then first copied from X_host into X by a kernel of the launch chain, and Y is also stored into Y_host.
int launch_decode(const uint16_t* X, const float* xscale, int64_t M, int64_t K, const uint32_t* qweight,
                  const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                  const DecodePlan& plan, cudaStream_t stream, const uint16_t* X_host = nullptr,
                  uint16_t* Y_host = nullptr);
int num_sms_current();

// The BF16 tensor-core GEMV (gemv_bf.cu) for quantisation groups of `group` (32, 64, 128) weights, K / group
// a multiple of 8: scratch = bf_workspace_bytes (after the shared counters); runs M in chunks of 32 tokens.
size_t bf_workspace_bytes(int64_t M, int64_t N, int64_t K, int group, int num_sms);
int launch_decode_bf(const uint16_t* X, const float* xscale, int64_t M, int64_t K, int group, const uint32_t* qweight,
                     const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* scratch,
                     cudaStream_t stream);

// Chunk sums of the one-token GEMVs (gemv.cu, gemv_sub.cu): partial [row_tiles][cpt][128] -> Y [N] (and Y_host
// when given: a mapped host buffer), each row's slots added in slot order; a dependent launch.
// tiles_a >= 0: row tiles from tiles_a on hold cpt_b slots each, after the first tiles_a * cpt slots.
int launch_cc_reduce(const float* partial, uint16_t* Y, int64_t N, int cpt, int row_tiles, cudaStream_t stream,
                     uint16_t* Y_host = nullptr, int tiles_a = -1, int cpt_b = 0);
// Split-K reduction of the decode GEMVs (gemv.cu): a dependent grid of one CTA per 128-row tile that
// adds the partial-sum slots of every tile the GEMV's CTAs shared, in slot order, into Y.
int launch_decode_reduce(const float* partial, uint16_t* Y, int64_t N, int M, int G, int units_base, int units_rem,
                         int max_slots, int row_tiles, cudaStream_t stream);

// The integer GEMV for 2-16 tokens per launch (gemv_mt.cu): needs K / 128 to be a multiple of 8;
// scratch (after the shared counters) = mt_workspace_bytes; runs M in chunks of 16 tokens.
bool mt_supported(int64_t K);
size_t mt_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
int launch_decode_mt(const uint16_t* X, const float* xscale, int64_t M, int64_t K, const uint32_t* qweight,
                     const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* scratch,
                     cudaStream_t stream);

// Prefill (tensor-core GEMM) path for large M.
constexpr int64_t kPrefillMinM = 64;  // W4A16_PATH_AUTO switches to the GEMM at this many tokens
// group: quantisation group size, 128 or 64 (one or two folds per 128 K).
size_t prefill_workspace_bytes(int64_t M, int64_t K, int group = kGroup);
int launch_prefill(const uint16_t* X, const float* xscale, int64_t M, int64_t K, int group, const uint32_t* qweight,
                   const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                   cudaStream_t stream);

// Quantisation groups of 32 or 64 weights (pack.cu, gemv.cu): the quantiser, and the integer
// GEMV one token per launch.
int launch_quantize_pack_small(const float* W, int64_t N, int64_t K, int group, bool symmetric, uint32_t* qweight,
                               uint16_t* scales, int32_t* zeros, int32_t* dev_status, cudaStream_t stream);
size_t decode_sub_workspace_bytes(int64_t N, int64_t K, int group);
int launch_decode_sub(const uint16_t* X, int64_t M, int64_t K, int group, const uint32_t* qweight,
                      const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                      cudaStream_t stream);

// W8A16: INT8 weights with one BF16 scale per row (w8.cu).
size_t w8_workspace_bytes(int64_t M, int64_t N, int64_t K);
int launch_w8(const uint16_t* X, int64_t M, int64_t K, const int8_t* q, const uint16_t* scales, int64_t N,
              uint16_t* Y, void* workspace, cudaStream_t stream);
int launch_w8_quantize(const float* W, int64_t N, int64_t K, int8_t* q, uint16_t* scales, int32_t* status,
                       cudaStream_t stream);
int launch_w8_dequant(const int8_t* q, const uint16_t* scales, int64_t N, int64_t K, uint16_t* out,
                      cudaStream_t stream);
}  // namespace w4a16
