// Pieces shared by the persistent split-K decode kernels (INT4 and INT8 weights):
// the unit deal (a unit = 128 weight rows x 128 K), exact powers of two and the
// warp-wide bounded barrier wait.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace w4a16 {
namespace {

// The CTA that owns unit u when units are dealt in contiguous ranges of base + 1
// (the first rem CTAs) or base units.
__device__ __forceinline__ int cta_of_unit(int64_t u, int base, int rem) {
    const int64_t big = (int64_t)(base + 1) * rem;
    if (u < big) return (int)(u / (base + 1));
    return rem + (int)((u - big) / base);
}

// Walks units in order without a division per step: unit = (row tile, group).
struct UnitCursor {
    int tile, g;
    __device__ __forceinline__ UnitCursor(int64_t u, int G) : tile((int)(u / G)), g((int)(u - (u / G) * G)) {}
    __device__ __forceinline__ void next(int G) {
        if (++g == G) {
            g = 0;
            ++tile;
        }
    }
};

// 2^e as FP32 for e in [-149, 127] (subnormal below -126).
__device__ __forceinline__ float pow2f(int e) {
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << (e + 149));
}

// The integer form of one group of 128 BF16 activations, computed by one warp (lane l holds the values
// 4l .. 4l + 3 as BF16 bits).  E is the exponent of the group's largest magnitude (-127 for a group of
// zeros and subnormals); x_int = x 2^(21 - E), rounded to nearest (exact for every value within 2^14
// of the maximum), is written in balanced base 256, x_int = 65536 d2 + 256 d1 + d0 with every digit in
// [-128, 127].  plane[p] receives this lane's word of digit plane p in the order in which the INT4
// kernels unpack a packed code word: lane 2w + h owns bytes 8w + 4h .. 8w + 4h + 3 of a 128-byte digit
// row, where codes (0, 2, 4, 6) of word w sit at 8w and codes (1, 3, 5, 7) at 8w + 4.  Returns
// sum_k x_int (exact: |sum| < 2^29) and E through *E_out.
__device__ __forceinline__ int group_digits_i4(const uint32_t (&bits)[4], int lane, uint32_t (&plane)[3],
                                               int* E_out) {
    uint32_t amax = max(max(bits[0] & 0x7FFFu, bits[1] & 0x7FFFu), max(bits[2] & 0x7FFFu, bits[3] & 0x7FFFu));
    amax = __reduce_max_sync(0xFFFFFFFFu, amax);
    const int ef = (int)(amax >> 7);
    const int E = ef == 0 ? -127 : ef - 127;  // every |x| of the group is below 2^(E + 1)
    const int kx = 21 - E;                    // in [-106, 148]
    const int k1 = min(kx, 127);
    const float s1 = pow2f(k1), s2 = pow2f(kx - k1);  // exact scalings, |x 2^kx| < 2^22
    int xi[4];
    uint32_t dg[3] = {0u, 0u, 0u};  // this lane's digit bytes per plane, as (i0, i2, i1, i3)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xi[i] = __float2int_rn(__uint_as_float(bits[i] << 16) * s1 * s2);
        const int d0 = ((xi[i] + 128) & 255) - 128;
        const int t = (xi[i] - d0) >> 8;
        const int d1 = ((t + 128) & 255) - 128;
        const int d2 = (t - d1) >> 8;
        const int pos = (i & 1) ? 16 + 8 * (i >> 1) : 8 * (i >> 1);  // i0 -> 0, i2 -> 8, i1 -> 16, i3 -> 24
        dg[0] |= (uint32_t)(d0 & 255) << pos;
        dg[1] |= (uint32_t)(d1 & 255) << pos;
        dg[2] |= (uint32_t)(d2 & 255) << pos;
    }
    // lane (w, h) holds codes 4h .. 4h + 3 of word w; h = 0 assembles the even-code word (its codes 0,
    // 2 and the partner's 4, 6), h = 1 the odd one (the partner's 1, 3, its own 5, 7)
    const int h = lane & 1;
#pragma unroll
    for (int p = 0; p < 3; ++p) {
        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, dg[p], 1);
        const uint32_t lo = h ? other : dg[p], hi = h ? dg[p] : other;
        plane[p] = h ? __byte_perm(lo, hi, 0x7632) : __byte_perm(lo, hi, 0x5410);
    }
    *E_out = E;
    return __reduce_add_sync(0xFFFFFFFFu, (xi[0] + xi[1]) + (xi[2] + xi[3]));
}

// All lanes wait; the warp gives up together if any lane's wait ran out.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, int parity, int* fault, int site) {
    const bool ok = mbar_wait(bar, parity, fault, site);
    return __all_sync(0xFFFFFFFFu, ok);
}

}  // namespace
}  // namespace w4a16
