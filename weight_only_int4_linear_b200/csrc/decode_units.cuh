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

// All lanes wait; the warp gives up together if any lane's wait ran out.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, int parity, int* fault, int site) {
    const bool ok = mbar_wait(bar, parity, fault, site);
    return __all_sync(0xFFFFFFFFu, ok);
}

}  // namespace
}  // namespace w4a16
