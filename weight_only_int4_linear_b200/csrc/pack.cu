// Offline and inspection kernels: quantise + pack, unpack, BF16 dequantisation,
// and the row renormalisation used between chained layers.
//
// Quantise + pack follows the "Axe Corsa 28B" model card, "How the Compression
// Works" (asymmetric INT4, one scale and one zero point per 128 consecutive
// weights, all 16 levels used) under the min/max affine reading documented in
// include/w4a16.h; the symmetric variant ("Quantization I: int8, int4, the
// basics", Concept: a scale and no zero point) stores signed codes as q + 8
// with the zero point 8, so the linear kernels read both formats unchanged.  Every decision that sets a code or a stored parameter is
// taken in binary64 with IEEE division and round-half-even, so the packed
// output is bit-exact with any correct implementation of the same reading.
#include "common.cuh"

namespace w4a16 {

// One warp per group of 128 weights: lane l holds w[4l .. 4l+3].
// kSym: s = bf16(max|w| / 7), q = clamp(rint(w / s), -8, 7) stored as q + 8, z = 8.
// col_scale (nullable): the AWQ transform, w[n][k] * col_scale[k] rounded once to FP32, is
// quantised in place of w.
template <bool kSym>
__global__ void __launch_bounds__(256) quantize_pack_kernel(const float* __restrict__ W,
                                                            const float* __restrict__ col_scale, int64_t N, int64_t K,
                                                            uint32_t* __restrict__ qweight,
                                                            uint16_t* __restrict__ scales,
                                                            int32_t* __restrict__ zeros, int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t ng = K / kGroup;
    const int64_t total = N * ng;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t grp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; grp < total; grp += warps) {
        const int64_t n = grp / ng, g = grp % ng;
        float4 v = reinterpret_cast<const float4*>(W + n * K + g * kGroup)[lane];
        if (col_scale) {
            const float4 c = reinterpret_cast<const float4*>(col_scale + g * kGroup)[lane];
            v = make_float4(__fmul_rn(v.x, c.x), __fmul_rn(v.y, c.y), __fmul_rn(v.z, c.z), __fmul_rn(v.w, c.w));
        }
        const bool finite = isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
        if (!__all_sync(0xFFFFFFFFu, finite)) {
            if (lane == 0) {
                atomicCAS(status, 0, (int)W4A16_ERR_NONFINITE);
                scales[grp] = 0;
                zeros[grp] = 0;
            }
            if ((lane & 1) == 0) qweight[n * (K / 8) + g * kWordsPerGroup + lane / 2] = 0u;
            continue;
        }
        float lo = fminf(fminf(v.x, v.y), fminf(v.z, v.w));
        float hi = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
        }
        const double mag = fmax(fabs((double)lo), fabs((double)hi));
        uint16_t sb = double_to_bf16_bits(kSym ? __ddiv_rn(mag, 7.0)
                                               : __ddiv_rn(__dsub_rn((double)hi, (double)lo), 15.0));
        if ((sb & 0x7FFFu) == 0) {
            sb = double_to_bf16_bits(mag);
            if ((sb & 0x7FFFu) == 0) sb = 0x3F80u;  // 1.0
        }
        const double s = (double)bf16_bits_to_float(sb);
        const double z = kSym ? 8.0 : rint(__ddiv_rn(-(double)lo, s));
        if (z > 2147483647.0 || z < -2147483648.0) {
            if (lane == 0) {
                atomicCAS(status, 0, (int)W4A16_ERR_ZERO_RANGE);
                scales[grp] = 0;
                zeros[grp] = 0;
            }
            if ((lane & 1) == 0) qweight[n * (K / 8) + g * kWordsPerGroup + lane / 2] = 0u;
            continue;
        }
        const float w4[4] = {v.x, v.y, v.z, v.w};
        uint32_t half = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            double t = __dadd_rn(rint(__ddiv_rn((double)w4[i], s)), z);
            t = fmin(fmax(t, 0.0), 15.0);
            half |= ((uint32_t)t) << (4 * i);
        }
        // word j = codes of lanes 2j (low half) and 2j+1 (high half)
        const uint32_t upper = __shfl_down_sync(0xFFFFFFFFu, half, 1);
        if ((lane & 1) == 0) qweight[n * (K / 8) + g * kWordsPerGroup + lane / 2] = half | (upper << 16);
        if (lane == 0) {
            scales[grp] = sb;
            zeros[grp] = (int32_t)z;
        }
    }
}

// Groups of GS = 32 or 64 weights ("Quantization I: int8, int4, the basics", Concept: groups of
// 32-128 values; "Weight-Only Quantization and Mixed Precision", section 8), same per-group rule
// as quantize_pack_kernel.  One warp per 128 weights (lane l holds w[4l .. 4l+3]); each group is
// a segment of GS/4 lanes and every collective runs on the segment's mask, so a failing group
// leaves its neighbours alone.  Scales and zero points are [N][K/GS].
template <bool kSym, int GS>
__global__ void __launch_bounds__(256) quantize_pack_small_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                                                  uint32_t* __restrict__ qweight,
                                                                  uint16_t* __restrict__ scales,
                                                                  int32_t* __restrict__ zeros, int32_t* status) {
    constexpr int kLanes = GS / 4;
    const int lane = threadIdx.x & 31;
    const unsigned seg = ((1u << kLanes) - 1u) << (lane & ~(kLanes - 1));
    const bool leader = (lane & (kLanes - 1)) == 0;
    const int64_t blocks_per_row = K / 128, groups_per_row = K / GS;
    const int64_t total = N * blocks_per_row;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t blk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; blk < total; blk += warps) {
        const int64_t n = blk / blocks_per_row, b = blk % blocks_per_row;
        const int64_t grp = n * groups_per_row + (b * 128 + 4 * lane) / GS;
        const int64_t word = n * (K / 8) + b * 16 + lane / 2;
        const float4 v = reinterpret_cast<const float4*>(W + n * K + b * 128)[lane];
        const bool finite = isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
        const bool ok = __all_sync(seg, finite);
        float lo = fminf(fminf(v.x, v.y), fminf(v.z, v.w));
        float hi = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
#pragma unroll
        for (int o = kLanes / 2; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(seg, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(seg, hi, o));
        }
        const double mag = fmax(fabs((double)lo), fabs((double)hi));
        uint16_t sb = double_to_bf16_bits(kSym ? __ddiv_rn(mag, 7.0)
                                               : __ddiv_rn(__dsub_rn((double)hi, (double)lo), 15.0));
        if ((sb & 0x7FFFu) == 0) {
            sb = double_to_bf16_bits(mag);
            if ((sb & 0x7FFFu) == 0) sb = 0x3F80u;  // 1.0
        }
        const double s = (double)bf16_bits_to_float(sb);
        const double z = kSym ? 8.0 : rint(__ddiv_rn(-(double)lo, s));
        const bool z_ok = z <= 2147483647.0 && z >= -2147483648.0;
        uint32_t half = 0;
        if (ok && z_ok) {
            const float w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                double t = __dadd_rn(rint(__ddiv_rn((double)w4[i], s)), z);
                t = fmin(fmax(t, 0.0), 15.0);
                half |= ((uint32_t)t) << (4 * i);
            }
        }
        // word j = codes of lanes 2j (low half) and 2j + 1 (high half), both in one segment
        const uint32_t upper = __shfl_xor_sync(seg, half, 1);
        if ((lane & 1) == 0) qweight[word] = half | (upper << 16);
        if (leader) {
            if (!ok || !z_ok) atomicCAS(status, 0, ok ? (int)W4A16_ERR_ZERO_RANGE : (int)W4A16_ERR_NONFINITE);
            scales[grp] = ok && z_ok ? sb : (uint16_t)0;
            zeros[grp] = ok && z_ok ? (int32_t)z : 0;
        }
    }
}

// One thread per packed word -> 8 codes.
__global__ void unpack_kernel(const uint32_t* __restrict__ qweight, int64_t words, uint8_t* __restrict__ codes) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words; i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t w = qweight[i];
        uint2 out;
        out.x = (w & 0xFu) | ((w >> 4) & 0xFu) << 8 | ((w >> 8) & 0xFu) << 16 | ((w >> 12) & 0xFu) << 24;
        out.y = ((w >> 16) & 0xFu) | ((w >> 20) & 0xFu) << 8 | ((w >> 24) & 0xFu) << 16 | ((w >> 28) & 0xFu) << 24;
        reinterpret_cast<uint2*>(codes)[i] = out;
    }
}

// Dequantisation from unpacked codes (the middle kernel of the unfused three-kernel
// W4A16 pipeline, "Weight-Only Quantization and Mixed Precision", section 7): one
// thread per 16 codes -> 16 BF16 values of (q - z) * s.  (q - z) * s is exact in
// FP32 (a 5-bit integer times an 8-bit significand), so the one rounding to BF16
// gives the same bits as dequant_kernel.
__global__ void dequant_codes_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                                     const int32_t* __restrict__ zeros, int64_t chunks, int64_t chunks_per_row,
                                     uint16_t* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / chunks_per_row, c = i - n * chunks_per_row;
        const int64_t grp = n * (chunks_per_row / (kGroup / 16)) + c / (kGroup / 16);
        const float s = bf16_bits_to_float(scales[grp]);
        const float z = (float)zeros[grp];
        const uint4 q = reinterpret_cast<const uint4*>(codes)[i];
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
        uint32_t o[8];
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float lo = ((float)((qw[w] >> (16 * h)) & 0xFFu) - z) * s;
                const float hi = ((float)((qw[w] >> (16 * h + 8)) & 0xFFu) - z) * s;
                o[2 * w + h] = (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
            }
        uint4* dst = reinterpret_cast<uint4*>(out) + 2 * i;
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// One thread per packed word -> 8 BF16 values of (q - z) * s (exact product in
// binary64, one rounding to BF16).
__global__ void dequant_kernel(const uint32_t* __restrict__ qweight, const uint16_t* __restrict__ scales,
                               const int32_t* __restrict__ zeros, int64_t words, int64_t words_per_row,
                               uint16_t* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / words_per_row, j = i % words_per_row;
        const int64_t grp = n * (words_per_row / kWordsPerGroup) + j / kWordsPerGroup;
        const double s = (double)bf16_bits_to_float(scales[grp]);
        const double z = (double)zeros[grp];
        const uint32_t w = qweight[i];
        uint32_t packed[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const double lo = ((double)((w >> (8 * p)) & 0xFu) - z) * s;
            const double hi = ((double)((w >> (8 * p + 4)) & 0xFu) - z) * s;
            packed[p] = (uint32_t)double_to_bf16_bits(lo) | ((uint32_t)double_to_bf16_bits(hi) << 16);
        }
        reinterpret_cast<uint4*>(out)[i] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

// One CTA per row: sum of squares in FP32, then y / sqrt(mean) rounded to BF16.
__global__ void __launch_bounds__(256) renorm_kernel(const uint16_t* __restrict__ y, int64_t N,
                                                     uint16_t* __restrict__ out) {
    const uint16_t* row = y + (int64_t)blockIdx.x * N;
    uint16_t* orow = out + (int64_t)blockIdx.x * N;
    float ss = 0.f;
    for (int64_t j = threadIdx.x; j < N; j += blockDim.x) {
        const float v = bf16_bits_to_float(row[j]);
        ss = fmaf(v, v, ss);
    }
    __shared__ float red[32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
        if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    const float rms = sqrtf(red[0] / (float)N);
    for (int64_t j = threadIdx.x; j < N; j += blockDim.x) {
        const float v = bf16_bits_to_float(row[j]);
        orow[j] = float_to_bf16_bits(rms > 0.f ? v / rms : 0.f);
    }
}

// The same for rows of N <= kRenormMaxN values, N a multiple of 8 and 16-byte aligned rows: 1024 threads per
// row, each holding up to four 8-value chunks in registers (one read of the row), as a kernel of the
// programmatic-launch chain: the next kernel may start its own loads while this one waits for y.
constexpr int kRenormThreads = 1024, kRenormChunks = 4;
constexpr int64_t kRenormMaxN = (int64_t)kRenormThreads * kRenormChunks * 8;
__global__ void __launch_bounds__(kRenormThreads) renorm_wide_kernel(const uint16_t* __restrict__ y, int64_t N,
                                                                     uint16_t* __restrict__ out) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");  // y comes from the preceding kernel
    const uint4* row = reinterpret_cast<const uint4*>(y + (int64_t)blockIdx.x * N);
    uint4* orow = reinterpret_cast<uint4*>(out + (int64_t)blockIdx.x * N);
    const int n8 = (int)(N / 8);
    uint4 v[kRenormChunks];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < kRenormChunks; ++c) {
        const int j = threadIdx.x + c * kRenormThreads;
        v[c] = j < n8 ? row[j] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
        }
    }
    __shared__ float red[32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = red[threadIdx.x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
        if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    const float rms = sqrtf(red[0] / (float)N);
#pragma unroll
    for (int c = 0; c < kRenormChunks; ++c) {
        const int j = threadIdx.x + c * kRenormThreads;
        if (j < n8) {
            const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
                o4[e] = (uint32_t)float_to_bf16_bits(rms > 0.f ? lo / rms : 0.f) |
                        ((uint32_t)float_to_bf16_bits(rms > 0.f ? hi / rms : 0.f) << 16);
            }
            orow[j] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
    }
}

static int grid_for(int64_t items, int threads) {
    int64_t blocks = ceil_div(items, threads);
    const int64_t cap = (int64_t)num_sms_current() * 32;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

int launch_quantize_pack(const float* W, const float* col_scale, int64_t N, int64_t K, uint32_t* qweight,
                         uint16_t* scales, int32_t* zeros, int32_t* dev_status, bool symmetric, cudaStream_t stream) {
    if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), stream) != cudaSuccess) return W4A16_ERR_CUDA;
    const int64_t groups = N * (K / kGroup);
    const int grid = grid_for(groups * 32, 256);
    if (symmetric)
        quantize_pack_kernel<true><<<grid, 256, 0, stream>>>(W, col_scale, N, K, qweight, scales, zeros, dev_status);
    else
        quantize_pack_kernel<false><<<grid, 256, 0, stream>>>(W, col_scale, N, K, qweight, scales, zeros, dev_status);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

int launch_quantize_pack_small(const float* W, int64_t N, int64_t K, int group, bool symmetric, uint32_t* qweight,
                               uint16_t* scales, int32_t* zeros, int32_t* dev_status, cudaStream_t stream) {
    if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), stream) != cudaSuccess) return W4A16_ERR_CUDA;
    const int grid = grid_for(N * (K / 128) * 32, 256);
    if (group == 64) {
        if (symmetric)
            quantize_pack_small_kernel<true, 64><<<grid, 256, 0, stream>>>(W, N, K, qweight, scales, zeros, dev_status);
        else
            quantize_pack_small_kernel<false, 64><<<grid, 256, 0, stream>>>(W, N, K, qweight, scales, zeros, dev_status);
    } else {
        if (symmetric)
            quantize_pack_small_kernel<true, 32><<<grid, 256, 0, stream>>>(W, N, K, qweight, scales, zeros, dev_status);
        else
            quantize_pack_small_kernel<false, 32><<<grid, 256, 0, stream>>>(W, N, K, qweight, scales, zeros, dev_status);
    }
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

int launch_unpack(const uint32_t* qweight, int64_t N, int64_t K, uint8_t* codes, cudaStream_t stream) {
    const int64_t words = N * (K / 8);
    unpack_kernel<<<grid_for(words, 256), 256, 0, stream>>>(qweight, words, codes);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

int launch_dequant_codes(const uint8_t* codes, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                         uint16_t* out, cudaStream_t stream) {
    const int64_t chunks = N * K / 16;
    dequant_codes_kernel<<<grid_for(chunks, 256), 256, 0, stream>>>(codes, scales, zeros, chunks, K / 16, out);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

int launch_dequant(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                   uint16_t* out, cudaStream_t stream) {
    const int64_t words = N * (K / 8);
    dequant_kernel<<<grid_for(words, 256), 256, 0, stream>>>(qweight, scales, zeros, words, K / 8, out);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

int launch_renorm(const uint16_t* y, int64_t M, int64_t N, uint16_t* out, cudaStream_t stream) {
    const bool wide = N % 8 == 0 && N <= kRenormMaxN && ((uintptr_t)y & 15) == 0 && ((uintptr_t)out & 15) == 0;
    if (!wide) {
        renorm_kernel<<<(unsigned)M, 256, 0, stream>>>(y, N, out);
        return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)M);
    cfg.blockDim = dim3(kRenormThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, renorm_wide_kernel, y, N, out) == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

}  // namespace w4a16
