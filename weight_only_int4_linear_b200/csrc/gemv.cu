// Decode path of the W4A16 linear layer: persistent split-K GEMV for small M
// (up to 32 tokens per launch).
//
// Only the packed codes (0.5 byte per weight) and the per-group scale and zero
// point cross the memory bus: each code is turned into a BF16 operand on chip
// and consumed at once ("Quantization I: int8, int4, the basics", Concept:
// dequantise tile by tile inside the multiply; "Weight-Only Quantization and
// Mixed Precision", section 7: one read of the packed INT4 weights, unpack
// with bit operations, asynchronous copies overlapping the math, nothing
// written back).
//
// Arithmetic per group g of 128 weights of row n and token m:
//   sum_k (q - z) s x  =  s * ( sum_k (128 + q) x  -  (128 + z) * sum_k x ).
// (128 + q) is exact in BF16 and comes out of a packed word with one lop3 per
// two codes (0x4300 | q encodes 128 + q).  The inner sums run on the 5th-gen
// tensor cores (tcgen05.mma, BF16 in, FP32 accumulate in tensor memory); the
// fold s * (P - (128 + z) * xsum) is applied in FP32 once per group, with
// xsum = sum_k x prepared alongside X.  The BF16 scale is never folded into a
// rounded operand, so the only rounding besides FP32 summation is the final
// BF16 rounding of Y.
//
// Work decomposition: a unit is 128 weight rows x one group (8 KB of codes).
// Units are numbered row tile by row tile and dealt out to a persistent grid
// in contiguous, equal ranges (+-1 unit), so every CTA streams the same number
// of bytes.  A row tile split between CTAs is reduced by the last CTA to
// finish it (arrival counter), summing the partials in a fixed order.
#include "common.cuh"
#include "sm100.cuh"

#include <mutex>

namespace w4a16 {
namespace {

constexpr int kRowsPerCta = 128;
constexpr int kStageWords = kRowsPerCta * kWordsPerGroup;  // 2048 words = 8 KB
constexpr int kXsStride = 32;  // tokens per group row of xsum
constexpr int kMaxTokens = 32;  // tokens per launch

struct DecodeArgs {
    const uint16_t* Xp;  // [Mc][K] BF16, 8-blocks reordered (0,4,1,5,2,6,3,7)
    const float* xs;     // [G][32] per-group sums of X (zero for tokens >= Mc)
    const uint16_t* scales;
    const int32_t* zeros;
    uint16_t* Y;         // [Mc][N]
    float* partial;      // [row_tiles][max_slots][Mc][128]
    int* counters;       // [row_tiles]
    int* fault;
    int M, N, K, G;
    int units_base, units_rem;
    int max_slots;
};

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

__device__ __forceinline__ uint32_t magic_pair(uint32_t w) {
    uint32_t r;
    asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(w));  // (w & m) | c
    return r;
}

__device__ __forceinline__ uint4 permute_block(uint4 v) {
    uint4 o;
    o.x = __byte_perm(v.x, v.z, 0x5410);  // x0, x4
    o.y = __byte_perm(v.x, v.z, 0x7632);  // x1, x5
    o.z = __byte_perm(v.y, v.w, 0x5410);  // x2, x6
    o.w = __byte_perm(v.y, v.w, 0x7632);  // x3, x7
    return o;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// X -> per-group sums xs, plus the operand layout the GEMV reads:
//  * tensor-core kernels: BF16 Xp with each 8-block reordered (0,4,1,5,2,6,3,7);
//  * CUDA-core kernel (fp32_layout): FP32 x_k * 16^-e, e = (0,1,2,3,4,2,3,4)[k mod 8],
//    as pairs (0,1), (2,5), (3,6), (4,7) of every 8-block, one 144-byte block per
//    quarter group (32 values + 16 bytes padding so the four quarter readers of a
//    warp hit distinct banks), then a 32-byte extras block per group:
//    [xsum, xoff_0..3, 0, 0, 0] with xoff_c = sum over quarter c of
//    2048 (x_3 + x_6) + 128 (x_4 + x_7) per 8-block (the 2^23 offsets that the
//    GEMV leaves in its high-position products, removed per quarter instead).
// Lets the GEMV launch early (PDL).
constexpr int kQuarterFloats = 36;                       // 32 values + 4 padding
constexpr int kGroupXfBytes = 4 * kQuarterFloats * 4 + 32;  // 576 + extras = 608 B per group

__global__ void __launch_bounds__(256) prep_x_kernel(const uint16_t* __restrict__ X, int M, int K, uint16_t* __restrict__ Xp,
                                                     float* __restrict__ xs, int fp32_layout) {
    pdl_launch_dependents();
    const int G = K / kGroup;
    const int64_t units = (int64_t)kXsStride * G * 16;  // multiple of 32
    for (int64_t u0 = (int64_t)blockIdx.x * blockDim.x; u0 < units; u0 += (int64_t)gridDim.x * blockDim.x) {
        const int64_t u = u0 + threadIdx.x;
        const bool active = u < units;
        const int m = (int)(u / (G * 16));
        const int rem = (int)(u - (int64_t)m * G * 16);
        const int g = rem >> 4, blk = rem & 15;
        float sum = 0.f, off = 0.f;
        if (active && m < M) {
            const int64_t xoff = (int64_t)m * K + (int64_t)g * kGroup + blk * 8;
            const uint4 v = *reinterpret_cast<const uint4*>(X + xoff);
            const float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                                bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
            if (fp32_layout) {
                // word blk of the group: quarter blk / 4, 32 bytes per word inside it
                float* dst = reinterpret_cast<float*>(reinterpret_cast<char*>(Xp) + ((int64_t)m * G + g) * kGroupXfBytes) +
                             (blk >> 2) * kQuarterFloats + 8 * (blk & 3);
                reinterpret_cast<float4*>(dst)[0] = make_float4(f[0], f[1] * 0x1p-4f, f[2] * 0x1p-8f, f[5] * 0x1p-8f);
                reinterpret_cast<float4*>(dst)[1] =
                    make_float4(f[3] * 0x1p-12f, f[6] * 0x1p-12f, f[4] * 0x1p-16f, f[7] * 0x1p-16f);
                off = 2048.f * (f[3] + f[6]) + 128.f * (f[4] + f[7]);
            } else {
                *reinterpret_cast<uint4*>(Xp + xoff) = permute_block(v);
            }
            sum = (f[0] + f[1]) + (f[2] + f[3]) + (f[4] + f[5]) + (f[6] + f[7]);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        // quarter sums of the offsets: lanes 4q..4q+3 of each 16-lane half hold quarter q
        off += __shfl_xor_sync(0xFFFFFFFFu, off, 1);
        off += __shfl_xor_sync(0xFFFFFFFFu, off, 2);
        if (active && blk == 0) xs[(int64_t)g * kXsStride + m] = sum;
        if (active && fp32_layout && m < M) {
            float* ext = reinterpret_cast<float*>(reinterpret_cast<char*>(Xp) + ((int64_t)m * G + g) * kGroupXfBytes +
                                                  4 * kQuarterFloats * 4);
            if (blk == 0) {
                ext[0] = sum;
                ext[5] = 0.f;
                ext[6] = 0.f;
                ext[7] = 0.f;
            }
            if ((blk & 3) == 0) ext[1 + (blk >> 2)] = off;
        }
    }
}

// --------------------------------------------------------------------------
// Tensor-core decode kernel (tcgen05 / TMEM), one persistent CTA per SM.
//
// Per unit (128 weight rows x one group): a dequantiser warp set (4 warps, one
// weight row per thread = one TMEM lane) turns the row's 16 packed words into
// 64 BF16 pairs (128 + q) and stores them with tcgen05.st as the A operand
// (128 x 128 BF16 = 64 columns) in tensor memory.  Column 4w + j holds codes
// j and j + 4 of word w; the prepared X uses the matching K order, so the B
// operand (NTOK tokens x 128, K-major) is a plain 128-byte-swizzled TMA tile.
// One thread issues eight tcgen05.mma (M = 128, N = NTOK, K = 16) per unit
// into its own TMEM accumulator; the fold warps read it back and apply
// acc += s * (D - (128 + z) * xsum).
//
// Warp roles (448 threads): 0-3 fold (TMEM lane quadrants 0-3, also the row
// tile epilogue), 4-7 and 8-11 dequantise even and odd units, 12 issues the
// MMAs, 13 drives TMA.  Rings: shared-memory stages (codes, X tile, xsum),
// 4 A buffers and 8 (NTOK = 16) or 4 (NTOK = 32) accumulators, each with a
// full/free mbarrier pair, so loads, dequantisation, MMAs and folds overlap.
template <int NTOK>
struct TcCfg {
    static constexpr int kXBlockBytes = NTOK * 128;  // 64 BF16 of K for NTOK tokens
    static constexpr int kXBytes = 2 * kXBlockBytes;  // one group of K
    static constexpr int kCodeOff = kXBytes;
    static constexpr int kXsOff = kXBytes + kStageWords * 4;
    static constexpr int kStageBytes = kXsOff + 1024;  // xsum slot, keeps stages 1024-aligned
    static constexpr int kStages = NTOK == 16 ? 12 : 10;
    static constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024;  // + alignment slack
    static constexpr uint32_t kIdesc = idesc_bf16_f32(128, NTOK);
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kNumA = 4;                  // A buffers of 64 columns at 0..255
    static constexpr int kNumD = NTOK == 16 ? 8 : 4;  // accumulators at 256..383
    static constexpr uint32_t kColD = 256;
};

constexpr int kFoldWarps = 4;
constexpr int kDqWarps = 8;
constexpr int kMmaWarp = kFoldWarps + kDqWarps;  // 12
constexpr int kTmaWarp = kMmaWarp + 1;           // 13
constexpr int kTcThreads = (kTmaWarp + 1) * 32;  // 448

template <int NTOK>
__global__ void __launch_bounds__(kTcThreads, 1) decode_tc_kernel(const __grid_constant__ CUtensorMap tq,
                                                                  const __grid_constant__ CUtensorMap tx,
                                                                  const DecodeArgs a) {
    using C = TcCfg<NTOK>;
    constexpr int S = C::kStages;
    constexpr int NA = C::kNumA, ND = C::kNumD;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[S], empty[S], afull[NA], afree[NA], mdone[ND], dfree[ND];
    __shared__ uint32_t s_tmem;
    __shared__ int s_last;
    __shared__ volatile int s_issued;

    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-aligned stages

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int64_t u_first = (int64_t)b * a.units_base + min(b, a.units_rem);
    const int nunits = a.units_base + (b < a.units_rem ? 1 : 0);
    const int G = a.G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4 + 1 + kFoldWarps);  // dequantiser set, MMA commit, fold warps (xsum)
        }
        for (int i = 0; i < NA; ++i) {
            mbar_init(&afull[i], 4);
            mbar_init(&afree[i], 1);
        }
        for (int i = 0; i < ND; ++i) {
            mbar_init(&mdone[i], 1);
            mbar_init(&dfree[i], kFoldWarps);
        }
        s_issued = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&s_tmem, C::kTmemCols);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == kTmaWarp) {  // ------------------------------------------------ TMA
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tx);
            const int pre = min(S, nunits);
            // the weights do not depend on the preparation kernel: start streaming them at once
            UnitCursor cur(u_first, G);
            for (int i = 0; i < pre; ++i, cur.next(G)) {
                mbar_arrive_expect_tx(&full[i], C::kStageBytes - 1024 + 128);
                tma_load_2d(ring + i * C::kStageBytes + C::kCodeOff, &tq, cur.g * kWordsPerGroup,
                            cur.tile * kRowsPerCta, &full[i]);
            }
            pdl_wait_primary();  // X and xsum come from the preparation kernel
            UnitCursor cx(u_first, G);
            for (int i = 0; i < pre; ++i, cx.next(G)) {
                const int g = cx.g;
                unsigned char* st = ring + i * C::kStageBytes;
                tma_load_2d(st, &tx, g * kGroup, 0, &full[i]);
                tma_load_2d(st + C::kXBlockBytes, &tx, g * kGroup + 64, 0, &full[i]);
                bulk_load(st + C::kXsOff, a.xs + (int64_t)g * kXsStride, 128, &full[i]);
            }
            int issued = pre;
            for (int i = pre; i < nunits; ++i, cur.next(G)) {
                const int s = i % S;
                if (!mbar_wait(&empty[s], ((i / S) - 1) & 1, a.fault, 21)) break;
                const int tile = cur.tile, g = cur.g;
                unsigned char* st = ring + s * C::kStageBytes;
                mbar_arrive_expect_tx(&full[s], C::kStageBytes - 1024 + 128);
                tma_load_2d(st + C::kCodeOff, &tq, g * kWordsPerGroup, tile * kRowsPerCta, &full[s]);
                tma_load_2d(st, &tx, g * kGroup, 0, &full[s]);
                tma_load_2d(st + C::kXBlockBytes, &tx, g * kGroup + 64, 0, &full[s]);
                bulk_load(st + C::kXsOff, a.xs + (int64_t)g * kXsStride, 128, &full[s]);
                ++issued;
            }
            // every copy issued must land before the CTA may exit
            for (int i = max(0, issued - S); i < issued; ++i) mbar_wait(&full[i % S], (i / S) & 1, a.fault, 22);
        }
        return;
    }

    if (warp == kMmaWarp) {  // ------------------------------------------ MMA issue
        if (lane == 0) {
            for (int i = 0; i < nunits; ++i) {
                const int s = i % S, ai = i % NA, di = i % ND;
                if (!mbar_wait(&afull[ai], (i / NA) & 1, a.fault, 31)) break;
                if (i >= ND && !mbar_wait(&dfree[di], ((i / ND) - 1) & 1, a.fault, 32)) break;
                if (!mbar_wait(&full[s], (i / S) & 1, a.fault, 33)) break;
                tc_fence_after();
                const uint32_t xaddr = smem_u32(ring + s * C::kStageBytes);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bdesc = sw128_kmajor_desc(xaddr + (kk >> 2) * C::kXBlockBytes + (kk & 3) * 32);
                    umma_ts(tmem + C::kColD + di * NTOK, tmem + ai * 64 + kk * 8, bdesc, C::kIdesc, kk > 0);
                }
                umma_commit(&afree[ai]);
                umma_commit(&mdone[di]);
                umma_commit(&empty[s]);
                s_issued = i + 1;
            }
        }
        return;
    }

    if (warp >= kFoldWarps) {  // ---------------------------------- dequantisers
        const int set = (warp - kFoldWarps) >> 2;         // 0: even units, 1: odd units
        const int quad = warp & 3;                        // TMEM lane quadrant
        const int row_local = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const int sw = (row_local >> 1) & 3;              // 64-byte swizzle of the codes tile
        for (int i = set; i < nunits; i += 2) {
            const int s = i % S, ai = i % NA;
            if (i >= NA && !mbar_wait(&afree[ai], ((i / NA) - 1) & 1, a.fault, 41)) break;
            if (!mbar_wait(&full[s], (i / S) & 1, a.fault, 42)) break;
            // logical 16-byte chunk q of row r sits at chunk q ^ ((r >> 1) & 3): conflict-free reads
            const unsigned char* codes = ring + s * C::kStageBytes + C::kCodeOff + row_local * 64;
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 v = *reinterpret_cast<const uint4*>(codes + 16 * (q ^ sw));
                w[4 * q] = v.x;
                w[4 * q + 1] = v.y;
                w[4 * q + 2] = v.z;
                w[4 * q + 3] = v.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pr[32];
#pragma unroll
                for (int ww = 0; ww < 8; ++ww) {
                    const uint32_t x = w[8 * half + ww];
                    pr[4 * ww + 0] = magic_pair(x);
                    pr[4 * ww + 1] = magic_pair(x >> 4);
                    pr[4 * ww + 2] = magic_pair(x >> 8);
                    pr[4 * ww + 3] = magic_pair(x >> 12);
                }
                tmem_st32(tl + ai * 64 + half * 32, pr);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[ai]);
        }
        return;
    }

    // ------------------------------------------------------- fold warps 0-3
    const int row_local = warp * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const int N = a.N, M = a.M;
    float acc[NTOK];
#pragma unroll
    for (int m = 0; m < NTOK; ++m) acc[m] = 0.f;
    bool aborted = false;
    int cur_tile = -1;

    auto flush = [&](int tile) {
        const int n = tile * kRowsPerCta + row_local;
        const int first = cta_of_unit((int64_t)tile * G, a.units_base, a.units_rem);
        const int last = cta_of_unit((int64_t)tile * G + G - 1, a.units_base, a.units_rem);
        if (first == last) {
            if (n < N) {
#pragma unroll
                for (int m = 0; m < NTOK; ++m)
                    if (m < M) a.Y[(int64_t)m * N + n] = float_to_bf16_bits(acc[m]);
            }
        } else {
            const int slot = b - first, nseg = last - first + 1;
            float* part = a.partial + ((int64_t)tile * a.max_slots + slot) * M * kRowsPerCta;
#pragma unroll
            for (int m = 0; m < NTOK; ++m)
                if (m < M) part[m * kRowsPerCta + row_local] = acc[m];
            __threadfence();
            named_barrier_sync(1, kFoldWarps * 32);
            if (threadIdx.x == 0) {
                const int prev = atomicAdd(&a.counters[tile], 1);
                s_last = (prev == nseg - 1);
            }
            named_barrier_sync(1, kFoldWarps * 32);
            if (s_last) {
                __threadfence();
                const int rows = min(kRowsPerCta, N - tile * kRowsPerCta);
                const float* pb = a.partial + (int64_t)tile * a.max_slots * M * kRowsPerCta;
                for (int idx = threadIdx.x; idx < M * rows; idx += kFoldWarps * 32) {
                    const int m = idx / rows, rl = idx - m * rows;
                    float sum = 0.f;
                    for (int sl = 0; sl < nseg; ++sl) sum += __ldcg(pb + ((int64_t)sl * M + m) * kRowsPerCta + rl);
                    a.Y[(int64_t)m * N + tile * kRowsPerCta + rl] = float_to_bf16_bits(sum);
                }
                if (threadIdx.x == 0) a.counters[tile] = 0;
            }
            named_barrier_sync(1, kFoldWarps * 32);
        }
#pragma unroll
        for (int m = 0; m < NTOK; ++m) acc[m] = 0.f;
    };

    // scale and 128 + zero of this thread's row, one unit ahead
    auto load_meta = [&](int j, int tile, int g, float& sv, float& zv) {
        sv = 0.f;
        zv = 0.f;
        if (j < nunits) {
            const int n = tile * kRowsPerCta + row_local;
            if (n < N) {
                sv = bf16_bits_to_float(__ldg(a.scales + (int64_t)n * G + g));
                zv = 128.f + (float)__ldg(a.zeros + (int64_t)n * G + g);
            }
        }
    };

    auto fold_unit = [&](int j, int tile, float sv, float zv) {
        if (tile != cur_tile) {
            if (cur_tile >= 0) flush(cur_tile);
            cur_tile = tile;
        }
        if (aborted) return;
        const int di = j % ND, s = j % S;
        if (!mbar_wait(&mdone[di], (j / ND) & 1, a.fault, 13)) {
            aborted = true;
            return;
        }
        tc_fence_after();
        uint32_t d0[16], d1[16];
        tmem_ld16(tl + C::kColD + di * NTOK, d0);
        if (NTOK == 32) tmem_ld16(tl + C::kColD + di * NTOK + 16, d1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dfree[di]);
        const float* xs = reinterpret_cast<const float*>(ring + s * C::kStageBytes + C::kXsOff);
#pragma unroll
        for (int q = 0; q < NTOK / 4; ++q) {
            if (4 * q < M) {
                const float4 xv = *reinterpret_cast<const float4*>(xs + 4 * q);
                const float xq[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = 4 * q + e;
                    const uint32_t dm = m < 16 ? d0[m & 15] : d1[m & 15];
                    acc[m] = fmaf(sv, fmaf(-zv, xq[e], __uint_as_float(dm)), acc[m]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // xsum read
    };

    // two cursors: `fc` at the unit being folded, `mc` one unit ahead for the metadata loads
    UnitCursor fc(u_first, G), mc(u_first, G);
    float s0, z0, s1, z1;
    load_meta(0, mc.tile, mc.g, s0, z0);
    mc.next(G);
    for (int j = 0; j < nunits; j += 2) {
        load_meta(j + 1, mc.tile, mc.g, s1, z1);
        mc.next(G);
        fold_unit(j, fc.tile, s0, z0);
        fc.next(G);
        if (j + 1 < nunits) {
            load_meta(j + 2, mc.tile, mc.g, s0, z0);
            mc.next(G);
            fold_unit(j + 1, fc.tile, s1, z1);
            fc.next(G);
        }
    }
    if (cur_tile >= 0) flush(cur_tile);

    // teardown: every MMA issued must be complete before the columns are released
    named_barrier_sync(1, kFoldWarps * 32);
    if (warp == 0) {
        if (aborted) {
            const int issued = s_issued;
            for (int j = max(0, issued - ND); j < issued; ++j) mbar_wait(&mdone[j % ND], (j / ND) & 1, a.fault, 14);
        }
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// --------------------------------------------------------------------------
// Single-token decode kernel on the CUDA cores.
//
// At M = 1 a tensor-core MMA would waste most of its columns and each MMA
// instruction costs about a hundred cycles however small, so the dot product
// runs on the FP32 pipes.  Per packed word: one lop3 per code places its
// nibble in the mantissa of 2^23 (bits 4e, e = 0..4; codes 5-7 after one
// shift), giving 2^23 + 16^e q; packed FP32 FMAs (fma.f32x2) multiply by
// x * 16^-e (prepared once per call, exact).  For the low positions (e <= 2)
// a packed subtract removes 2^23 first; for e = 3, 4 the product keeps
// 2^(23-4e) x, which is small next to q x and is removed once per quarter
// group with the prepared offset sum.  Per group, each thread adds
// s * (its partial sum) to each of its rows, and one of the four threads
// sharing the group subtracts s * z * xsum.
//
// CTA: warp 4 drives TMA (codes of 128 rows x one group with the 64-byte
// swizzle, the matching 128 x 8 scales and 128 x 4 zero points, the scaled X
// and its extras) into a 4-stage ring; warps 0-3 compute, thread t taking
// words 4c..4c+3 (c = t % 4) of rows t/4 + 32i, i = 0..3.  Up to four CTAs
// share an SM.
constexpr int kCcWarps = 4;
constexpr int kCcThreads = (kCcWarps + 1) * 32;
constexpr int kCcStages = 4;
constexpr int kCcCodeBytes = kStageWords * 4;           // 8 KB, 64-byte swizzle
constexpr int kCcScOff = kCcCodeBytes;                  // scales box: 128 rows x 8 groups (BF16)
constexpr int kCcZeOff = kCcScOff + kRowsPerCta * 16;   // zeros box: 128 rows x 4 groups (int32)
constexpr int kCcXOff = kCcZeOff + kRowsPerCta * 16;    // scaled FP32 X of the group + extras (608 B)
constexpr int kCcExtOff = kCcXOff + 4 * kQuarterFloats * 4;
constexpr int kCcStageBytes = 13 * 1024;                // keeps stages 1024-aligned
constexpr size_t kCcSmem = (size_t)kCcStages * kCcStageBytes + 1024;
static_assert(kCcXOff + kGroupXfBytes <= kCcStageBytes, "stage layout");

// acc (two FP32 lanes) (+)= sum over one packed word of q_k * x_k (plus the
// 2^(23-4e) x offsets of the e = 3, 4 positions).  xp0..xp3 are the scaled X
// pairs (0,1), (2,5), (3,6), (4,7); m2 holds (2^23, 2^23).
#define W4A16_WORD_DOT_BODY(FIRST_FMA)                                    \
    "{\n\t"                                                                \
    ".reg .b32 h, a0, a1, a2, a5, a3, a6, a4, a7;\n\t"                     \
    ".reg .b64 v0, v1, v2, v3;\n\t"                                        \
    "shr.b32 h, %1, 12;\n\t"                                               \
    "lop3.b32 a0, %1, 0x0000000F, 0x4B000000, 0xEA;\n\t"                   \
    "lop3.b32 a1, %1, 0x000000F0, 0x4B000000, 0xEA;\n\t"                   \
    "lop3.b32 a2, %1, 0x00000F00, 0x4B000000, 0xEA;\n\t"                   \
    "lop3.b32 a5, h, 0x00000F00, 0x4B000000, 0xEA;\n\t"                    \
    "lop3.b32 a3, %1, 0x0000F000, 0x4B000000, 0xEA;\n\t"                   \
    "lop3.b32 a6, h, 0x0000F000, 0x4B000000, 0xEA;\n\t"                    \
    "lop3.b32 a4, %1, 0x000F0000, 0x4B000000, 0xEA;\n\t"                   \
    "lop3.b32 a7, h, 0x000F0000, 0x4B000000, 0xEA;\n\t"                    \
    "mov.b64 v0, {a0, a1};\n\t"                                            \
    "mov.b64 v1, {a2, a5};\n\t"                                            \
    "mov.b64 v2, {a3, a6};\n\t"                                            \
    "mov.b64 v3, {a4, a7};\n\t"                                            \
    "sub.rn.f32x2 v0, v0, %6;\n\t"                                         \
    "sub.rn.f32x2 v1, v1, %6;\n\t" FIRST_FMA                              \
    "fma.rn.f32x2 %0, v1, %3, %0;\n\t"                                     \
    "fma.rn.f32x2 %0, v2, %4, %0;\n\t"                                     \
    "fma.rn.f32x2 %0, v3, %5, %0;\n\t"                                     \
    "}"

// acc (two FP32 lanes) (+)= sum over one packed word of q_k * x_k (plus the
// 2^(23-4e) x offsets of the e = 3, 4 positions).  xp0..xp3 are the scaled X
// pairs (0,1), (2,5), (3,6), (4,7); m2 holds (2^23, 2^23).  FIRST starts acc.
template <bool FIRST>
__device__ __forceinline__ void word_dot(unsigned long long& acc, uint32_t w, unsigned long long xp0,
                                         unsigned long long xp1, unsigned long long xp2, unsigned long long xp3,
                                         unsigned long long m2) {
    if (FIRST)
        asm(W4A16_WORD_DOT_BODY("mul.rn.f32x2 %0, v0, %2;\n\t")
            : "=l"(acc)
            : "r"(w), "l"(xp0), "l"(xp1), "l"(xp2), "l"(xp3), "l"(m2));
    else
        asm(W4A16_WORD_DOT_BODY("fma.rn.f32x2 %0, v0, %2, %0;\n\t")
            : "+l"(acc)
            : "r"(w), "l"(xp0), "l"(xp1), "l"(xp2), "l"(xp3), "l"(m2));
}

__device__ __forceinline__ float lanes_sum(unsigned long long v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo + hi;
}

__global__ void __launch_bounds__(kCcThreads) decode_cc_kernel(const __grid_constant__ CUtensorMap tq,
                                                               const __grid_constant__ CUtensorMap tsc,
                                                               const __grid_constant__ CUtensorMap tze,
                                                               const DecodeArgs a) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kCcStages], empty[kCcStages];
    __shared__ int s_last;
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((1024u - (raw & 1023u)) & 1023u);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int64_t u_first = (int64_t)b * a.units_base + min(b, a.units_rem);
    const int nunits = a.units_base + (b < a.units_rem ? 1 : 0);
    const int G = a.G, N = a.N;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kCcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCcWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kCcWarps) {  // ---------------------------------------------- TMA
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tsc);
            prefetch_tmap(&tze);
            constexpr uint32_t kTx = kCcCodeBytes + 2 * kRowsPerCta * 16 + kGroupXfBytes;
            const char* xf = reinterpret_cast<const char*>(a.Xp);
            const int pre = min(kCcStages, nunits);
            UnitCursor cur(u_first, G);
            for (int i = 0; i < pre; ++i, cur.next(G)) {  // the weights need nothing from the preparation kernel
                unsigned char* st = ring + i * kCcStageBytes;
                mbar_arrive_expect_tx(&full[i], kTx);
                tma_load_2d(st, &tq, cur.g * kWordsPerGroup, cur.tile * kRowsPerCta, &full[i]);
                tma_load_2d(st + kCcScOff, &tsc, cur.g & ~7, cur.tile * kRowsPerCta, &full[i]);
                tma_load_2d(st + kCcZeOff, &tze, cur.g & ~3, cur.tile * kRowsPerCta, &full[i]);
            }
            pdl_wait_primary();  // scaled X and its extras come from the preparation kernel
            UnitCursor cx(u_first, G);
            for (int i = 0; i < pre; ++i, cx.next(G))
                bulk_load(ring + i * kCcStageBytes + kCcXOff, xf + (int64_t)cx.g * kGroupXfBytes, kGroupXfBytes,
                          &full[i]);
            int issued = pre;
            for (int i = pre; i < nunits; ++i, cur.next(G)) {
                const int s = i % kCcStages;
                if (!mbar_wait(&empty[s], ((i / kCcStages) - 1) & 1, a.fault, 51)) break;
                unsigned char* st = ring + s * kCcStageBytes;
                mbar_arrive_expect_tx(&full[s], kTx);
                tma_load_2d(st, &tq, cur.g * kWordsPerGroup, cur.tile * kRowsPerCta, &full[s]);
                tma_load_2d(st + kCcScOff, &tsc, cur.g & ~7, cur.tile * kRowsPerCta, &full[s]);
                tma_load_2d(st + kCcZeOff, &tze, cur.g & ~3, cur.tile * kRowsPerCta, &full[s]);
                bulk_load(st + kCcXOff, xf + (int64_t)cur.g * kGroupXfBytes, kGroupXfBytes, &full[s]);
                ++issued;
            }
            for (int i = max(0, issued - kCcStages); i < issued; ++i)
                mbar_wait(&full[i % kCcStages], (i / kCcStages) & 1, a.fault, 52);
        }
        return;
    }

    // ---------------------------------------------------- compute warps 0-3
    const int t = threadIdx.x;
    const int c = t & 3;   // words 4c..4c+3 of the group
    const int rg = t >> 2; // rows rg + 32 i
    // the 64-byte swizzle of the codes tile: logical chunk c of row r sits at chunk c ^ ((r >> 1) & 3);
    // (r >> 1) & 3 is the same for the four rows rg + 32 i
    const int code_off = rg * 64 + 16 * (c ^ ((rg >> 1) & 3));
    const int meta_off = rg * 16;
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    int cur_tile = -1;
    bool aborted = false;

    auto flush = [&](int tile) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // reduce over the four threads of each row
            y[i] += __shfl_xor_sync(0xFFFFFFFFu, y[i], 1);
            y[i] += __shfl_xor_sync(0xFFFFFFFFu, y[i], 2);
        }
        const int first = cta_of_unit((int64_t)tile * G, a.units_base, a.units_rem);
        const int last = cta_of_unit((int64_t)tile * G + G - 1, a.units_base, a.units_rem);
        if (first == last) {
            if (c == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int n = tile * kRowsPerCta + rg + 32 * i;
                    if (n < N) a.Y[n] = float_to_bf16_bits(y[i]);
                }
            }
        } else {
            const int slot = b - first, nseg = last - first + 1;
            float* part = a.partial + ((int64_t)tile * a.max_slots + slot) * kRowsPerCta;
            if (c == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) part[rg + 32 * i] = y[i];
            }
            __threadfence();
            named_barrier_sync(1, kCcWarps * 32);
            if (t == 0) {
                const int prev = atomicAdd(&a.counters[tile], 1);
                s_last = (prev == nseg - 1);
            }
            named_barrier_sync(1, kCcWarps * 32);
            if (s_last) {
                __threadfence();
                const int rows = min(kRowsPerCta, N - tile * kRowsPerCta);
                const float* pb = a.partial + (int64_t)tile * a.max_slots * kRowsPerCta;
                for (int rl = t; rl < rows; rl += kCcWarps * 32) {
                    float sum = 0.f;
                    for (int sl = 0; sl < nseg; ++sl) sum += __ldcg(pb + (int64_t)sl * kRowsPerCta + rl);
                    a.Y[tile * kRowsPerCta + rl] = float_to_bf16_bits(sum);
                }
                if (t == 0) a.counters[tile] = 0;
            }
            named_barrier_sync(1, kCcWarps * 32);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) y[i] = 0.f;
    };

    const unsigned long long m2 = 0x4B0000004B000000ull;
    UnitCursor uc(u_first, G);
    for (int i = 0; i < nunits; ++i, uc.next(G)) {
        const int tile = uc.tile, g = uc.g;
        if (tile != cur_tile) {
            if (cur_tile >= 0) flush(cur_tile);
            cur_tile = tile;
        }
        if (aborted) continue;
        const int s = i % kCcStages;
        if (!mbar_wait(&full[s], (i / kCcStages) & 1, a.fault, 53)) {
            aborted = true;
            continue;
        }
        const unsigned char* st = ring + s * kCcStageBytes;
        uint4 w[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) w[r] = *reinterpret_cast<const uint4*>(st + code_off + 2048 * r);
        const ulonglong2* xq = reinterpret_cast<const ulonglong2*>(st + kCcXOff + c * kQuarterFloats * 4);
        ulonglong2 xw[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) xw[j] = xq[j];
        const float* ext = reinterpret_cast<const float*>(st + kCcExtOff);
        const float xsum = ext[0], xoff = ext[1 + c];
        const unsigned char* scb = st + kCcScOff + meta_off + 2 * (g & 7);
        const unsigned char* zeb = st + kCcZeOff + meta_off + 4 * (g & 3);
        float sv[4], zv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            // rows past N were zero-filled by TMA: s = 0 folds them away
            sv[r] = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(scb + 512 * r));
            zv[r] = (float)*reinterpret_cast<const int32_t*>(zeb + 512 * r);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        const float corr = (c == 0) ? xsum : 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            unsigned long long acc;
            word_dot<true>(acc, w[r].x, xw[0].x, xw[0].y, xw[1].x, xw[1].y, m2);
            word_dot<false>(acc, w[r].y, xw[2].x, xw[2].y, xw[3].x, xw[3].y, m2);
            word_dot<false>(acc, w[r].z, xw[4].x, xw[4].y, xw[5].x, xw[5].y, m2);
            word_dot<false>(acc, w[r].w, xw[6].x, xw[6].y, xw[7].x, xw[7].y, m2);
            // y += s * (sum q x + offsets - xoff  -  [one thread of four] z xsum)
            y[r] = fmaf(sv[r], fmaf(-zv[r], corr, lanes_sum(acc) - xoff), y[r]);
        }
    }
    if (cur_tile >= 0) flush(cur_tile);
}

template <int NTOK>
int occupancy_nt() {
    static int occ = 0;
    if (occ == 0) {
        if (cudaFuncSetAttribute(decode_tc_kernel<NTOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)TcCfg<NTOK>::kSmem) != cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, decode_tc_kernel<NTOK>, kTcThreads,
                                                          TcCfg<NTOK>::kSmem) != cudaSuccess ||
            o < 1)
            return 0;
        occ = 1;  // one CTA per SM: it owns all 512 TMEM columns
    }
    return occ;
}

int occupancy_cc() {
    static int occ = 0;
    if (occ == 0) {
        if (cudaFuncSetAttribute(decode_cc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCcSmem) !=
            cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, decode_cc_kernel, kCcThreads, kCcSmem) != cudaSuccess ||
            o < 1)
            return 0;
        occ = o;
    }
    return occ;
}

int occupancy(int ntok) {
    if (ntok == 1) return occupancy_cc();
    return ntok == 16 ? occupancy_nt<16>() : occupancy_nt<32>();
}

// Tensor maps keyed by base pointer and shape (encoding costs a few
// microseconds of host time; a decode step reuses the same few tensors).
struct TmapEntry {
    const void* ptr;
    int64_t rows, cols;
    int kind;
    CUtensorMap map;
};
std::mutex g_tmap_mu;
TmapEntry g_tmaps[128];
int g_tmap_next = 0;

bool cached_tmap(int kind, const void* ptr, int64_t rows, int64_t cols, CUtensorMap* out) {
    std::lock_guard<std::mutex> lk(g_tmap_mu);
    for (auto& e : g_tmaps)
        if (e.ptr == ptr && e.rows == rows && e.cols == cols && e.kind == kind) {
            *out = e.map;
            return true;
        }
    TmapEntry& e = g_tmaps[g_tmap_next];
    bool ok;
    if (kind == 0)  // packed weights: uint32 [rows = N][cols = K/8], box = one group x 128 rows, 64-B swizzle
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT32, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 4, kWordsPerGroup, kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_64B);
    else if (kind == 2)  // scales: bf16 [rows = N][cols = G], box = 8 groups x 128 rows
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 2, 8, kRowsPerCta);
    else if (kind == 3)  // zeros: int32 [rows = N][cols = G], box = 4 groups x 128 rows
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_INT32, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 4, 4, kRowsPerCta);
    else  // prepared X: bf16 [rows = Mc][cols = K], box = 64 x NTOK (kind), 128-byte swizzle
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 2, 64, (uint32_t)kind, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return false;
    e.ptr = ptr;
    e.rows = rows;
    e.cols = cols;
    e.kind = kind;
    g_tmap_next = (g_tmap_next + 1) % 128;
    *out = e.map;
    return true;
}

int launch_cc(const CUtensorMap& tq, const CUtensorMap& tsc, const CUtensorMap& tze, const DecodeArgs& args, int grid,
              cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kCcThreads);
    cfg.dynamicSmemBytes = kCcSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_cc_kernel, tq, tsc, tze, args) == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

template <int NTOK>
int launch_tc(const CUtensorMap& tq, const CUtensorMap& tx, const DecodeArgs& args, int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = TcCfg<NTOK>::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_tc_kernel<NTOK>, tq, tx, args) == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int num_sms) {
    DecodePlan p{};
    const int64_t Mc = M < kMaxTokens ? M : kMaxTokens;
    const int64_t G = K / kGroup;
    // 1: CUDA-core kernel (needs 16-byte metadata rows: G % 8 == 0); else tensor-core MMA N
    p.nt = (Mc == 1 && G % 8 == 0) ? 1 : (Mc <= 16 ? 16 : 32);
    p.row_tiles = (int)ceil_div(N, kRowsPerCta);
    const int64_t units = (int64_t)p.row_tiles * G;
    int occ = occupancy(p.nt);
    if (occ < 1) occ = 1;
    int64_t grid = (int64_t)occ * num_sms;
    if (grid > units) grid = units;
    p.grid = (int)grid;
    p.units_base = (int)(units / grid);
    p.units_rem = (int)(units % grid);
    p.max_slots = (int)((G - 1) / p.units_base + 2);
    p.ws_xp_bytes = align256(p.nt == 1 ? (size_t)G * kGroupXfBytes : (size_t)Mc * K * 2);
    p.ws_xs_bytes = align256((size_t)G * kXsStride * 4);
    p.ws_partial_bytes = align256((size_t)p.row_tiles * p.max_slots * Mc * kRowsPerCta * 4);
    p.ws_counter_bytes = align256((size_t)p.row_tiles * 4);
    return p;
}

size_t DecodePlan::workspace_bytes() const { return ws_xp_bytes + ws_xs_bytes + ws_partial_bytes + ws_counter_bytes; }

int launch_decode(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                  const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace, const DecodePlan& plan,
                  cudaStream_t stream) {
    CUtensorMap tq;
    if (!cached_tmap(0, qweight, N, K / 8, &tq)) return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    char* ws = reinterpret_cast<char*>(workspace);
    uint16_t* Xp = reinterpret_cast<uint16_t*>(ws);
    float* xs = reinterpret_cast<float*>(ws + plan.ws_xp_bytes);
    float* partial = reinterpret_cast<float*>(ws + plan.ws_xp_bytes + plan.ws_xs_bytes);
    int* counters = reinterpret_cast<int*>(ws + plan.ws_xp_bytes + plan.ws_xs_bytes + plan.ws_partial_bytes);
    const int G = (int)(K / kGroup);
    for (int64_t m0 = 0; m0 < M; m0 += kMaxTokens) {
        const int Mc = (int)((M - m0) < kMaxTokens ? (M - m0) : kMaxTokens);
        CUtensorMap tx;
        if (plan.nt > 1 && !cached_tmap(plan.nt, Xp, Mc, K, &tx)) return W4A16_ERR_CUDA;
        const int64_t prep_units = (int64_t)kXsStride * G * 16;
        int prep_grid = (int)ceil_div(prep_units, 256);
        if (prep_grid > num_sms_current() * 8) prep_grid = num_sms_current() * 8;
        prep_x_kernel<<<prep_grid, 256, 0, stream>>>(X + m0 * K, Mc, (int)K, Xp, xs, plan.nt == 1 ? 1 : 0);
        if (cudaGetLastError() != cudaSuccess) return W4A16_ERR_CUDA;
        DecodeArgs args;
        args.Xp = Xp;
        args.xs = xs;
        args.scales = scales;
        args.zeros = zeros;
        args.Y = Y + m0 * N;
        args.partial = partial;
        args.counters = counters;
        args.fault = fault;
        args.M = Mc;
        args.N = (int)N;
        args.K = (int)K;
        args.G = G;
        args.units_base = plan.units_base;
        args.units_rem = plan.units_rem;
        args.max_slots = plan.max_slots;
        CUtensorMap tsc, tze;
        if (plan.nt == 1 && (!cached_tmap(2, scales, N, G, &tsc) || !cached_tmap(3, zeros, N, G, &tze)))
            return W4A16_ERR_CUDA;
        const int st = plan.nt == 1    ? launch_cc(tq, tsc, tze, args, plan.grid, stream)
                       : plan.nt == 16 ? launch_tc<16>(tq, tx, args, plan.grid, stream)
                                       : launch_tc<32>(tq, tx, args, plan.grid, stream);
        if (st != W4A16_OK) return st;
    }
    return W4A16_OK;
}

}  // namespace w4a16
