// Tensor-core GEMV for up to 32 tokens per launch on BF16 operands: the
// decode path for token counts where the integer GEMV's digit planes cost too
// many MMAs, and for quantisation groups of 32 and 64 ("Quantization I: int8,
// int4, the basics", Concept: dequantise tile by tile inside the multiply,
// groups of 32-128; "Weight-Only Quantization and Mixed Precision", sections 1,
// 5 and 8).
//
// Per unit (128 weight rows x 128 K of codes, 8 KB):
//  * eight dequantiser warps (two per row, half of its codes each) turn each
//    row's codes into BF16 (q - c) -- one
//    lop3 makes two BF16 values 128 + q from a packed word, one packed
//    subtraction removes 128 + c; exact, since |q - c| <= 256 -- and store the
//    row's 64 words to tensor memory (the A operand, 128 lanes x 64 columns),
//    with c = z when |z| <= 128 and c = 0 otherwise;
//  (scales and zero points arrive by TMA with the codes, in blocks of 8
//  quantisation groups x 128 rows, into a small ring of shared-memory slots;)
//  * one thread issues eight tcgen05.mma kind::f16 (M = 128, N = tokens,
//    K = 16), A from tensor memory, B = the tokens' BF16 activations (TMA,
//    128-byte swizzle, K-major), FP32 accumulation in tensor memory, one
//    accumulator per quantisation group;
//  * four fold warps take one row each per thread and apply the group's scale
//    to the FP32 sums: T += s D, or T += s (D - z sum_k x) for a row whose zero
//    point was not subtracted (|z| > 128).
// The products (q - c) x are exact in FP32 and the scale multiplies FP32
// partial sums, as in the GEMM.  The activations' K order is the one in which
// a packed word's codes come out of the lop3 (0, 4, 1, 5, 2, 6, 3, 7 in every
// 8-block): prep_bf_kernel writes X in that order with the per-group sums.
//
// Work decomposition as in the integer GEMVs (units dealt to a persistent grid
// in contiguous ranges, a row tile shared by CTAs written as partial-sum slots
// that decode_reduce_kernel adds); one CTA per SM, which owns all 512 tensor-
// memory columns.
#include "common.cuh"
#include "decode_units.cuh"
#include "sm100.cuh"

namespace w4a16 {
namespace {

constexpr int kRows = 128;
constexpr int kCodeBytes = kRows * kWordsPerGroup * 4;  // 8 KB per unit, 64-byte swizzle
constexpr int kFoldWarps = 4;                           // warps 0-3, TMEM lane quadrant = warp
constexpr int kDqWarps = 8;                             // warps 4-11: lane quadrant, half of the row's words
constexpr int kMmaWarp = kFoldWarps + kDqWarps;         // 12
constexpr int kTmaWarp = kMmaWarp + 1;                  // 13
constexpr int kThreads = (kTmaWarp + 1) * 32;           // 448
constexpr int kMetaGroups = 8;                          // quantisation groups per metadata block
constexpr int kScBytes = kRows * kMetaGroups * 2;       // 128 rows x 8 BF16 scales
constexpr int kMetaBytes = kScBytes + kRows * kMetaGroups * 4;  // + 128 rows x 8 int32 zero points

template <int NTOK, int GS>
struct BfCfg {
    static constexpr int SUB = kGroup / GS;                  // quantisation groups per 128-K unit
    static constexpr int kXBlock = NTOK * 128;               // X: one 64-K block (NTOK rows x 128 B, swizzled)
    static constexpr int kXBytes = 2 * kXBlock;              // the unit's 128 K
    static constexpr int kCodeOff = kXBytes;                 // 1024-aligned
    static constexpr int kXsOff = kCodeOff + kCodeBytes;
    static constexpr int kXsBytes = SUB * NTOK * 4;          // sum of x per quantisation group and token
    static constexpr int kStageBytes = (kXsOff + kXsBytes + 1023) & ~1023;
    static constexpr int kStages = (200 * 1024) / kStageBytes < 8 ? (200 * 1024) / kStageBytes : 8;
    static constexpr int kUnitsPerBlock = kMetaGroups / SUB;  // units per metadata block
    // a slot is rewritten when its block's last unit is at least kStages units behind the TMA thread
    static constexpr int kMetaSlots = 1 + (kStages + kUnitsPerBlock - 1) / kUnitsPerBlock;
    static constexpr int kMetaOff = kStages * kStageBytes;
    static constexpr size_t kSmem = (size_t)kMetaOff + (size_t)kMetaSlots * kMetaBytes + 1024;  // + alignment slack
    static constexpr int kACols = 64;                        // 128 rows x 128 BF16
    static constexpr int kNumA = 4;
    static constexpr uint32_t kColD = kNumA * kACols;        // accumulators after the A buffers
    static constexpr int kNumD = (512 - kNumA * kACols) / NTOK;  // accumulators of NTOK columns
    static constexpr int kMmaPerGroup = 8 / SUB;             // K = 16 per MMA
    static_assert(kXsBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
    static_assert(kNumD >= 2 * SUB, "two units' accumulators in flight");
};

struct BfArgs {
    const float* xs;       // [G][SUB][NTOK]: sums of the launch's activations per quantisation group
    uint16_t* Y;           // [M][N]
    float* partial;        // [row_tiles][max_slots][M][128]
    int* fault;
    int M, N, G;           // G: 128-K units per row (K / 128); scales and zeros have G * SUB columns (a multiple of 8)
    int units_base, units_rem;
    int max_slots;
};

__device__ __forceinline__ uint32_t magic_pair(uint32_t w) {  // (128 + q0, 128 + q4) as a BF16 pair
    uint32_t r;
    asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(w));  // (w & m) | c
    return r;
}

__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b) {  // exact for integers <= 256
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// (128 + c) as a BF16 pair for a zero point z: c = z when |z| <= 128 (subtracted exactly in the
// dequantiser), else 0 (the fold subtracts z sum x).
__device__ __forceinline__ uint32_t zero_pair(int z) {
    const int c = (z >= -128 && z <= 128) ? z : 0;
    const uint32_t cb = __float_as_uint(128.f + (float)c) >> 16;
    return cb | (cb << 16);
}

// One thread per (token m < NTOK, 128-K unit g, 8-block b): Xp (each 8-block in the order
// 0, 4, 1, 5, 2, 6, 3, 7) for m < M, and xs[g][sg][m] = sum over quantisation group sg (zero for
// m >= M).  xscale (nullable): each x is first replaced by bf16(x * xscale[k]) (AWQ).
template <int NTOK, int GS>
__global__ void __launch_bounds__(256) prep_bf_kernel(const uint16_t* __restrict__ X, const float* __restrict__ xscale,
                                                      int M, int K, uint16_t* __restrict__ Xp, float* __restrict__ xs) {
    constexpr int SUB = kGroup / GS, LPG = GS / 8;  // lanes (8-blocks) per quantisation group
    pdl_launch_dependents();
    pdl_wait_primary();  // X may come from the preceding kernel
    const int G = K / kGroup;
    const int64_t items = (int64_t)NTOK * G * 16;  // multiple of 16
    for (int64_t u0 = (int64_t)blockIdx.x * blockDim.x; u0 < items; u0 += (int64_t)gridDim.x * blockDim.x) {
        const int64_t u = u0 + threadIdx.x;
        const bool active = u < items;
        const int64_t mg = u >> 4;
        const int blk = (int)(u & 15);
        const int m = (int)(mg / G), g = (int)(mg - (int64_t)m * G);
        float sum = 0.f;
        if (active && m < M) {
            const int64_t off = (int64_t)m * K + (int64_t)g * kGroup + blk * 8;
            uint4 v = *reinterpret_cast<const uint4*>(X + off);
            if (xscale) {
                const float4* r = reinterpret_cast<const float4*>(xscale + (int64_t)g * kGroup + blk * 8);
                const float4 r0 = __ldg(r), r1 = __ldg(r + 1);
                v = make_uint4(bf16x2_scaled(v.x, r0.x, r0.y), bf16x2_scaled(v.y, r0.z, r0.w),
                               bf16x2_scaled(v.z, r1.x, r1.y), bf16x2_scaled(v.w, r1.z, r1.w));
            }
            uint4 o;
            o.x = __byte_perm(v.x, v.z, 0x5410);  // x0, x4
            o.y = __byte_perm(v.x, v.z, 0x7632);  // x1, x5
            o.z = __byte_perm(v.y, v.w, 0x5410);  // x2, x6
            o.w = __byte_perm(v.y, v.w, 0x7632);  // x3, x7
            *reinterpret_cast<uint4*>(Xp + off) = o;
            auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
            auto hi = [](uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); };
            sum = (lo(v.x) + hi(v.x)) + (lo(v.y) + hi(v.y)) + (lo(v.z) + hi(v.z)) + (lo(v.w) + hi(v.w));
        }
        // the lanes of one quantisation group are LPG consecutive lanes of one (m, g) block of 16
#pragma unroll
        for (int o = LPG / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (active && blk % LPG == 0) xs[((int64_t)g * SUB + blk / LPG) * NTOK + m] = sum;
    }
}

template <int NTOK, int GS>
__global__ void __launch_bounds__(kThreads, 1) decode_bf_kernel(const __grid_constant__ CUtensorMap tq,
                                                                const __grid_constant__ CUtensorMap tx,
                                                                const __grid_constant__ CUtensorMap tsc,
                                                                const __grid_constant__ CUtensorMap tze,
                                                                const BfArgs a) {
    using C = BfCfg<NTOK, GS>;
    constexpr int S = C::kStages, NA = C::kNumA, ND = C::kNumD, SUB = C::SUB;
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, NTOK);
    constexpr int UPB = C::kUnitsPerBlock, NS = C::kMetaSlots;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[S], empty[S], afull[NA], afree[NA], mdone[ND], dfree[ND];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_issued;

    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-aligned stages
    unsigned char* meta = ring + C::kMetaOff;                                // NS slots of kMetaBytes

    pdl_launch_dependents();  // the next call may start its weight loads as this grid's CTAs retire
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int64_t u_first = (int64_t)b * a.units_base + min(b, a.units_rem);
    const int nunits = a.units_base + (b < a.units_rem ? 1 : 0);
    const int G = a.G, N = a.N, M = a.M;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDqWarps + 1 + kFoldWarps);  // dequantisers, MMA commit, fold warps (sums)
        }
        for (int i = 0; i < NA; ++i) {
            mbar_init(&afull[i], kDqWarps);
            mbar_init(&afree[i], 1);
        }
        for (int i = 0; i < ND; ++i) {
            mbar_init(&mdone[i], 1);
            mbar_init(&dfree[i], kFoldWarps);
        }
        s_issued = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&s_tmem, 512);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == kTmaWarp) {  // ------------------------------------------------------------ TMA
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tx);
            prefetch_tmap(&tsc);
            prefetch_tmap(&tze);
            constexpr uint32_t kTx = C::kXBytes + kCodeBytes + C::kXsBytes;
            const int pre = min(S, nunits);
            int mb = -1;
            // codes of unit i and, with the first unit of a block of 8 quantisation groups, the block's scales
            // and zero points into slot mb % NS
            auto codes_meta = [&](int i, const UnitCursor& c) {
                const int s = i % S;
                const bool new_block = i == 0 || c.g % UPB == 0;
                if (new_block) ++mb;
                mbar_arrive_expect_tx(&full[s], kTx + (new_block ? kMetaBytes : 0));
                tma_load_2d(ring + s * C::kStageBytes + C::kCodeOff, &tq, c.g * kWordsPerGroup, c.tile * kRows, &full[s]);
                if (new_block) {
                    unsigned char* ms = meta + (mb % NS) * kMetaBytes;
                    const int gq8 = (c.g * SUB) & ~(kMetaGroups - 1);
                    tma_load_2d(ms, &tsc, gq8, c.tile * kRows, &full[s]);
                    tma_load_2d(ms + kScBytes, &tze, gq8, c.tile * kRows, &full[s]);
                }
            };
            // the weights do not depend on the preparation kernel: start streaming them at once
            UnitCursor cur(u_first, G);
            for (int i = 0; i < pre; ++i, cur.next(G)) codes_meta(i, cur);
            pdl_wait_primary();  // X and its sums come from the preparation kernel
            UnitCursor cx(u_first, G);
            for (int i = 0; i < pre; ++i, cx.next(G)) {
                unsigned char* st = ring + i * C::kStageBytes;
                tma_load_2d(st, &tx, cx.g * kGroup, 0, &full[i]);
                tma_load_2d(st + C::kXBlock, &tx, cx.g * kGroup + 64, 0, &full[i]);
                bulk_load(st + C::kXsOff, a.xs + (int64_t)cx.g * SUB * NTOK, C::kXsBytes, &full[i]);
            }
            int issued = pre;
            for (int i = pre; i < nunits; ++i, cur.next(G)) {
                const int s = i % S;
                if (!mbar_wait(&empty[s], ((i / S) - 1) & 1, a.fault, 131)) break;
                unsigned char* st = ring + s * C::kStageBytes;
                codes_meta(i, cur);
                tma_load_2d(st, &tx, cur.g * kGroup, 0, &full[s]);
                tma_load_2d(st + C::kXBlock, &tx, cur.g * kGroup + 64, 0, &full[s]);
                bulk_load(st + C::kXsOff, a.xs + (int64_t)cur.g * SUB * NTOK, C::kXsBytes, &full[s]);
                ++issued;
            }
            // every copy issued must land before the CTA may exit
            for (int i = max(0, issued - S); i < issued; ++i) mbar_wait(&full[i % S], (i / S) & 1, a.fault, 132);
        }
        return;
    }

    if (warp == kMmaWarp) {  // -------------------------------------------------------- MMA issue
        if (lane == 0) {
            for (int i = 0; i < nunits; ++i) {
                const int s = i % S, ai = i % NA;
                if (!mbar_wait(&afull[ai], (i / NA) & 1, a.fault, 141)) break;
                if (!mbar_wait(&full[s], (i / S) & 1, a.fault, 142)) break;
                bool ok = true;
#pragma unroll
                for (int sg = 0; sg < SUB; ++sg) {  // accumulator jd = i SUB + sg, freed by the fold
                    const int jd = i * SUB + sg;
                    if (jd >= ND && !mbar_wait(&dfree[jd % ND], ((jd / ND) - 1) & 1, a.fault, 143)) ok = false;
                }
                if (!ok) break;
                tc_fence_after();
                const uint32_t xaddr = smem_u32(ring + s * C::kStageBytes);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int sg = kk / C::kMmaPerGroup, di = (i * SUB + sg) % ND;
                    const uint64_t bd = sw128_kmajor_desc(xaddr + (kk >> 2) * C::kXBlock + (kk & 3) * 32);
                    umma_ts(tmem + C::kColD + di * NTOK, tmem + ai * C::kACols + kk * 8, bd, kIdesc,
                            (kk % C::kMmaPerGroup) != 0);
                    if ((kk + 1) % C::kMmaPerGroup == 0) umma_commit(&mdone[di]);
                }
                umma_commit(&afree[ai]);
                umma_commit(&empty[s]);
                s_issued = i + 1;
            }
        }
        return;
    }

    if (warp >= kFoldWarps) {  // ------------------------------------------------ dequantisers
        const int quad = (warp - kFoldWarps) & 3, half = (warp - kFoldWarps) >> 2;
        const int row_local = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const int sw = (row_local >> 1) & 3;  // 64-byte swizzle of the codes tile
        UnitCursor zc(u_first, G);
        int mb = -1;
        for (int i = 0; i < nunits; ++i, zc.next(G)) {
            if (i == 0 || zc.g % UPB == 0) ++mb;
            const int s = i % S, ai = i % NA;
            if (i >= NA && !mbar_wait(&afree[ai], ((i / NA) - 1) & 1, a.fault, 151)) break;
            if (!mbar_wait(&full[s], (i / S) & 1, a.fault, 152)) break;
            // the zero points of this half's words (quantisation groups (8 half .. 8 half + 7) / (GS / 8)) from
            // the block's slot; rows past N were zero-filled (c = 0)
            const int* zrow = reinterpret_cast<const int*>(meta + (mb % NS) * kMetaBytes + kScBytes +
                                                           row_local * (kMetaGroups * 4)) +
                              ((zc.g * SUB) & (kMetaGroups - 1));
            const int q0 = GS == 32 ? 2 * half : (GS == 64 ? half : 0);
            const uint32_t c2a = zero_pair(zrow[q0]), c2b = GS == 32 ? zero_pair(zrow[q0 + 1]) : c2a;
            // this half's 8 words (chunks 2 half, 2 half + 1); logical 16-byte chunk q of row r sits at chunk
            // q ^ ((r >> 1) & 3)
            const unsigned char* codes = ring + s * C::kStageBytes + C::kCodeOff + row_local * 64;
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint4 v = *reinterpret_cast<const uint4*>(codes + 16 * ((2 * half + q) ^ sw));
                w[4 * q] = v.x;
                w[4 * q + 1] = v.y;
                w[4 * q + 2] = v.z;
                w[4 * q + 3] = v.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // word j (codes 8j .. 8j + 7) -> columns 4j .. 4j + 3 holding the pairs (q0, q4), (q1, q5),
            // (q2, q6), (q3, q7), each minus its c
            uint32_t pr[32];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const uint32_t x = w[jj], c2 = jj < 4 ? c2a : c2b;
                pr[4 * jj] = sub_bf16x2(magic_pair(x), c2);
                pr[4 * jj + 1] = sub_bf16x2(magic_pair(x >> 4), c2);
                pr[4 * jj + 2] = sub_bf16x2(magic_pair(x >> 8), c2);
                pr[4 * jj + 3] = sub_bf16x2(magic_pair(x >> 12), c2);
            }
            tmem_st32(tl + ai * C::kACols + 32 * half, pr);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[ai]);
        }
        return;
    }

    // --------------------------------------------------------------------------- fold warps 0-3
    const int quad = warp;
    const int row_local = quad * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    float acc[NTOK];
#pragma unroll
    for (int m = 0; m < NTOK; ++m) acc[m] = 0.f;
    bool aborted = false;
    int cur_tile = (int)(u_first / G);

    // A row tile leaves the CTA as Y (all of its units here) or as this CTA's partial-sum slot.
    auto flush = [&](int tile) {
        const int first = cta_of_unit((int64_t)tile * G, a.units_base, a.units_rem);
        const int last = cta_of_unit((int64_t)tile * G + G - 1, a.units_base, a.units_rem);
        const int n = tile * kRows + row_local;
        if (first == last) {
            if (n < N) {
#pragma unroll
                for (int m = 0; m < NTOK; ++m)
                    if (m < M) a.Y[(int64_t)m * N + n] = float_to_bf16_bits(acc[m]);
            }
        } else {
            float* part = a.partial + ((int64_t)tile * a.max_slots + (b - first)) * M * kRows;
#pragma unroll
            for (int m = 0; m < NTOK; ++m)
                if (m < M) part[m * kRows + row_local] = acc[m];
        }
#pragma unroll
        for (int m = 0; m < NTOK; ++m) acc[m] = 0.f;
    };

    UnitCursor fc(u_first, G);
    int mb = -1;
    for (int i = 0; i < nunits; ++i, fc.next(G)) {
        if (i == 0 || fc.g % UPB == 0) ++mb;
        const int tile = fc.tile;
        while (cur_tile < tile) flush(cur_tile++);
        if (aborted) continue;
        const int s = i % S;
        const float* xsum = reinterpret_cast<const float*>(ring + s * C::kStageBytes + C::kXsOff);
        // this row's scales and zero points from the block's slot (the MMA that this warp waits for
        // below was issued after the slot's copy completed); rows past N were zero-filled (s = 0)
        const unsigned char* ms = meta + (mb % NS) * kMetaBytes;
        const int gq = (fc.g * SUB) & (kMetaGroups - 1);
#pragma unroll
        for (int sg = 0; sg < SUB; ++sg) {
            const int jd = i * SUB + sg, di = jd % ND;
            if (!mbar_wait(&mdone[di], (jd / ND) & 1, a.fault, 161)) {
                aborted = true;
                break;
            }
            tc_fence_after();
            const float sv = bf16_bits_to_float(
                *reinterpret_cast<const uint16_t*>(ms + row_local * (kMetaGroups * 2) + 2 * (gq + sg)));
            const int zi = *reinterpret_cast<const int32_t*>(ms + kScBytes + row_local * (kMetaGroups * 4) + 4 * (gq + sg));
            const bool corr = !(zi >= -128 && zi <= 128);  // zero point left for the fold
            const bool any_corr = __any_sync(0xFFFFFFFFu, corr);
            const float zc = corr ? (float)zi : 0.f;
#pragma unroll
            for (int c0 = 0; c0 < NTOK; c0 += 16) {  // 16 tokens' sums at a time
                uint32_t d[16];
                tmem_ld16(tl + C::kColD + di * NTOK + c0, d);
                tmem_wait_ld();
                if (c0 + 16 == NTOK) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&dfree[di]);
                }
                if (any_corr) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        acc[c0 + e] =
                            fmaf(sv, fmaf(-zc, xsum[sg * NTOK + c0 + e], __uint_as_float(d[e])), acc[c0 + e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) acc[c0 + e] = fmaf(sv, __uint_as_float(d[e]), acc[c0 + e]);
                }
            }
        }
        if (aborted) continue;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // the stage's sums read
    }
    const int tile_last = nunits > 0 ? (int)((u_first + nunits - 1) / G) : cur_tile - 1;
    while (cur_tile <= tile_last) flush(cur_tile++);

    // teardown: every MMA issued must be complete before the columns are released
    named_barrier_sync(1, kFoldWarps * 32);
    if (warp == 0) {
        if (aborted) {
            const int issued = s_issued;
            for (int j = max(0, issued * SUB - ND); j < issued * SUB; ++j)
                mbar_wait(&mdone[j % ND], (j / ND) & 1, a.fault, 162);
        }
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int NTOK, int GS>
int bf_occupancy() {
    static PerContext<int> cache;  // the attribute belongs to a context
    return cache.get([]() -> int {
        if (cudaFuncSetAttribute(decode_bf_kernel<NTOK, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)BfCfg<NTOK, GS>::kSmem) != cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, decode_bf_kernel<NTOK, GS>, kThreads,
                                                          BfCfg<NTOK, GS>::kSmem) != cudaSuccess ||
            o < 1)
            return 0;
        return 1;  // one CTA per SM: it owns all 512 tensor-memory columns
    });
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BfPlan {
    int grid, units_base, units_rem, max_slots, row_tiles;
};

BfPlan plan_bf(int64_t N, int64_t K, int num_sms) {
    BfPlan p{};
    const int64_t G = K / kGroup;
    p.row_tiles = (int)ceil_div(N, kRows);
    const int64_t units = (int64_t)p.row_tiles * G;
    int64_t grid = num_sms;
    if (grid > units) grid = units;
    p.grid = (int)grid;
    p.units_base = (int)(units / grid);
    p.units_rem = (int)(units % grid);
    p.max_slots = (int)((G - 1) / p.units_base + 2);
    return p;
}

template <int NTOK, int GS>
int launch_bf_chunk(const uint16_t* X, const float* xscale, int Mc, int64_t K, const CUtensorMap& tq,
                    const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, char* scratch,
                    const BfPlan& p, int* fault, cudaStream_t stream) {
    if (bf_occupancy<NTOK, GS>() < 1) return W4A16_ERR_CUDA;
    const int G = (int)(K / kGroup);
    // scratch: [Xp bf16 Mc x K][xs fp32 G x SUB x NTOK][partials]
    uint16_t* Xp = reinterpret_cast<uint16_t*>(scratch);
    float* xs = reinterpret_cast<float*>(scratch + align256((size_t)Mc * K * 2));
    float* partial =
        reinterpret_cast<float*>(scratch + align256((size_t)Mc * K * 2) + align256((size_t)G * (kGroup / GS) * NTOK * 4));
    CUtensorMap tx;
    if (!tmap_2d_cached(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Xp, (uint64_t)K, (uint64_t)Mc, (uint64_t)K * 2, 64,
                        NTOK, CU_TENSOR_MAP_SWIZZLE_128B))
        return W4A16_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    {
        const int64_t items = (int64_t)NTOK * G * 16;
        int grid = (int)ceil_div(items, 256);
        if (grid > num_sms_current() * 8) grid = num_sms_current() * 8;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, prep_bf_kernel<NTOK, GS>, X, xscale, Mc, (int)K, Xp, xs) != cudaSuccess)
            return W4A16_ERR_CUDA;
    }
    BfArgs args;
    args.xs = xs;
    args.Y = Y;
    args.partial = partial;
    args.fault = fault;
    args.M = Mc;
    args.N = (int)N;
    args.G = G;
    args.units_base = p.units_base;
    args.units_rem = p.units_rem;
    args.max_slots = p.max_slots;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = BfCfg<NTOK, GS>::kSmem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int GQ = G * (kGroup / GS);  // quantisation groups per row
    CUtensorMap tsc, tze;
    if (!tmap_2d_cached(&tsc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, scales, (uint64_t)GQ, (uint64_t)N, (uint64_t)GQ * 2,
                        kMetaGroups, kRows) ||
        !tmap_2d_cached(&tze, CU_TENSOR_MAP_DATA_TYPE_INT32, zeros, (uint64_t)GQ, (uint64_t)N, (uint64_t)GQ * 4,
                        kMetaGroups, kRows))
        return W4A16_ERR_CUDA;
    if (cudaLaunchKernelEx(&cfg, decode_bf_kernel<NTOK, GS>, tq, tx, tsc, tze, args) != cudaSuccess)
        return W4A16_ERR_CUDA;
    return launch_decode_reduce(partial, Y, N, Mc, G, p.units_base, p.units_rem, p.max_slots, p.row_tiles, stream);
}

template <int GS>
int launch_bf_gs(int ntok, const uint16_t* X, const float* xscale, int Mc, int64_t K, const CUtensorMap& tq,
                 const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, char* scratch, const BfPlan& p,
                 int* fault, cudaStream_t stream) {
    return ntok == 16 ? launch_bf_chunk<16, GS>(X, xscale, Mc, K, tq, scales, zeros, N, Y, scratch, p, fault, stream)
                      : launch_bf_chunk<32, GS>(X, xscale, Mc, K, tq, scales, zeros, N, Y, scratch, p, fault, stream);
}

}  // namespace

size_t bf_workspace_bytes(int64_t M, int64_t N, int64_t K, int group, int num_sms) {
    const int64_t Mc = M < 32 ? M : 32;
    const int ntok = Mc <= 16 ? 16 : 32;
    const BfPlan p = plan_bf(N, K, num_sms);
    const int64_t G = K / kGroup;
    return align256((size_t)Mc * K * 2) + align256((size_t)G * (kGroup / group) * ntok * 4) +
           align256((size_t)p.row_tiles * p.max_slots * Mc * kRows * 4);
}

int launch_decode_bf(const uint16_t* X, const float* xscale, int64_t M, int64_t K, int group, const uint32_t* qweight,
                     const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* scratch,
                     cudaStream_t stream) {
    if ((K / group) % kMetaGroups != 0) return W4A16_ERR_SHAPE;  // metadata blocks of 8 quantisation groups
    CUtensorMap tq;
    if (!tmap_2d_cached(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)K / 8, (uint64_t)N, (uint64_t)K / 2,
                        kWordsPerGroup, kRows, CU_TENSOR_MAP_SWIZZLE_64B))
        return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    const BfPlan p = plan_bf(N, K, num_sms_current());
    for (int64_t m0 = 0; m0 < M; m0 += 32) {
        const int Mc = (int)(M - m0 < 32 ? M - m0 : 32);
        const int ntok = Mc <= 16 ? 16 : 32;
        const uint16_t* Xc = X + m0 * K;
        uint16_t* Yc = Y + m0 * N;
        char* sc = reinterpret_cast<char*>(scratch);
        const int st = group == 128  ? launch_bf_gs<128>(ntok, Xc, xscale, Mc, K, tq, scales, zeros, N, Yc, sc, p, fault, stream)
                       : group == 64 ? launch_bf_gs<64>(ntok, Xc, xscale, Mc, K, tq, scales, zeros, N, Yc, sc, p, fault, stream)
                                     : launch_bf_gs<32>(ntok, Xc, xscale, Mc, K, tq, scales, zeros, N, Yc, sc, p, fault, stream);
        if (st != W4A16_OK) return st;
    }
    return W4A16_OK;
}

}  // namespace w4a16
