// Decode path of the W4A16 linear layer: persistent split-K GEMVs for small M
// (up to 32 tokens per launch; more in consecutive launches).
//
// Only the packed codes (0.5 byte per weight) and the per-group scale and zero
// point cross the memory bus; each code is consumed on chip straight from its
// packed word ("Quantization I: int8, int4, the basics", Concept: dequantise
// tile by tile inside the multiply; "Weight-Only Quantization and Mixed
// Precision", section 7: one read of the packed INT4 weights, unpack with bit
// operations, asynchronous copies overlapping the math, nothing written back).
//
// Arithmetic per group g of 128 weights of row n and token m, exact in integers:
//   sum_k (q - z) s x  =  s 2^(-k) ( sum_k q x_int  -  z sum_k x_int ),
// x_int = x 2^k an integer (k from the exponent of the group's largest |x|).
// The codes q stay unsigned bytes (w & 0x0F0F0F0F, (w >> 4) & 0x0F0F0F0F); x_int
// is written as three signed base-256 digits, so sum_k q x_int is three exact
// int32 dot products, combined and scaled in FP32 once per group.  The BF16 scale
// is never folded into a rounded operand.  In this file:
//   * M = 1: decode_cc_kernel, the dot products as mma.sync m16n8k32 (codes u8 x
//     X digits s8) in the warps' registers, X prepared inside the kernel, and
//     decode_cc_reduce_kernel for its split-K sums;
//   * 17 or more tokens (32 per launch), and any M when K / 128 is not a
//     multiple of 8: decode_tc_kernel, tcgen05.mma kind::i8 with the codes in
//     tensor memory and the digit planes of all tokens as B;
//   * prep_x8_kernel: the digit planes for the tensor-core kernel.
// 2-16 tokens run the register-MMA GEMV of gemv_mt.cu; groups of 32 and 64
// run gemv_sub.cu (one token) and gemv_bf.cu (more).
// With AWQ inverse channel scales (the activation half of the equivalence
// transform), X' = bf16(x * inv_s[k]) is formed where X is prepared: inside
// prep_x8_kernel, and for M = 1 by awq_prescale_kernel ahead of the integer
// kernel, which then reads X' (doing it in the kernel's single X warp made
// that warp the bottleneck).
//
// Work decomposition: a unit is 128 weight rows x one group (8 KB of codes).
// The tensor-core kernel deals units, numbered row tile by row tile, to a
// persistent grid in contiguous, equal ranges (+-1 unit), and a row tile split
// between CTAs is reduced by the last CTA to finish its part (arrival counter);
// the one-token kernel hands out chunks of 2 or 4 units from a counter and a
// dependent reduction kernel adds the chunks' partial sums.  Either way the
// partials are summed in a fixed order.
#include "common.cuh"
#include "decode_units.cuh"
#include "sm100.cuh"

#include <mutex>

namespace w4a16 {
namespace {

constexpr int kRowsPerCta = 128;
constexpr int kStageWords = kRowsPerCta * kWordsPerGroup;  // 2048 words = 8 KB
constexpr int kMaxTokens = 32;  // tokens per launch
// Token counts up to this take the integer mma.sync GEMV (when K / 128 is a multiple of 8): its MMAs grow
// with 3 digit planes per token; at 9-16 tokens it still beats the tcgen05 GEMV by 8-18 % (gate+up and down
// at hidden size 8192), and the tcgen05 GEMV takes 17-32 tokens per launch.
constexpr int64_t kMtMaxTokens = 16;

struct DecodeArgs {
    const uint16_t* Xp;  // [Mc][K] BF16, 8-blocks reordered (0,4,1,5,2,6,3,7); the input X itself for M = 1
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


// --------------------------------------------------------------------------
// Tensor-core decode kernel (tcgen05, 8-bit integer MMA), one persistent CTA
// per SM, for up to 32 tokens per launch (17 or more tokens; any count when
// K / 128 is not a multiple of 8).
//
// The codes are the A operand as unsigned bytes, exactly: per packed word,
// w & 0x0F0F0F0F holds codes 0, 2, 4, 6 and (w >> 4) & 0x0F0F0F0F codes
// 1, 3, 5, 7, and a dequantiser thread stores its row's 32 such words into
// tensor memory (K order (0,2,4,6,1,3,5,7) in every 8-block).  X is the B
// operand as signed bytes: per group and token, x_int = x * 2^(21 - E) (E the
// exponent of the group's largest |x|; exact for every x within 2^14 of it,
// smaller values rounded at 2^(E - 21)) is written in balanced base 256,
// x_int = 65536 d2 + 256 d1 + d0 with every digit in [-128, 127], and the
// three digit planes of NTOK tokens are the 3 NTOK rows of B.  One
// tcgen05.mma kind::i8 (M = 128, N = 3 NTOK, K = 32) thus takes 32 codes of
// every row against all planes of all tokens, with exact int32 sums; a unit
// (128 rows x one group) is four MMAs, half the instructions of BF16 operands.
// The fold warps combine the planes and apply scale and zero point in FP32:
//   acc += s 2^(E - 21) (65536 D2 + 256 D1 + D0 - z sum_k x_int).
//
// Warp roles (448 threads): 0-7 fold (warp w: TMEM lane quadrant w % 4, half
// w / 4 of the tokens; also the row tile epilogue), 8-11 dequantise, 12 issues
// the MMAs, 13 drives TMA.  Rings:
// shared-memory stages (codes, X planes, per token X sums and scales), 4 A
// buffers and 8 (NTOK = 16) or 4 (NTOK = 32) accumulators, each with a
// full/free mbarrier pair, and (K / 128 a multiple of 8) three slots of
// scale and zero-point blocks that TMA fills with the codes (per-row loads
// of the fold warps otherwise: 9-12 % slower on 24 and 32 tokens).

// X planes of one launch, prepared by prep_x8_kernel: for group g, row
// p NTOK + m of the B tile holds digit plane p of token m (128 bytes, MMA K
// order); xs holds per group [sum_k x_int (FP32) for each token, then
// 2^(E - 21) for each token].
// Scales and zero points: with TM (K / 128 a multiple of 8, so that their
// rows are 16-byte aligned) TMA brings them with the codes, in blocks of 8
// groups x 128 rows (2 KB of BF16 scales, then 4 KB of int32 zero points),
// into a ring of kMetaSlots shared-memory slots: block b of a CTA's range
// goes to slot b % kMetaSlots with the first unit of the block; otherwise
// the fold warps load their rows' values from global memory, a few units
// ahead.
constexpr int kTcMetaGroups = 8;
constexpr int kTcScBytes = 128 * kTcMetaGroups * 2;
constexpr int kTcMetaBytes = kTcScBytes + 128 * kTcMetaGroups * 4;  // 6 KB
template <int NTOK, bool TM>
struct TcCfg {
    static constexpr int kBRows = 3 * NTOK;                  // MMA N
    static constexpr int kBBytes = kBRows * 128;             // one group of K, 128-byte swizzle
    static constexpr int kCodeOff = kBBytes;                 // 1024-aligned
    static constexpr int kXsOff = kCodeOff + kStageWords * 4;
    static constexpr int kXsBytes = 2 * NTOK * 4;
    static constexpr int kStageBytes = (kXsOff + kXsBytes + 1023) & ~1023;
    static constexpr int kMetaSlots = TM ? 3 : 0;
    static constexpr int kStages = (220 * 1024 - kMetaSlots * kTcMetaBytes) / kStageBytes;
    static constexpr int kMetaOff = kStages * kStageBytes;
    static constexpr size_t kSmem = (size_t)kMetaOff + (size_t)kMetaSlots * kTcMetaBytes + 1024;  // + alignment slack
    // A block's slot is rewritten kMetaSlots blocks later, with the first unit of that block; the blocks in
    // between hold 8 units each (blocks are aligned to 8 groups inside a row tile), and the TMA thread issues
    // a unit only once the fold is done with the unit kStages back.
    static_assert(!TM || 8 * (kMetaSlots - 1) >= kStages - 1, "metadata slot reuse");
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kACols = 32;                        // 128 rows x 128 bytes
    static constexpr int kNumA = 4;                          // A buffers at 0..127
    static constexpr uint32_t kColD = kNumA * kACols;
    static constexpr int kNumD = (512 - kNumA * kACols) / kBRows;  // accumulators of kBRows columns
};

// Instruction descriptor, kind::i8: A unsigned 8-bit, B signed 8-bit, D s32, both K-major.
__host__ __device__ constexpr uint32_t idesc_u8s8_s32(int M, int N) {
    return (2u << 4)                          // D format: S32
           | (0u << 7)                        // A format: unsigned 8-bit
           | (1u << 10)                       // B format: signed 8-bit
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// D[tmem] (+)= A[tmem] x B[smem desc]; kind::i8, int32 accumulate.
__device__ __forceinline__ void umma_ts_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// One warp per (group g, token m < NTOK): lane l holds x at k = 4l .. 4l + 3 (word w = l / 2,
// half h = l % 2).  Tokens m >= M get zero planes.
// xscale (nullable): each x is first replaced by bf16(x * xscale[k]) (the AWQ activation transform).
template <int NTOK>
__global__ void __launch_bounds__(256) prep_x8_kernel(const uint16_t* __restrict__ X, const float* __restrict__ xscale,
                                                      int M, int K, uint8_t* __restrict__ planes,
                                                      float* __restrict__ xs) {
    pdl_launch_dependents();
    const int G = K / kGroup;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)G * NTOK;
    for (int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid < warps;
         wid += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int g = (int)(wid / NTOK), m = (int)(wid - (int64_t)g * NTOK);
        uint32_t bits[4] = {0u, 0u, 0u, 0u};
        if (m < M) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(X + (int64_t)m * K + (int64_t)g * kGroup + lane * 4));
            bits[0] = v.x & 0xFFFFu;
            bits[1] = v.x >> 16;
            bits[2] = v.y & 0xFFFFu;
            bits[3] = v.y >> 16;
            if (xscale) {
                const float4 r = __ldg(reinterpret_cast<const float4*>(xscale + (int64_t)g * kGroup + lane * 4));
                bits[0] = bf16_scaled(bits[0], r.x);
                bits[1] = bf16_scaled(bits[1], r.y);
                bits[2] = bf16_scaled(bits[2], r.z);
                bits[3] = bf16_scaled(bits[3], r.w);
            }
        }
        uint32_t amax = max(max(bits[0] & 0x7FFFu, bits[1] & 0x7FFFu), max(bits[2] & 0x7FFFu, bits[3] & 0x7FFFu));
        amax = __reduce_max_sync(0xFFFFFFFFu, amax);
        const int ef = (int)(amax >> 7);
        const int E = ef == 0 ? -127 : ef - 127;  // every |x| of the group is below 2^(E + 1)
        const int kx = 21 - E;                    // in [-106, 148]
        const int k1 = min(kx, 127);
        const float s1 = pow2f(k1), s2 = pow2f(kx - k1);  // exact scalings, |x * 2^kx| < 2^22
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
        // word w's 8 MMA-order bytes: [h0.i0, h0.i2, h1.i0, h1.i2, h0.i1, h0.i3, h1.i1, h1.i3]
        const int h = lane & 1, w = lane >> 1;
#pragma unroll
        for (int p = 0; p < 3; ++p) {
            const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, dg[p], 1);
            const uint32_t lo = h ? other : dg[p], hi = h ? dg[p] : other;  // halves of lanes h = 0 and 1
            const uint32_t out = h ? __byte_perm(lo, hi, 0x7632) : __byte_perm(lo, hi, 0x5410);
            *reinterpret_cast<uint32_t*>(planes + ((int64_t)g * 3 * NTOK + p * NTOK + m) * 128 + 8 * w + 4 * h) = out;
        }
        const int sum = __reduce_add_sync(0xFFFFFFFFu, (xi[0] + xi[1]) + (xi[2] + xi[3]));  // |sum| < 2^29
        if (lane == 0) {
            xs[(int64_t)g * 2 * NTOK + m] = (float)sum;
            xs[(int64_t)g * 2 * NTOK + NTOK + m] = pow2f(E - 21);
        }
    }
}

constexpr int kFoldWarps = 8;                    // two per TMEM lane quadrant, each with half the tokens
constexpr int kDqWarps = 4;
constexpr int kMmaWarp = kFoldWarps + kDqWarps;  // 12
constexpr int kTmaWarp = kMmaWarp + 1;           // 13
constexpr int kTcThreads = (kTmaWarp + 1) * 32;  // 448

template <int NTOK, bool TM>
__global__ void __launch_bounds__(kTcThreads, 1) decode_tc_kernel(const __grid_constant__ CUtensorMap tq,
                                                                  const __grid_constant__ CUtensorMap tx,
                                                                  const __grid_constant__ CUtensorMap tsc,
                                                                  const __grid_constant__ CUtensorMap tze,
                                                                  const DecodeArgs a) {
    using C = TcCfg<NTOK, TM>;
    constexpr int NS = C::kMetaSlots;
    constexpr int S = C::kStages;
    constexpr int NA = C::kNumA, ND = C::kNumD;
    constexpr uint32_t kIdesc = idesc_u8s8_s32(128, C::kBRows);
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[S], empty[S], afull[NA], afree[NA], mdone[ND], dfree[ND];
    __shared__ uint32_t s_tmem;
    __shared__ int s_last;
    __shared__ volatile int s_issued;
    __shared__ float s_split[kRowsPerCta * (NTOK / 2)];  // odd fold warps' row-tile sums (alternate units)

    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-aligned stages
    unsigned char* meta = ring + C::kMetaOff;                                // NS metadata slots (TM)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int64_t u_first = (int64_t)b * a.units_base + min(b, a.units_rem);
    const int nunits = a.units_base + (b < a.units_rem ? 1 : 0);
    const int G = a.G;

    // With at most NTOK / 2 tokens the second token half of the fold has nothing to do: the two fold
    // warps of a lane quadrant then take alternate units instead (four fold warps read each unit).
    const bool split_units = a.M <= NTOK / 2;
    const int unit_folders = split_units ? kFoldWarps / 2 : kFoldWarps;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4 + 1 + unit_folders);  // dequantiser set, MMA commit, fold warps (X sums)
        }
        for (int i = 0; i < NA; ++i) {
            mbar_init(&afull[i], 4);
            mbar_init(&afree[i], 1);
        }
        for (int i = 0; i < ND; ++i) {
            mbar_init(&mdone[i], 1);
            mbar_init(&dfree[i], unit_folders);
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
            if constexpr (TM) {
                prefetch_tmap(&tsc);
                prefetch_tmap(&tze);
            }
            constexpr uint32_t kTx = C::kBBytes + kStageWords * 4 + C::kXsBytes;
            const int pre = min(S, nunits);
            int mb = -1;  // metadata blocks started (TM)
            // codes of unit i into stage s and, with the first unit of a block of 8 groups, the block's scales
            // and zero points into slot mb % NS
            auto codes_meta = [&](int i, int s, const UnitCursor& c) {
                const bool new_block = TM && (i == 0 || (c.g & (kTcMetaGroups - 1)) == 0);
                if (new_block) ++mb;
                mbar_arrive_expect_tx(&full[s], kTx + (new_block ? kTcMetaBytes : 0));
                tma_load_2d(ring + s * C::kStageBytes + C::kCodeOff, &tq, c.g * kWordsPerGroup, c.tile * kRowsPerCta,
                            &full[s]);
                if constexpr (TM) {
                    if (new_block) {
                        unsigned char* ms = meta + (mb % NS) * kTcMetaBytes;
                        const int g8 = c.g & ~(kTcMetaGroups - 1);
                        tma_load_2d(ms, &tsc, g8, c.tile * kRowsPerCta, &full[s]);
                        tma_load_2d(ms + kTcScBytes, &tze, g8, c.tile * kRowsPerCta, &full[s]);
                    }
                }
            };
            // the weights do not depend on the preparation kernel: start streaming them at once
            UnitCursor cur(u_first, G);
            for (int i = 0; i < pre; ++i, cur.next(G)) codes_meta(i, i, cur);
            pdl_wait_primary();  // X planes come from the preparation kernel
            UnitCursor cx(u_first, G);
            for (int i = 0; i < pre; ++i, cx.next(G)) {
                const int g = cx.g;
                unsigned char* st = ring + i * C::kStageBytes;
                tma_load_2d(st, &tx, 0, g * C::kBRows, &full[i]);
                bulk_load(st + C::kXsOff, a.xs + (int64_t)g * 2 * NTOK, C::kXsBytes, &full[i]);
            }
            int issued = pre;
            for (int i = pre; i < nunits; ++i, cur.next(G)) {
                const int s = i % S;
                if (!mbar_wait(&empty[s], ((i / S) - 1) & 1, a.fault, 21)) break;
                const int g = cur.g;
                unsigned char* st = ring + s * C::kStageBytes;
                codes_meta(i, s, cur);
                tma_load_2d(st, &tx, 0, g * C::kBRows, &full[s]);
                bulk_load(st + C::kXsOff, a.xs + (int64_t)g * 2 * NTOK, C::kXsBytes, &full[s]);
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
                const uint32_t baddr = smem_u32(ring + s * C::kStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // K = 32 bytes per MMA: 32 bytes along the swizzled row
                    umma_ts_i8(tmem + C::kColD + di * C::kBRows, tmem + ai * C::kACols + kk * 8,
                               sw128_kmajor_desc(baddr + kk * 32), kIdesc, kk > 0);
                umma_commit(&afree[ai]);
                umma_commit(&mdone[di]);
                umma_commit(&empty[s]);
                s_issued = i + 1;
            }
        }
        return;
    }

    if (warp >= kFoldWarps) {  // ---------------------------------- dequantisers
        const int quad = warp & 3;                        // TMEM lane quadrant (warps 8-11: 0-3)
        const int row_local = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const int sw = (row_local >> 1) & 3;              // 64-byte swizzle of the codes tile
        for (int i = 0; i < nunits; ++i) {
            const int s = i % S, ai = i % NA;
            if (i >= NA && !mbar_wait(&afree[ai], ((i / NA) - 1) & 1, a.fault, 41)) break;
            if (!mbar_wait(&full[s], (i / S) & 1, a.fault, 42)) break;
            // logical 16-byte chunk q of row r sits at chunk q ^ ((r >> 1) & 3): conflict-free reads
            const unsigned char* codes = ring + s * C::kStageBytes + C::kCodeOff + row_local * 64;
            uint32_t pr[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 v = *reinterpret_cast<const uint4*>(codes + 16 * (q ^ sw));
                const uint32_t wq[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    pr[2 * (4 * q + j)] = wq[j] & 0x0F0F0F0Fu;             // codes 0, 2, 4, 6
                    pr[2 * (4 * q + j) + 1] = (wq[j] >> 4) & 0x0F0F0F0Fu;  // codes 1, 3, 5, 7
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            tmem_st32(tl + ai * C::kACols, pr);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[ai]);
        }
        return;
    }

    // ------------------------------------------------------- fold warps 0-7
    constexpr int TH = NTOK / 2;                  // tokens per fold thread
    const int quad = warp & 3, th = warp >> 2;    // lane quadrant, token half (or unit parity)
    const int row_local = quad * 32 + lane;
    const int m_base = split_units ? 0 : th * TH;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const int N = a.N, M = a.M;
    float acc[TH];
#pragma unroll
    for (int m = 0; m < TH; ++m) acc[m] = 0.f;
    bool aborted = false;
    int cur_tile = (int)(u_first / G);  // the row tile acc accumulates

    // One row tile's sums leave the CTA (every fold thread calls this once per row tile of the CTA's
    // range, in order).  With alternate units, the odd warps' sums are added to the even warps'.
    auto flush = [&](int tile) {
        if (split_units) {
            if (th == 1) {
#pragma unroll
                for (int e = 0; e < TH; ++e) s_split[e * kRowsPerCta + row_local] = acc[e];
            }
            named_barrier_sync(1, kFoldWarps * 32);
            if (th == 0) {
#pragma unroll
                for (int e = 0; e < TH; ++e) acc[e] += s_split[e * kRowsPerCta + row_local];
            }
        }
        const bool writer = !split_units || th == 0;
        const int n = tile * kRowsPerCta + row_local;
        const int first = cta_of_unit((int64_t)tile * G, a.units_base, a.units_rem);
        const int last = cta_of_unit((int64_t)tile * G + G - 1, a.units_base, a.units_rem);
        if (first == last) {
            if (n < N && writer) {
#pragma unroll
                for (int e = 0; e < TH; ++e)
                    if (m_base + e < M) a.Y[(int64_t)(m_base + e) * N + n] = float_to_bf16_bits(acc[e]);
            }
            if (split_units) named_barrier_sync(1, kFoldWarps * 32);  // s_split is reused by the next tile
        } else {
            const int slot = b - first, nseg = last - first + 1;
            float* part = a.partial + ((int64_t)tile * a.max_slots + slot) * M * kRowsPerCta;
            if (writer) {
#pragma unroll
                for (int e = 0; e < TH; ++e)
                    if (m_base + e < M) part[(m_base + e) * kRowsPerCta + row_local] = acc[e];
            }
            named_barrier_sync(1, kFoldWarps * 32);
            if (threadIdx.x == 0) s_last = (arrive_acq_rel_gpu(&a.counters[tile]) == nseg - 1);
            named_barrier_sync(1, kFoldWarps * 32);
            if (s_last) {
                const int rows = min(kRowsPerCta, N - tile * kRowsPerCta);
                const float* pb = a.partial + (int64_t)tile * a.max_slots * M * kRowsPerCta;
                for (int idx = threadIdx.x; idx < M * rows; idx += kFoldWarps * 32) {
                    const int m = idx / rows, rl = idx - m * rows;
                    const float sum = sum_slots(pb + (int64_t)m * kRowsPerCta + rl, (int64_t)M * kRowsPerCta, nseg);
                    a.Y[(int64_t)m * N + tile * kRowsPerCta + rl] = float_to_bf16_bits(sum);
                }
                if (threadIdx.x == 0) a.counters[tile] = 0;
            }
            named_barrier_sync(1, kFoldWarps * 32);
        }
#pragma unroll
        for (int e = 0; e < TH; ++e) acc[e] = 0.f;
    };

    // scale and zero point of this thread's row, one unit ahead
    // raw loads, converted only when used, so that nothing waits on them before then; the row is
    // clamped into the matrix (rows past N, and units past the last, are masked at use)
    auto load_meta = [&](int tile, int g, uint32_t& sraw, int& zraw) {
        const int n = min(tile * kRowsPerCta + row_local, N - 1);
        sraw = __ldg(a.scales + (int64_t)n * G + g);
        zraw = __ldg(a.zeros + (int64_t)n * G + g);
    };

    // unit j of row tile `tile`; sv, zv: its scale and zero point, or (TM) read here from metadata slot
    // `slot`, group g (the MMA waited for below was issued after the slot's copy landed; rows past N were
    // zero-filled: s = 0)
    auto fold_unit = [&](int j, int tile, float sv, float zv, int slot, int g) {
        while (cur_tile < tile) flush(cur_tile++);
        if (split_units && (j & 1) != th) return;  // the other warp of the quadrant folds this unit
        if (aborted) return;
        const int di = j % ND, s = j % S;
        if (!mbar_wait(&mdone[di], (j / ND) & 1, a.fault, 13)) {
            aborted = true;
            return;
        }
        tc_fence_after();
        if constexpr (TM) {
            const unsigned char* ms = meta + slot * kTcMetaBytes;
            const int gb = g & (kTcMetaGroups - 1);
            sv = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(ms + row_local * (kTcMetaGroups * 2) + 2 * gb));
            zv = (float)*reinterpret_cast<const int32_t*>(ms + kTcScBytes + row_local * (kTcMetaGroups * 4) + 4 * gb);
        }
        const float* xs = reinterpret_cast<const float*>(ring + s * C::kStageBytes + C::kXsOff);
        const uint32_t dcol = tl + C::kColD + di * C::kBRows + m_base;
        // integer -> FP32 by the 2^23 + 2^22 magic (exact for |v| < 2^22; every plane sum is: 128 codes of at
        // most 15 times digits of at most 128); the two low planes are first combined as the integer
        // 256 D1 + D0 (|.| < 2^27) and converted once -- the same rounding as the FP32 fma(D1, 256, D0) of the
        // exact plane values, one instruction for four
        auto to_f = [](uint32_t v) { return __int_as_float((int)v + 0x4B400000) - 12582912.f; };
#pragma unroll
        for (int h = 0; h < TH / 8; ++h) {  // 8 tokens at a time: their three digit planes
            uint32_t d0[8], d1[8], d2[8];
            tmem_ld8(dcol + h * 8, d0);
            tmem_ld8(dcol + NTOK + h * 8, d1);
            tmem_ld8(dcol + 2 * NTOK + h * 8, d2);
            tmem_wait_ld();
            if (h + 1 == TH / 8) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dfree[di]);
            }
            if (m_base + h * 8 >= M) continue;  // padding tokens only
            const float4 xs0 = *reinterpret_cast<const float4*>(xs + m_base + h * 8);
            const float4 xs1 = *reinterpret_cast<const float4*>(xs + m_base + h * 8 + 4);
            const float4 xc0 = *reinterpret_cast<const float4*>(xs + NTOK + m_base + h * 8);
            const float4 xc1 = *reinterpret_cast<const float4*>(xs + NTOK + m_base + h * 8 + 4);
            const float xsum[8] = {xs0.x, xs0.y, xs0.z, xs0.w, xs1.x, xs1.y, xs1.z, xs1.w};
            const float xsc[8] = {xc0.x, xc0.y, xc0.z, xc0.w, xc1.x, xc1.y, xc1.z, xc1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                // sum q x_int = 65536 D2 + 256 D1 + D0; the power of two last, so that a group of
                // tiny activations does not underflow in s 2^(E - 21)
                const float qx = fmaf(to_f(d2[e]), 65536.f, __int2float_rn((int)d1[e] * 256 + (int)d0[e]));
                acc[h * 8 + e] = fmaf(sv * fmaf(-zv, xsum[e], qx), xsc[e], acc[h * 8 + e]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // X sums and scales read
    };

    if constexpr (TM) {
        UnitCursor fc(u_first, G);
        int mb = -1;  // metadata block of unit j, counted as the TMA thread counts them
        for (int j = 0; j < nunits; ++j, fc.next(G)) {
            if (j == 0 || (fc.g & (kTcMetaGroups - 1)) == 0) ++mb;
            fold_unit(j, fc.tile, 0.f, 0.f, mb % NS, fc.g);
        }
    } else {
        // metadata loads run kMetaAhead units ahead of the folds (scattered 2- and 4-byte loads of L2
        // latency): unit j's scale and zero point live in slot j % kMetaAhead of a register ring
        constexpr int kMetaAhead = 4;
        UnitCursor fc(u_first, G), mc(u_first, G);
        uint32_t sr[kMetaAhead];
        int zr[kMetaAhead];
#pragma unroll
        for (int u = 0; u < kMetaAhead; ++u) {
            load_meta(mc.tile, mc.g, sr[u], zr[u]);
            mc.next(G);
        }
        for (int j0 = 0; j0 < nunits; j0 += kMetaAhead) {
#pragma unroll
            for (int u = 0; u < kMetaAhead; ++u) {
                const int j = j0 + u;
                if (j < nunits) {
                    const bool row_ok = fc.tile * kRowsPerCta + row_local < N;
                    const float sv = row_ok ? bf16_bits_to_float((uint16_t)sr[u]) : 0.f;
                    const float zv = (float)zr[u];
                    load_meta(mc.tile, mc.g, sr[u], zr[u]);
                    mc.next(G);
                    fold_unit(j, fc.tile, sv, zv, 0, 0);
                    fc.next(G);
                }
            }
        }
    }
    const int tile_last = nunits > 0 ? (int)((u_first + nunits - 1) / G) : cur_tile - 1;
    while (cur_tile <= tile_last) flush(cur_tile++);

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
// One-token decode kernel (M = 1).
//
// At M = 1 a tcgen05 MMA would waste most of its columns, and its operands
// would have to pass through tensor memory; the dot products instead run as
// warp-level mma.sync m16n8k32 in registers: A = 16 rows x 32 codes as
// unsigned bytes, straight from the packed words, B = 32 codes x 8 columns of
// X digits as signed bytes, D = exact int32 sums.  Each packed word gives its
// A bytes in one instruction per half: w & 0x0F0F0F0F holds codes 0, 2, 4, 6,
// and w & 0xF0F0F0F0 holds 16 times codes 1, 3, 5, 7.  X is expanded into
// integers per group: with E the exponent of the group's largest |x|, an
// even code's activation is x_int = rint(x 2^(21 - E)) and an odd code's is
// rint(x 2^(17 - E)) -- the factor 16 of its A byte makes the product the
// same q x 2^(21 - E) -- so every activation within 2^10 of the group
// maximum is exact (within 2^14 for even codes) and smaller ones are rounded
// at 2^(E - 21) or 2^(E - 17), far below FP32 accumulation error.  x_int is
// written in balanced base 256, 65536 d2 + 256 d1 + d0 with every digit in
// [-128, 127]; columns 0-2 of B hold digit planes 0-2, columns 4-6 the same
// planes again (so that the lanes holding accumulator columns 4-7 have every
// plane of the second row block), columns 3 and 7 are zero.  Per group and
// row, with X_k the represented activations (x_int, or 16 x_int for odd codes):
//   acc += s (65536 D2 + 256 D1 + D0 - z sum_k X_k) 2^(E - 21).
// One MMA takes 32 codes of 16 rows against every plane: a compute thread
// issues 8 MMAs per group where byte-plane dp4a would take 96 instructions,
// and each lane of a quad folds one of the quad's four rows.
//
// X of one group in the layout the kernel reads: 3 digit rows of 128 bytes
// (word w's codes 0,2,4,6 at 8w, codes 1,3,5,7 at 8w + 4: the order in which
// the two masks above hold the codes, so a lane's B fragment of MMA j is
// bytes 32 tig + 8 j .. + 7 of its row), then (sum_k X_k as FP32, 2^(E - 21)),
// padded to 400 bytes.
// A unit is 128 rows x one group (8 KB of codes).  Units are dealt out in
// chunks of U consecutive groups of one row tile (U = 4, or 2 where the CTAs
// have fewer than 12 units each): chunk c is row tile c / cpt, groups
// U (c % cpt) onwards (cpt = G / U chunks per row tile); with U = 4 the last
// row tiles (about two chunks per CTA) are cut into chunks of 2, so that the
// chunks drawn last are short.  A chunk's partial sums go to slot c.  CTA b takes chunk b first, then asks a global counter for the
// next free chunk while it issues the current one, so a CTA that starts early
// or streams fast takes more chunks and every CTA finishes within about a
// chunk of the others.  (An equal, static deal left the CTAs that started
// late -- launched as the preceding call's CTAs freed their SMs -- finishing
// several microseconds after the rest, and the next call cannot begin its
// arithmetic until the last one is done.)  Each chunk leaves its 128 partial
// sums in a slot of its own, and decode_cc_reduce_kernel, launched as a
// dependent grid, adds each row tile's slots in slot order, so Y has the same
// bits however the chunks were shared out.  (Adding them inside this kernel,
// by the CTA that completed a tile's last chunk, measured slower: the arrival
// and the reads of the last tiles kept CTAs resident for microseconds after
// their arithmetic ended.)
// Warp roles (192 threads, four CTAs per SM), with a 4-stage ring:
//  * warp 4 (one thread) takes chunks and drives TMA: per unit it publishes
//    (row tile, group, chunk slot, metadata slot) in a descriptor ring, then
//    loads the codes (64-byte swizzle) and, with a chunk's first unit, the
//    128 x 8 scales and zero points of the 8-group block that holds the chunk
//    into one of three metadata slots;
//  * warp 5 prepares X: the groups of a chunk are loaded at its first unit,
//    and each unit's digit rows, group sum and power of two are written into
//    its stage;
//  * warps 0-3 compute: warp w takes rows 32 w .. 32 w + 31 of each unit as
//    two 16-row MMA blocks (below); at a chunk's last unit each lane stores
//    its row's sum into the chunk's slot.
constexpr int kCcWarps = 4;                              // compute warps
constexpr int kCcTmaWarp = kCcWarps;                     // warp 4
constexpr int kCcXWarp = kCcWarps + 1;                   // warp 5
constexpr int kCcThreads = (kCcWarps + 2) * 32;
constexpr int kCcStages = 4;                             // ring depth: 32 KB of codes in flight per CTA
constexpr int kCcMinBlocks = 4;                          // CTAs per SM
constexpr int kCcChunkMax = 4;                           // units (groups) per chunk: 2 or 4
constexpr int kCcRowBytes = 64;                          // codes of one row in a unit
constexpr int kCcSwizzleSpan = 8 * kCcRowBytes;          // 64-byte swizzle: 8-row pattern
constexpr int kCcCodeBytes = kStageWords * 4;            // 8 KB
constexpr int kCcXOff = kCcCodeBytes;                    // X of the unit's group, after the codes
constexpr int kCcXGroupBytes = 400;                      // 3 digit rows + sum and scale, 16-byte aligned
constexpr int kCcStageBytes = (kCcCodeBytes + kCcXGroupBytes + kCcSwizzleSpan - 1) / kCcSwizzleSpan * kCcSwizzleSpan;
constexpr int kCcMetaGroups = 8;                         // groups per metadata block
constexpr int kCcScBytes = kRowsPerCta * kCcMetaGroups * 2;  // 128 rows x 8 BF16 scales
constexpr int kCcZeBytes = kRowsPerCta * kCcMetaGroups * 4;  // 128 rows x 8 int32 zero points
constexpr int kCcMetaBytes = kCcScBytes + kCcZeBytes;    // one slot, 6 KB
constexpr int kCcMetaSlots = 3;
constexpr int kCcMetaOff = kCcStages * kCcStageBytes;    // the metadata slots after the ring
constexpr size_t kCcSmem = (size_t)kCcMetaOff + kCcMetaSlots * kCcMetaBytes + 1024;  // + alignment slack
static_assert(kCcMetaGroups % kCcChunkMax == 0, "a chunk lies inside one metadata block");
// A chunk's block goes into slot (chunk number) % kCcMetaSlots, overwriting the block of the chunk
// kCcMetaSlots chunks earlier, whose last unit is then at least (kCcMetaSlots - 1) 2 + 1 units back
// (chunks of 2 or more units); the TMA thread issues a unit only after the unit kCcStages back has been
// released.
static_assert((kCcMetaSlots - 1) * 2 + 1 >= kCcStages, "metadata slot reuse");
// MMA accumulators start at the bits of 1.5 2^23: a plane sum P then ends as the FP32 number 1.5 2^23 + P
// (|P| < 2^22; here |P| < 2^22 even with the odd codes' factor 16: 128 codes x 240 x 128).
constexpr int kCcPlaneBias = 0x4B400000;

struct CcArgs {
    const uint16_t* X;  // [K] BF16: the activations (X' = bf16(x * xscale) for the AWQ entry)
    uint16_t* Y;        // [N]
    float* partial;     // [row_tiles][cpt][128]: one slot of sums per chunk
    int* counters;      // counters[row_tiles]: the chunk counter (the row tiles' own counters stay unused)
    int* fault;
    int N, G;           // G: groups per row (a multiple of 8)
    int U;              // units per chunk in row tiles [0, tiles_a) (2 or 4); 2 in the tiles after them
    int cpt, chunks;    // chunks per row tile (G / U) in the first region, chunks in all
    int tiles_a, chunks_a;  // row tiles and chunks of the first region (chunk c is slot c of the partials)
    int row_tiles;
};

// This lane's four BF16 values of group g: lane 2w + h holds values 4h..4h+3 of word w.
__device__ __forceinline__ uint2 load_group_x(const uint16_t* __restrict__ X, int g, int lane) {
    return __ldg(reinterpret_cast<const uint2*>(X + (int64_t)g * kGroup + lane * 4));
}

// mma.sync m16n8k32, A 16 x 32 unsigned bytes (row-major fragments), B 32 x 8 signed bytes
// (column-major fragments), D (+)= int32: exact integer dot products.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One warp writes the X of one group (its lanes' values v from load_group_x) in the layout above.
//
// The integers come from one FFMA with the 1.5 2^23 magic constant (|x 2^k| < 2^22, so the sum's last
// place is 1 and its rounding is the rounding to the nearest integer, ties to even), and
// x_int + 0x808080 = (d0 + 128) + 256 (d1 + 128) + 65536 (d2 + 128) holds the three balanced base-256
// digits, each plus 128, in its three low bytes: the digit bytes are that word XOR 0x808080.
__device__ __forceinline__ void prep_group_x8(const uint2 v, unsigned char* dst, int lane) {
    const uint32_t a2 = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
    uint32_t amax = max(a2 & 0xFFFFu, a2 >> 16);
    amax = __reduce_max_sync(0xFFFFFFFFu, amax);
    const int ef = (int)(amax >> 7);
    const int E = ef == 0 ? -127 : ef - 127;  // every |x| of the group is below 2^(E + 1)
    const int kx = 21 - E;                    // in [-106, 148]
    const int k1 = min(kx, 127);
    const float s1 = pow2f(k1), s2 = pow2f(kx - k1);  // exact scalings, |x 2^kx| < 2^22
    // lane (w, h) holds codes 4h .. 4h + 3 of word w: values 1 and 3 belong to odd codes (scale 2^(kx - 4))
    const float xv[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                         __uint_as_float(v.y & 0xFFFF0000u)};
    uint32_t D[4];
    int xi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float f = __fmaf_rn(xv[i] * s1, (i & 1) ? s2 * 0.0625f : s2, 12582912.f);  // 1.5 2^23 + x_int
        const uint32_t yb = __float_as_uint(f) - (0x4B400000u - 0x808080u);          // x_int + 0x808080
        xi[i] = (int)yb - 0x808080;
        D[i] = yb ^ 0x808080u;  // bytes 0..2: digits d0, d1, d2 as signed bytes
    }
    // planes as (i0, i2, i1, i3): P = [d0 i0, d0 i2, d1 i0, d1 i2], Q = the same for i1, i3; R, S plane 2
    const uint32_t P = __byte_perm(D[0], D[2], 0x5140), Q = __byte_perm(D[1], D[3], 0x5140);
    const uint32_t R = __byte_perm(D[0], D[2], 0x0062), S = __byte_perm(D[1], D[3], 0x0062);
    uint32_t dg[3];
    dg[0] = __byte_perm(P, Q, 0x5410);
    dg[1] = __byte_perm(P, Q, 0x7632);
    dg[2] = __byte_perm(R, S, 0x5410);
    // h = 0 assembles the even-code word (its codes 0, 2 and the partner's 4, 6), h = 1 the odd one
    // (the partner's 1, 3 and its own 5, 7)
    const int h = lane & 1, w = lane >> 1;
#pragma unroll
    for (int p = 0; p < 3; ++p) {
        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, dg[p], 1);
        const uint32_t lo = h ? other : dg[p], hi = h ? dg[p] : other;
        const uint32_t out = h ? __byte_perm(lo, hi, 0x7632) : __byte_perm(lo, hi, 0x5410);
        *reinterpret_cast<uint32_t*>(dst + p * 128 + 8 * w + 4 * h) = out;
    }
    // sum of the represented activations: odd codes' integers count 16 times (|sum| < 2^29)
    const int sum = __reduce_add_sync(0xFFFFFFFFu, (xi[0] + xi[2]) + 16 * (xi[1] + xi[3]));
    if (lane == 0) {
        float* ext = reinterpret_cast<float*>(dst + 3 * 128);
        ext[0] = (float)sum;
        ext[1] = pow2f(E - 21);
    }
}

__global__ void __launch_bounds__(kCcThreads, kCcMinBlocks) decode_cc_kernel(const __grid_constant__ CUtensorMap tq,
                                                                  const __grid_constant__ CUtensorMap tsc,
                                                                  const __grid_constant__ CUtensorMap tze,
                                                                  const CcArgs a) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kCcStages], empty[kCcStages], dready[kCcStages];
    __shared__ int4 s_desc[kCcStages];   // (row tile, group, chunk slot, flags) of the unit in each stage
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-aligned (the swizzle's span)
    unsigned char* meta = ring + kCcMetaOff;
    // descriptor flags: first unit of its chunk, last unit of its chunk, end of the stream; metadata slot
    // and the chunk's unit count
    constexpr int kFirst = 1, kLast = 2, kEnd = 4, kSlotShift = 4, kUnitsShift = 8;

    pdl_launch_dependents();  // the next call may start its weight loads as this grid's CTAs retire
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    int* const next_chunk = a.counters + a.row_tiles;  // chunks taken beyond the first gridDim.x

    if (threadIdx.x == 0) {
        for (int s = 0; s < kCcStages; ++s) {
            mbar_init(&full[s], 2);  // TMA thread (with the transaction bytes) + X warp
            mbar_init(&empty[s], kCcWarps);
            mbar_init(&dready[s], 1);  // TMA thread: the stage's descriptor is written
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kCcTmaWarp) {  // ------------------------------------------- TMA
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tsc);
            prefetch_tmap(&tze);
            int i = 0, nchunks = 0;  // units and chunks issued
            bool ok = true;
            auto issue_chunk = [&](int c) {
                // chunk c: U units of one row tile; the row tiles from tiles_a on are cut into chunks of 2
                int tile, U, g0;
                if (c < a.chunks_a) {
                    tile = c / a.cpt;
                    U = a.U;
                    g0 = (c - tile * a.cpt) * U;
                } else {
                    const int cb = c - a.chunks_a, cpt_b = a.G / 2;
                    tile = a.tiles_a + cb / cpt_b;
                    U = 2;
                    g0 = (cb - (tile - a.tiles_a) * cpt_b) * 2;
                }
                const int mslot = nchunks++ % kCcMetaSlots;
                for (int u = 0; u < U; ++u, ++i) {
                    const int s = i % kCcStages;
                    if (i >= kCcStages && !mbar_wait(&empty[s], ((i / kCcStages) - 1) & 1, a.fault, 51)) {
                        ok = false;
                        return;
                    }
                    const int g = g0 + u;
                    s_desc[s] = make_int4(tile, g, c,
                                          (u == 0 ? kFirst : 0) | (u + 1 == U ? kLast : 0) | (mslot << kSlotShift) |
                                              (U << kUnitsShift));
                    mbar_arrive(&dready[s]);
                    unsigned char* st = ring + s * kCcStageBytes;
                    mbar_arrive_expect_tx(&full[s], kCcCodeBytes + (u == 0 ? kCcMetaBytes : 0));
                    tma_load_2d(st, &tq, g * kWordsPerGroup, tile * kRowsPerCta, &full[s]);
                    if (u == 0) {
                        unsigned char* ms = meta + mslot * kCcMetaBytes;
                        const int g8 = g & ~(kCcMetaGroups - 1);
                        tma_load_2d(ms, &tsc, g8, tile * kRowsPerCta, &full[s]);
                        tma_load_2d(ms + kCcScBytes, &tze, g8, tile * kRowsPerCta, &full[s]);
                    }
                }
            };
            // the weights need nothing from the preceding kernel: the first chunk streams at once
            issue_chunk(b);  // gridDim.x <= chunks
            // the chunk counter is this launch's once the preceding launch has completed (which leaves it zero)
            pdl_wait_primary();
            // Each CTA takes chunks until the counter runs past the end, so a launch draws exactly `chunks`
            // values, 0 .. chunks - 1: the CTA that draws the last one is the last to draw at all and
            // puts the counter back to zero for the next launch.
            int v = ok ? atomicAdd(next_chunk, 1) : 0;
            while (ok && (int)gridDim.x + v < a.chunks) {
                const int c = (int)gridDim.x + v;
                v = atomicAdd(next_chunk, 1);  // in flight while chunk c is issued
                issue_chunk(c);
            }
            if (ok && v == a.chunks - 1) *next_chunk = 0;
            // every copy issued must land before the CTA may exit; then the end of the stream, in the stage
            // after the last unit (posted after the drain, so that no stage sees a newer phase meanwhile)
            for (int j = max(0, i - kCcStages); j < i; ++j)
                mbar_wait(&full[j % kCcStages], (j / kCcStages) & 1, a.fault, 52);
            if (ok) {
                const int s = i % kCcStages;
                if (i < kCcStages || mbar_wait(&empty[s], ((i / kCcStages) - 1) & 1, a.fault, 51)) {
                    s_desc[s] = make_int4(-1, 0, 0, kEnd);
                    mbar_arrive(&dready[s]);
                    mbar_arrive(&full[s]);
                }
            }
        }
        return;
    }

    if (warp == kCcXWarp) {  // ------------------------------------------ X warp
        pdl_wait_primary();  // X may come from the preceding kernel
        uint2 xq[kCcChunkMax];  // the current chunk's groups, loaded together (one L2 round trip per chunk)
        for (int i = 0;; ++i) {
            const int s = i % kCcStages;
            if (!warp_wait(&dready[s], (i / kCcStages) & 1, a.fault, 54)) break;
            const int4 d = s_desc[s];
            if (!(d.w & kEnd)) {
                const int U = (d.w >> kUnitsShift) & 7;
                if (d.w & kFirst) {
#pragma unroll
                    for (int j = 0; j < kCcChunkMax; ++j)
                        if (j < U) xq[j] = load_group_x(a.X, d.y + j, lane);
                }
                const int u = d.y & (U - 1);
                uint2 v = xq[0];
#pragma unroll
                for (int j = 1; j < kCcChunkMax; ++j)
                    if (u == j) v = xq[j];
                // the stage was released before its descriptor was posted
                prep_group_x8(v, ring + s * kCcStageBytes + kCcXOff, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
            if (d.w & kEnd) break;
        }
        return;
    }

    // ---------------------------------------------------- compute warps 0-3
    // Warp w takes rows 32 w .. 32 w + 31 as two 16-row MMA blocks.  Lane (g8, tig) = (lane / 4,
    // lane % 4) holds, per block, rows g8 and g8 + 8 of its A fragments and words 4 tig .. 4 tig + 3
    // of each (one 16-byte chunk of the group's codes); MMA j takes word 4 tig + j of every lane, so
    // its K = 32 codes are words j, 4 + j, 8 + j, 12 + j, and the lane's B fragments are the same
    // words of its digit row.
    const int g8 = lane >> 2, tig = lane & 3;
    auto rrow = [&](int k) { return 32 * warp + 16 * (k >> 1) + g8 + 8 * (k & 1); };
    const int r_own = rrow(tig);  // the row this lane folds
    float y = 0.f;                // row r_own of the current chunk
    for (int i = 0;; ++i) {
        const int s = i % kCcStages;
        if (!warp_wait(&full[s], (i / kCcStages) & 1, a.fault, 53)) break;
        const int4 d = s_desc[s];
        if (d.w & kEnd) break;
        const unsigned char* st = ring + s * kCcStageBytes;
        const unsigned char* ms = meta + ((d.w >> kSlotShift) & 3) * kCcMetaBytes;
        // codes: 16-byte chunk tig of each 64-byte row, 64-byte swizzle (chunk c of row r at c ^ ((r >> 1) & 3))
        uint4 cw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = rrow(k);
            cw[k] = *reinterpret_cast<const uint4*>(st + r * kCcRowBytes + 16 * (tig ^ ((r >> 1) & 3)));
        }
        // B columns 4-6 repeat digit planes 0-2, so that lanes tig = 2, 3 hold every plane of the second
        // row block and each lane of a quad can fold one of its four rows; columns 3 and 7 are zero
        const unsigned char* xg = st + kCcXOff;
        uint32_t bx[8];
        const int xrow = g8 & 3;
        if (xrow < 3) {
            const uint4* xp = reinterpret_cast<const uint4*>(xg + xrow * 128 + tig * 32);
            const uint4 u0 = xp[0], u1 = xp[1];
            bx[0] = u0.x; bx[1] = u0.y; bx[2] = u0.z; bx[3] = u0.w;
            bx[4] = u1.x; bx[5] = u1.y; bx[6] = u1.z; bx[7] = u1.w;
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) bx[j] = 0u;
        }
        const float* ext = reinterpret_cast<const float*>(xg + 3 * 128);
        const float xsum = ext[0], xscale = ext[1];
        // this lane's row's metadata, from the chunk's block (loaded with the chunk's first unit, which
        // this warp has already waited for); rows past N were zero-filled by TMA: s = 0 folds them away
        const int gb = d.y & (kCcMetaGroups - 1);
        const float sv = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(ms + r_own * (kCcMetaGroups * 2) + 2 * gb));
        const float zv = (float)*reinterpret_cast<const int32_t*>(ms + kCcScBytes + r_own * (kCcMetaGroups * 4) + 4 * gb);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        int dd[2][4];
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
            const uint32_t w0[4] = {cw[2 * rb].x, cw[2 * rb].y, cw[2 * rb].z, cw[2 * rb].w};
            const uint32_t w1[4] = {cw[2 * rb + 1].x, cw[2 * rb + 1].y, cw[2 * rb + 1].z, cw[2 * rb + 1].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) dd[rb][j] = kCcPlaneBias;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_u8s8(dd[rb], w0[j] & 0x0F0F0F0Fu, w1[j] & 0x0F0F0F0Fu, w0[j] & 0xF0F0F0F0u, w1[j] & 0xF0F0F0F0u,
                         bx[2 * j], bx[2 * j + 1]);
        }
        // lane tig holds D columns 2 tig, 2 tig + 1 of rows g8 (d0, d1) and g8 + 8 (d2, d3): planes (0, 1)
        // at tig = 0 and 2, (2, -) at tig = 1 and 3.  Lane tig folds row rrow(tig): row block tig >> 1
        // (its own MMA results) and row g8 + 8 (tig & 1); one exchange with the neighbour completes its
        // planes.
        const bool hi = tig >> 1, even = !(tig & 1);
        int e[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) e[j] = hi ? dd[1][j] : dd[0][j];
        const int x0 = __shfl_xor_sync(0xFFFFFFFFu, even ? e[2] : e[0], 1);
        const int x1 = __shfl_xor_sync(0xFFFFFFFFu, e[3], 1);
        const int P0 = even ? e[0] : x0, P1 = even ? e[1] : x1, P2 = even ? x0 : e[2];
        // the plane sums are biased: read as FP32 each is 1.5 2^23 + P exactly (|P| < 2^22), so one
        // subtraction converts it.  sum q X = 65536 P2 + (256 P1 + P0), the bracket rounded once by the inner
        // FMA; then s (sum q X - z sum X) and the power of two last, so that neither product leaves the
        // FP32 range unless the group's result itself does
        const float F0 = __int_as_float(P0) - 12582912.f, F1 = __int_as_float(P1) - 12582912.f,
                    F2 = __int_as_float(P2) - 12582912.f;
        const float qx = fmaf(F2, 65536.f, fmaf(F1, 256.f, F0));
        y = fmaf(sv * fmaf(-zv, xsum, qx), xscale, y);

        if (d.w & kLast) {  // the chunk's sums leave through its slot (decode_cc_reduce_kernel adds them)
            a.partial[(int64_t)d.z * kRowsPerCta + r_own] = y;  // slot = chunk index
            y = 0.f;
        }
    }
}

// Copy of X from mapped host memory into the device buffer, as a kernel in the programmatic-launch chain (a
// copy-engine transfer would end the chain: the GEMV could no longer start its weight loads early).  It
// waits for the preceding kernel before reading (X may be that kernel's host-mapped output) and before
// writing (that kernel may still read the device buffer).
__global__ void __launch_bounds__(256) h2d_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                       int64_t n16) {
    pdl_launch_dependents();
    pdl_wait_primary();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = src[i];
}

// Split-K sums of the one-token kernel: Y[n] = the sum of row n's chunk slots in slot order.  A
// dependent grid: its CTAs become resident beside the GEMV's (256 threads of at most 32 registers fit next
// to four GEMV CTAs) and wait for it to complete.  An item is 256 / P rows of a row tile, P threads per
// row: part p adds slots p, p + P, ... of its row (at most 32 loads in flight per thread, so one L2 round
// trip serves tiles of up to 32 P chunks), then part 0 adds the P part sums in order.  P = 2 (whole row
// tiles) unless a tile has more than 64 slots, then P = 4 (half tiles).
constexpr int kCcRedThreads = 256;
constexpr int kCcRedLoads = 32;
template <int P>
__global__ void __launch_bounds__(kCcRedThreads) decode_cc_reduce_kernel(const float* __restrict__ partial,
                                                                          uint16_t* __restrict__ Y, int N, int cpt,
                                                                          int row_tiles, uint16_t* __restrict__ Yh,
                                                                          int tiles_a, int cpt_b) {
    constexpr int R = kCcRedThreads / P;   // rows per item
    constexpr int SUBT = kRowsPerCta / R;  // items per row tile
    __shared__ float s_part[P - 1][R];
    pdl_launch_dependents();
    pdl_wait_primary();
    const int r = threadIdx.x % R, p = threadIdx.x / R;
    for (int item = blockIdx.x; item < row_tiles * SUBT; item += gridDim.x) {
        const int tile = item / SUBT, row = (item % SUBT) * R + r;
        // the tile's slots: cpt from tile * cpt in the first region, cpt_b after the first region's
        const int64_t first = tile < tiles_a ? (int64_t)tile * cpt : (int64_t)tiles_a * cpt + (int64_t)(tile - tiles_a) * cpt_b;
        const int nslots = tile < tiles_a ? cpt : cpt_b;
        const float* pb = partial + first * kRowsPerCta + row;
        float acc = 0.f;
        for (int k0 = p; k0 < nslots; k0 += kCcRedLoads * P) {
            float v[kCcRedLoads];
#pragma unroll
            for (int e = 0; e < kCcRedLoads; ++e) {
                const int k = k0 + e * P;
                v[e] = k < nslots ? __ldcg(pb + (int64_t)k * kRowsPerCta) : 0.f;
            }
#pragma unroll
            for (int e = 0; e < kCcRedLoads; ++e) acc += v[e];
        }
        if (p > 0) s_part[p - 1][r] = acc;
        __syncthreads();
        if (p == 0) {
#pragma unroll
            for (int q = 0; q < P - 1; ++q) acc += s_part[q][r];
            const int n = tile * kRowsPerCta + row;
            if (n < N) {
                const uint16_t yb = float_to_bf16_bits(acc);
                Y[n] = yb;
                if (Yh) Yh[n] = yb;  // the host copy, stored straight into mapped host memory
            }
        }
        __syncthreads();
    }
}


template <int NTOK>
int occupancy_nt() {
    static PerContext<int> cache;  // the attribute belongs to a context
    return cache.get([]() -> int {
        if (cudaFuncSetAttribute(decode_tc_kernel<NTOK, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)TcCfg<NTOK, false>::kSmem) != cudaSuccess ||
            cudaFuncSetAttribute(decode_tc_kernel<NTOK, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)TcCfg<NTOK, true>::kSmem) != cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, decode_tc_kernel<NTOK, false>, kTcThreads,
                                                          TcCfg<NTOK, false>::kSmem) != cudaSuccess ||
            o < 1)
            return 0;
        return 1;  // one CTA per SM: it owns all 512 TMEM columns
    });
}

int occupancy_cc() {
    static PerContext<int> cache;  // the attribute and occupancy belong to a context
    return cache.get([]() -> int {
        if (cudaFuncSetAttribute(decode_cc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCcSmem) !=
            cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, decode_cc_kernel, kCcThreads, kCcSmem) != cudaSuccess ||
            o < 1)
            return 0;
        return o;
    });
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
    else if (kind == 3)  // zeros: int32 [rows = N][cols = G], box = 8 groups x 128 rows
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_INT32, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 4, kCcMetaGroups, kRowsPerCta);
    else  // X digit planes: uint8 [rows = G * 3 NTOK][cols = 128], box = 128 x 3 NTOK (kind = NTOK), 128-byte swizzle
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols, 128, (uint32_t)(3 * kind), CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return false;
    e.ptr = ptr;
    e.rows = rows;
    e.cols = cols;
    e.kind = kind;
    g_tmap_next = (g_tmap_next + 1) % 128;
    *out = e.map;
    return true;
}

int launch_cc(const CUtensorMap& tq, const CUtensorMap& tsc, const CUtensorMap& tze, const CcArgs& args, int grid,
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

// tsc, tze: the scales' and zero points' tensor maps with TM (unused, any map, without)
template <int NTOK, bool TM>
int launch_tc(const CUtensorMap& tq, const CUtensorMap& tx, const CUtensorMap& tsc, const CUtensorMap& tze,
              const DecodeArgs& args, int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = TcCfg<NTOK, TM>::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_tc_kernel<NTOK, TM>, tq, tx, tsc, tze, args) == cudaSuccess
               ? W4A16_OK
               : W4A16_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

// Split-K reduction of the decode GEMVs: a tile whose units one CTA held was written as Y by that CTA; a
// tile shared by CTAs first .. last is the sum of their partial-sum slots, added here in slot order (the
// same bits on every run).  A dependent grid of at most one small CTA per SM, looping over the row
// tiles: it fits beside the GEMV's CTAs, so all of it is resident (and has released its own dependents)
// while the GEMV still runs, and it waits for the GEMV only when it reaches a shared tile.
__global__ void __launch_bounds__(128) decode_reduce_kernel(const float* __restrict__ partial, uint16_t* __restrict__ Y,
                                                            int N, int M, int G, int units_base, int units_rem,
                                                            int max_slots, int row_tiles) {
    pdl_launch_dependents();
    bool waited = false;
    for (int tile = blockIdx.x; tile < row_tiles; tile += gridDim.x) {
        const int first = cta_of_unit((int64_t)tile * G, units_base, units_rem);
        const int last = cta_of_unit((int64_t)tile * G + G - 1, units_base, units_rem);
        if (first == last) continue;
        if (!waited) {
            pdl_wait_primary();
            waited = true;
        }
        const int nseg = last - first + 1, rows = min(kRowsPerCta, N - tile * kRowsPerCta);
        const float* pb = partial + (int64_t)tile * max_slots * M * kRowsPerCta;
        for (int idx = threadIdx.x; idx < M * rows; idx += 128) {
            const int m = idx / rows, rl = idx - m * rows;
            const float sum = sum_slots(pb + (int64_t)m * kRowsPerCta + rl, (int64_t)M * kRowsPerCta, nseg);
            Y[(int64_t)m * N + tile * kRowsPerCta + rl] = float_to_bf16_bits(sum);
        }
    }
}

int launch_decode_reduce(const float* partial, uint16_t* Y, int64_t N, int M, int G, int units_base, int units_rem,
                         int max_slots, int row_tiles, cudaStream_t stream) {
    const int sms = num_sms_current();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(row_tiles < sms ? row_tiles : sms));
    cfg.blockDim = dim3(128);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_reduce_kernel, partial, Y, (int)N, M, G, units_base, units_rem, max_slots,
                              row_tiles) == cudaSuccess
               ? W4A16_OK
               : W4A16_ERR_CUDA;
}

DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int num_sms) {
    DecodePlan p{};
    const int64_t Mc = M < kMaxTokens ? M : kMaxTokens;
    const int64_t G = K / kGroup;
    // the one-token integer kernel for M = 1 (needs 16-byte metadata rows: G % 8 == 0); the register-MMA
    // GEMV of gemv_mt.cu for 2-16 tokens (same condition); else the 8-bit tensor-core GEMV below with MMA
    // N = 3 x 16 or 3 x 32 (17 or more tokens, or K / 128 not a multiple of 8); the BF16 tensor-core GEMV
    // (gemv_bf.cu) serves quantisation groups of 32 and 64
    p.cc_tokens = (M <= 1 && G % 8 == 0) ? (int)M : 0;
    p.mt = !p.cc_tokens && mt_supported(K) && M <= kMtMaxTokens;
    p.bf = false;
    p.nt = p.cc_tokens ? 1 : (Mc <= 16 ? 16 : 32);
    p.row_tiles = (int)ceil_div(N, kRowsPerCta);
    if (p.cc_tokens) {  // chunks dealt out by a counter after the row tiles' arrival counters
        int occ = occupancy_cc();
        if (occ < 1) occ = 1;
        const int64_t grid = (int64_t)occ * num_sms;
        // chunks of 4 units where every CTA streams 12 or more units, else of 2 (finer sharing)
        p.cc_units = (int64_t)p.row_tiles * G >= 12 * grid ? 4 : 2;
        p.cc_cpt = (int)(G / p.cc_units);
        // with chunks of 4, the last row tiles (about two chunks of 2 per CTA) are cut into chunks of 2, so
        // that the CTAs' last chunks are short and they finish closer together
        int tiles_b = 0;
        if (p.cc_units == 4) {
            tiles_b = (int)ceil_div(4 * grid, G);
            if (tiles_b > p.row_tiles / 2) tiles_b = p.row_tiles / 2;
        }
        p.cc_tiles_a = p.row_tiles - tiles_b;
        p.cc_chunks_a = p.cc_tiles_a * p.cc_cpt;
        p.cc_chunks = p.cc_chunks_a + tiles_b * (int)(G / 2);
        p.grid = (int)(grid < p.cc_chunks ? grid : p.cc_chunks);
        p.ws_xp_bytes = align256((size_t)M * K * 2);  // X' = bf16(X * xscale) for the AWQ entry
        p.ws_xs_bytes = 0;
        p.ws_partial_bytes = align256((size_t)p.cc_chunks * kRowsPerCta * 4);
        const int64_t words = p.row_tiles + 1;
        p.ws_counter_bytes = align256((size_t)(words > kSharedCounterTiles ? words : kSharedCounterTiles) * 4);
        return p;
    }
    if (p.mt || p.bf) {  // these GEMVs keep their own plans per chunk; only their scratch is sized here
        p.ws_xp_bytes = p.mt ? mt_workspace_bytes(M, N, K, num_sms) : bf_workspace_bytes(M, N, K, kGroup, num_sms);
        p.ws_xs_bytes = 0;
        p.ws_partial_bytes = 0;
        p.ws_counter_bytes =
            align256((size_t)(p.row_tiles > kSharedCounterTiles ? p.row_tiles : kSharedCounterTiles) * 4);
        return p;
    }
    // units per row tile: one per group
    const int64_t ug = G;
    p.unit_groups = (int)ug;
    const int64_t units = (int64_t)p.row_tiles * ug;
    int occ = p.nt == 16 ? occupancy_nt<16>() : occupancy_nt<32>();
    if (occ < 1) occ = 1;
    int64_t grid = (int64_t)occ * num_sms;
    if (grid > units) grid = units;
    p.grid = (int)grid;
    p.units_base = (int)(units / grid);
    p.units_rem = (int)(units % grid);
    p.max_slots = (int)((ug - 1) / p.units_base + 2);
    // the tensor-core kernel reads X digit planes and per-token sums and scales prepared per launch
    p.ws_xp_bytes = align256((size_t)G * 3 * p.nt * 128);
    p.ws_xs_bytes = align256((size_t)G * 2 * p.nt * 4);
    p.ws_partial_bytes = align256((size_t)p.row_tiles * p.max_slots * Mc * kRowsPerCta * 4);
    p.ws_counter_bytes = align256((size_t)(p.row_tiles > kSharedCounterTiles ? p.row_tiles : kSharedCounterTiles) * 4);
    return p;
}

// X' = bf16(x * xscale[k]) ahead of the integer kernel, 8 values per thread.  The dependent
// layer kernel is released first, so it streams weights while this waits for X; its X warp
// reads X' only after this grid has completed.
__global__ void __launch_bounds__(256) awq_prescale_kernel(const uint16_t* __restrict__ X,
                                                           const float* __restrict__ xscale, int64_t n8, int K,
                                                           uint16_t* __restrict__ Xs) {
    pdl_launch_dependents();
    pdl_wait_primary();  // X may come from the preceding kernel
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int k = (int)((i * 8) % K);
        const uint4 v = reinterpret_cast<const uint4*>(X)[i];
        const float4 r0 = __ldg(reinterpret_cast<const float4*>(xscale + k));
        const float4 r1 = __ldg(reinterpret_cast<const float4*>(xscale + k + 4));
        reinterpret_cast<uint4*>(Xs)[i] =
            make_uint4(bf16x2_scaled(v.x, r0.x, r0.y), bf16x2_scaled(v.y, r0.z, r0.w),
                       bf16x2_scaled(v.z, r1.x, r1.y), bf16x2_scaled(v.w, r1.z, r1.w));
    }
}

size_t DecodePlan::workspace_bytes() const { return ws_xp_bytes + ws_xs_bytes + ws_partial_bytes + ws_counter_bytes; }

namespace {

// M = 1: the chunked integer GEMV (after awq_prescale_kernel for the AWQ entry); it adds its own split-K
// slots, so the call is one launch (two with the prescale).
int launch_cc_path(const uint16_t* X, const float* xscale, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                   const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace, const DecodePlan& plan,
                   cudaStream_t stream, const uint16_t* X_host, uint16_t* Y_host) {
    const int G = (int)(K / kGroup);
    CUtensorMap tq, tsc, tze;
    if (!cached_tmap(0, qweight, N, K / 8, &tq) || !cached_tmap(2, scales, N, G, &tsc) ||
        !cached_tmap(3, zeros, N, G, &tze))
        return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    char* ws = reinterpret_cast<char*>(workspace);
    if (X_host) {  // X arrives from host memory by a kernel of the chain
        const int64_t n16 = K * 2 / 16;
        int grid = (int)ceil_div(n16, 256 * 4);
        cudaLaunchConfig_t ccfg = {};
        ccfg.gridDim = dim3((unsigned)(grid < 1 ? 1 : grid));
        ccfg.blockDim = dim3(256);
        ccfg.stream = stream;
        cudaLaunchAttribute cattr[1];
        cattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        cattr[0].val.programmaticStreamSerializationAllowed = 1;
        ccfg.attrs = cattr;
        ccfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&ccfg, h2d_copy_kernel, reinterpret_cast<const uint4*>(X_host),
                               reinterpret_cast<uint4*>(const_cast<uint16_t*>(X)), n16) != cudaSuccess)
            return W4A16_ERR_CUDA;
    }
    CcArgs args;
    args.X = X;
    if (xscale) {
        uint16_t* Xs = reinterpret_cast<uint16_t*>(ws + plan.ws_counter_bytes);
        const int64_t n8 = K / 8;
        int pgrid = (int)ceil_div(n8, 256);
        if (pgrid > num_sms_current()) pgrid = num_sms_current();
        cudaLaunchConfig_t pcfg = {};
        pcfg.gridDim = dim3((unsigned)pgrid);
        pcfg.blockDim = dim3(256);
        pcfg.stream = stream;
        cudaLaunchAttribute pattr[1];
        pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pattr[0].val.programmaticStreamSerializationAllowed = 1;
        pcfg.attrs = pattr;
        pcfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&pcfg, awq_prescale_kernel, X, xscale, n8, (int)K, Xs) != cudaSuccess)
            return W4A16_ERR_CUDA;
        args.X = Xs;
    }
    args.Y = Y;
    args.partial = reinterpret_cast<float*>(ws + plan.ws_counter_bytes + plan.ws_xp_bytes + plan.ws_xs_bytes);
    args.counters = reinterpret_cast<int*>(ws);
    args.fault = fault;
    args.N = (int)N;
    args.G = G;
    args.U = plan.cc_units;
    args.cpt = plan.cc_cpt;
    args.chunks = plan.cc_chunks;
    args.tiles_a = plan.cc_tiles_a;
    args.chunks_a = plan.cc_chunks_a;
    args.row_tiles = plan.row_tiles;
    const int st = launch_cc(tq, tsc, tze, args, plan.grid, stream);
    if (st != W4A16_OK) return st;
    return launch_cc_reduce(args.partial, Y, N, plan.cc_cpt, plan.row_tiles, stream, Y_host, plan.cc_tiles_a,
                            G / 2);
}

}  // namespace

int launch_cc_reduce(const float* partial, uint16_t* Y, int64_t N, int cpt, int row_tiles, cudaStream_t stream,
                     uint16_t* Y_host, int tiles_a, int cpt_b) {
    const int sms = num_sms_current();
    if (tiles_a < 0) tiles_a = row_tiles;  // one region
    // four parts where a tile has more slots than two parts load in one round trip; at most one CTA per SM
    // (more would take the places that the next call's GEMV CTAs start in)
    const bool four = (cpt > cpt_b ? cpt : cpt_b) > 2 * kCcRedLoads;
    const int64_t items = (int64_t)row_tiles * (four ? 2 : 1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(items < sms ? items : sms));
    cfg.blockDim = dim3(kCcRedThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = four ? cudaLaunchKernelEx(&cfg, decode_cc_reduce_kernel<4>, partial, Y, (int)N, cpt,
                                                    row_tiles, Y_host, tiles_a, cpt_b)
                               : cudaLaunchKernelEx(&cfg, decode_cc_reduce_kernel<2>, partial, Y, (int)N, cpt,
                                                    row_tiles, Y_host, tiles_a, cpt_b);
    return e == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

int launch_decode(const uint16_t* X, const float* xscale, int64_t M, int64_t K, const uint32_t* qweight,
                  const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                  const DecodePlan& plan, cudaStream_t stream, const uint16_t* X_host, uint16_t* Y_host) {
    if (plan.mt)
        return launch_decode_mt(X, xscale, M, K, qweight, scales, zeros, N, Y,
                                reinterpret_cast<char*>(workspace) + plan.ws_counter_bytes, stream);
    if (plan.bf)
        return launch_decode_bf(X, xscale, M, K, kGroup, qweight, scales, zeros, N, Y,
                                reinterpret_cast<char*>(workspace) + plan.ws_counter_bytes, stream);
    if (plan.cc_tokens)
        return launch_cc_path(X, xscale, K, qweight, scales, zeros, N, Y, workspace, plan, stream, X_host, Y_host);
    if (X_host || Y_host) return W4A16_ERR_ARG;  // host-mapped transfers are the one-token path's
    CUtensorMap tq;
    if (!cached_tmap(0, qweight, N, K / 8, &tq)) return W4A16_ERR_CUDA;
    const int G = (int)(K / kGroup);
    // scales and zero points by TMA where their rows are 16-byte aligned (G % 8 == 0)
    const bool tm = G % kTcMetaGroups == 0;
    CUtensorMap tsc = tq, tze = tq;
    if (tm && (!cached_tmap(2, scales, N, G, &tsc) || !cached_tmap(3, zeros, N, G, &tze))) return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    char* ws = reinterpret_cast<char*>(workspace);
    int* counters = reinterpret_cast<int*>(ws);
    uint8_t* planes = reinterpret_cast<uint8_t*>(ws + plan.ws_counter_bytes);
    float* xs = reinterpret_cast<float*>(ws + plan.ws_counter_bytes + plan.ws_xp_bytes);
    float* partial = reinterpret_cast<float*>(ws + plan.ws_counter_bytes + plan.ws_xp_bytes + plan.ws_xs_bytes);
    for (int64_t m0 = 0; m0 < M; m0 += kMaxTokens) {
        const int Mc = (int)((M - m0) < kMaxTokens ? (M - m0) : kMaxTokens);
        CUtensorMap tx;
        if (!cached_tmap(plan.nt, planes, (int64_t)G * 3 * plan.nt, 128, &tx)) return W4A16_ERR_CUDA;
        const int64_t prep_threads = (int64_t)G * plan.nt * 32;
        int prep_grid = (int)ceil_div(prep_threads, 256);
        if (prep_grid > num_sms_current() * 8) prep_grid = num_sms_current() * 8;
        if (plan.nt == 16)
            prep_x8_kernel<16><<<prep_grid, 256, 0, stream>>>(X + m0 * K, xscale, Mc, (int)K, planes, xs);
        else
            prep_x8_kernel<32><<<prep_grid, 256, 0, stream>>>(X + m0 * K, xscale, Mc, (int)K, planes, xs);
        if (cudaGetLastError() != cudaSuccess) return W4A16_ERR_CUDA;
        DecodeArgs args;
        args.Xp = X + m0 * K;  // the tensor-core kernel reads the planes
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
        const int st = plan.nt == 16 ? (tm ? launch_tc<16, true>(tq, tx, tsc, tze, args, plan.grid, stream)
                                           : launch_tc<16, false>(tq, tx, tsc, tze, args, plan.grid, stream))
                                     : (tm ? launch_tc<32, true>(tq, tx, tsc, tze, args, plan.grid, stream)
                                           : launch_tc<32, false>(tq, tx, tsc, tze, args, plan.grid, stream));
        if (st != W4A16_OK) return st;
    }
    return W4A16_OK;
}

}  // namespace w4a16
