// Integer GEMV for 2 to 16 tokens per launch: the decode path between the
// one-token kernel and the tensor-core GEMVs ("Weight-Only Quantization and Mixed
// Precision", sections 1 and 5: decode stays bound by the weight stream for
// small batches, so the packed codes are read once for every token of the
// launch and nothing but codes and metadata crosses the memory bus).
//
// Same unit (128 weight rows x one group of 128 K: 8 KB of codes), TMA ring,
// metadata blocks and split-K protocol as the one-token integer GEMV in
// gemv.cu, and the same exact arithmetic: the codes are unsigned bytes
// (w & 0x0F0F0F0F holds codes 0, 2, 4, 6 of a packed word, (w >> 4) & 0x0F0F0F0F
// codes 1, 3, 5, 7), each token's group of activations is the integer
// x_int = x 2^(21 - E) in three signed base-256 digit planes, and
// mma.sync m16n8k32 u8 x s8 forms exact int32 plane sums, folded per group in
// FP32:  y += s (65536 D2 + 256 D1 + D0 - z sum_k x_int) 2^(E - 21).
//
// What changes with the token count is the B operand: the digit planes of all
// tokens are the columns of n8 tiles, laid out so that every lane finds all
// three planes of its own tokens in its own accumulators (no exchange):
//   NT = 16: tile 2p + t / 8 holds plane p of tokens 8 (t / 8) .. + 7;
//   NT = 8:  tile p holds plane p of tokens 0 .. 7;
//   NT = 4:  tile 0 holds (plane 0, plane 1) of tokens 0 .. 3 interleaved,
//            tile 1 holds plane 2 of tokens 0 .. 3 in its even columns.
// A lane (g8, tig) holds accumulator columns 2 tig and 2 tig + 1 of every
// tile, so it folds tokens 2 tig, 2 tig + 1 (and 8 + 2 tig, 9 + 2 tig at
// NT = 16), or token tig at NT = 4, for its four rows of each unit.
//
// The digit rows of a launch depend on the tokens only, so a small pre-pass
// (prep_mt_kernel) writes them once per group into the workspace, and the TMA
// thread fetches each unit's group of rows from L2 with one bulk copy beside
// the unit's codes (after the dependent-launch wait; the codes first).
#include "common.cuh"
#include "decode_units.cuh"
#include "sm100.cuh"

namespace w4a16 {
namespace {

constexpr int kRows = 128;                        // weight rows per unit
constexpr int kCodeBytes = kRows * kWordsPerGroup * 4;  // 8 KB per unit, 64-byte swizzle
#ifndef W4A16_MT_WARPS
#define W4A16_MT_WARPS 4
#endif
constexpr int kWarps = W4A16_MT_WARPS;            // compute warps (4: 32 rows each, 8: 16 rows each)
constexpr int kRB = 8 / kWarps;                   // 16-row MMA blocks per compute warp
static_assert(kWarps == 4 || kWarps == 8, "compute warps");
constexpr int kTmaWarp = kWarps;                  // warp 4
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kStages = 4;
constexpr int kMetaGroups = 8;                    // groups per metadata block
constexpr int kScBytes = kRows * kMetaGroups * 2;  // 128 rows x 8 BF16 scales
constexpr int kZeBytes = kRows * kMetaGroups * 4;  // 128 rows x 8 int32 zero points
constexpr int kMetaBytes = kScBytes + kZeBytes;
// A metadata slot is rewritten two blocks later; blocks are aligned to 8 groups inside a row tile
// (G % 8 == 0), so the block in between has 8 units, and at most kStages of them are in flight.
static_assert(kStages <= kMetaGroups, "metadata slot reuse");

// MMA accumulators start at the bits of 1.5 2^23 (0x4B400000): a plane sum P (|P| < 2^18: 128 codes of at
// most 15 times digits of at most 128) then ends as the FP32 number 1.5 2^23 + P, exactly, and one
// subtraction of 1.5 2^23 gives P as a float -- where an integer-to-float conversion would take a
// quarter-rate instruction per plane.
constexpr int kPlaneBias = 0x4B400000;

template <int NT>
struct MtCfg {
    static constexpr int kTiles = NT == 4 ? 2 : 3 * NT / 8;   // n8 tiles of the B operand
    static constexpr int kXRows = 8 * kTiles;                 // digit rows per group
    static constexpr int kXBytes = kXRows * 128 + 8 * NT;     // + per token (sum x_int, 2^(E - 21)) in FP32
    static constexpr int kXOff = kCodeBytes;                  // digit rows after the codes
    static constexpr int kStageBytes = (kCodeBytes + kXBytes + 511) / 512 * 512;  // 64-byte swizzle span
    static constexpr int kMetaOff = kStages * kStageBytes;
    static constexpr size_t kSmem = (size_t)kMetaOff + 2 * kMetaBytes + 512;  // + alignment slack
    static constexpr int kTokPerLane = NT == 4 ? 1 : NT == 8 ? 2 : 4;
    static_assert(kXBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
};

// Digit row of plane p, token m.
template <int NT>
__host__ __device__ constexpr int mt_row(int p, int m) {
    return NT == 4 ? (p < 2 ? 2 * m + p : 8 + 2 * m) : p * NT + m;
}

// Token of a lane's q-th accumulator column pair.
template <int NT>
__device__ __forceinline__ int mt_token(int tig, int q) {
    return NT == 4 ? tig : (q < 2 ? 2 * tig + q : 8 + 2 * tig + (q - 2));
}

struct MtArgs {
    const uint8_t* xrows;  // [G][kXBytes]: the launch's digit rows and per-token sums and scales
    const uint16_t* scales;
    const int32_t* zeros;
    uint16_t* Y;           // [M][N]
    float* partial;        // [row_tiles][max_slots][M][128]
    int* fault;
    int M, N, G;
    int units_base, units_rem;
    int max_slots;
};

// One warp per (group g, token m < NT): the digit rows of token m (zero for m >= M) and its
// (sum x_int, 2^(E - 21)).  xscale (nullable): each x is first replaced by bf16(x * xscale[k]) (the AWQ
// activation transform).
template <int NT>
__global__ void __launch_bounds__(256) prep_mt_kernel(const uint16_t* __restrict__ X, const float* __restrict__ xscale,
                                                      int M, int K, uint8_t* __restrict__ out) {
    using C = MtCfg<NT>;
    pdl_launch_dependents();
    pdl_wait_primary();  // X may come from the preceding kernel
    const int G = K / kGroup;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)G * NT;
    for (int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid < warps;
         wid += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int g = (int)(wid / NT), m = (int)(wid - (int64_t)g * NT);
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
        uint32_t plane[3];
        int E;
        const int sum = group_digits_i4(bits, lane, plane, &E);
        uint8_t* dst = out + (int64_t)g * C::kXBytes;
        const int off = 8 * (lane >> 1) + 4 * (lane & 1);
#pragma unroll
        for (int p = 0; p < 3; ++p) *reinterpret_cast<uint32_t*>(dst + mt_row<NT>(p, m) * 128 + off) = plane[p];
        if constexpr (NT == 4) *reinterpret_cast<uint32_t*>(dst + (9 + 2 * m) * 128 + off) = 0u;  // unused column
        if (lane == 0) {
            float* ext = reinterpret_cast<float*>(dst + C::kXRows * 128);
            ext[2 * m] = m < M ? (float)sum : 0.f;
            ext[2 * m + 1] = m < M ? pow2f(E - 21) : 0.f;
        }
    }
}

// mma.sync m16n8k32, A 16 x 32 unsigned bytes, B 32 x 8 signed bytes, D (+)= int32.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 3) decode_mt_kernel(const __grid_constant__ CUtensorMap tq,
                                                                const __grid_constant__ CUtensorMap tsc,
                                                                const __grid_constant__ CUtensorMap tze,
                                                                const MtArgs a) {
    using C = MtCfg<NT>;
    constexpr int TPL = C::kTokPerLane;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((512u - (raw & 511u)) & 511u);  // 512-aligned stages
    unsigned char* meta = ring + C::kMetaOff;

    pdl_launch_dependents();  // the next call may start its weight loads as this grid's CTAs retire
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int64_t u_first = (int64_t)b * a.units_base + min(b, a.units_rem);
    const int nunits = a.units_base + (b < a.units_rem ? 1 : 0);
    const int G = a.G, N = a.N, M = a.M;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);  // the TMA thread, with the transaction bytes
            mbar_init(&empty[s], kWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kTmaWarp) {  // --------------------------------------------------------- TMA
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tsc);
            prefetch_tmap(&tze);
            // codes and metadata need nothing from the preceding kernels: the first stages' loads go
            // out at once; their digit rows follow the dependent-launch wait
            const int pre = min(kStages, nunits);
            bool rows_first = false;  // digit rows of the first `pre` stages issued
            auto first_rows = [&]() {
                pdl_wait_primary();
                UnitCursor cx(u_first, G);
                for (int j = 0; j < pre; ++j, cx.next(G))
                    bulk_load(ring + j * C::kStageBytes + C::kXOff, a.xrows + (int64_t)cx.g * C::kXBytes, C::kXBytes,
                              &full[j]);
                rows_first = true;
            };
            UnitCursor cur(u_first, G);
            int mb = -1, issued = 0;
            for (int i = 0; i < nunits; ++i, cur.next(G)) {
                const int s = i % kStages;
                if (i == pre) first_rows();  // before waiting on a stage whose consumers need them
                if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, a.fault, 121)) break;
                const bool new_block = i == 0 || (cur.g & (kMetaGroups - 1)) == 0;
                if (new_block) ++mb;
                unsigned char* st = ring + s * C::kStageBytes;
                mbar_arrive_expect_tx(&full[s], kCodeBytes + C::kXBytes + (new_block ? kMetaBytes : 0));
                tma_load_2d(st, &tq, cur.g * kWordsPerGroup, cur.tile * kRows, &full[s]);
                if (new_block) {
                    unsigned char* ms = meta + (mb & 1) * kMetaBytes;
                    const int g8 = cur.g & ~(kMetaGroups - 1);
                    tma_load_2d(ms, &tsc, g8, cur.tile * kRows, &full[s]);
                    tma_load_2d(ms + kScBytes, &tze, g8, cur.tile * kRows, &full[s]);
                }
                if (i >= pre) bulk_load(st + C::kXOff, a.xrows + (int64_t)cur.g * C::kXBytes, C::kXBytes, &full[s]);
                ++issued;
            }
            if (!rows_first && pre > 0) first_rows();  // nunits <= kStages: every stage's rows still owed
            // no copy may still be in flight when the CTA exits
            for (int i = max(0, issued - kStages); i < issued; ++i)
                mbar_wait(&full[i % kStages], (i / kStages) & 1, a.fault, 122);
        }
        return;
    }

    // -------------------------------------------------------------------- compute warps 0-3
    // Warp w takes rows 16 kRB w .. as kRB 16-row MMA blocks; lane (g8, tig) = (lane / 4, lane % 4)
    // holds rows g8 and g8 + 8 of each block and words 4 tig .. 4 tig + 3 of each row's codes (one
    // 16-byte chunk); MMA j takes word 4 tig + j of every lane, and the lane's B fragments are the same
    // words of digit row 8 tile + g8.  Row k (k < 2 kRB) of the lane: block k / 2, half k % 2.
    constexpr int KR = 2 * kRB;
    const int g8 = lane >> 2, tig = lane & 3;
    auto rrow = [&](int k) { return 16 * kRB * warp + 16 * (k >> 1) + g8 + 8 * (k & 1); };
    float y[KR][TPL];
#pragma unroll
    for (int k = 0; k < KR; ++k)
#pragma unroll
        for (int q = 0; q < TPL; ++q) y[k][q] = 0.f;
    int cur_tile = -1;
    bool aborted = false;

    auto flush = [&](int tile) {
        const int first = cta_of_unit((int64_t)tile * G, a.units_base, a.units_rem);
        const int last = cta_of_unit((int64_t)tile * G + G - 1, a.units_base, a.units_rem);
        if (first == last) {
#pragma unroll
            for (int q = 0; q < TPL; ++q) {
                const int m = mt_token<NT>(tig, q);
                if (m < M) {
#pragma unroll
                    for (int k = 0; k < KR; ++k) {
                        const int n = tile * kRows + rrow(k);
                        if (n < N) a.Y[(int64_t)m * N + n] = float_to_bf16_bits(y[k][q]);
                    }
                }
            }
        } else {  // this CTA's partial-sum slot of the tile (decode_reduce_kernel adds the slots)
            float* part = a.partial + ((int64_t)tile * a.max_slots + (b - first)) * M * kRows;
#pragma unroll
            for (int q = 0; q < TPL; ++q) {
                const int m = mt_token<NT>(tig, q);
                if (m < M) {
#pragma unroll
                    for (int k = 0; k < KR; ++k) part[m * kRows + rrow(k)] = y[k][q];
                }
            }
        }
#pragma unroll
        for (int k = 0; k < KR; ++k)
#pragma unroll
            for (int q = 0; q < TPL; ++q) y[k][q] = 0.f;
    };

    UnitCursor uc(u_first, G);
    int mb = -1;
    for (int i = 0; i < nunits; ++i, uc.next(G)) {
        const int tile = uc.tile, g = uc.g;
        if (i == 0 || (g & (kMetaGroups - 1)) == 0) ++mb;
        if (tile != cur_tile) {
            if (cur_tile >= 0) flush(cur_tile);
            cur_tile = tile;
        }
        if (aborted) continue;
        const int s = i % kStages;
        if (!warp_wait(&full[s], (i / kStages) & 1, a.fault, 123)) {
            aborted = true;
            continue;
        }
        const unsigned char* st = ring + s * C::kStageBytes;
        // codes: chunk tig of each row, 64-byte swizzle (chunk c of row r at c ^ ((r >> 1) & 3)), as the
        // A fragments of both row blocks: A register set j of block rb = codes of word 4 tig + j of rows
        // g8 and g8 + 8, low nibbles then high nibbles
        uint32_t A[kRB][4][4];
#pragma unroll
        for (int rb = 0; rb < kRB; ++rb) {
            const int r0 = rrow(2 * rb), r1 = rrow(2 * rb + 1);
            const uint4 c0 = *reinterpret_cast<const uint4*>(st + r0 * 64 + 16 * (tig ^ ((r0 >> 1) & 3)));
            const uint4 c1 = *reinterpret_cast<const uint4*>(st + r1 * 64 + 16 * (tig ^ ((r1 >> 1) & 3)));
            const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w}, w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                A[rb][j][0] = w0[j] & 0x0F0F0F0Fu;
                A[rb][j][1] = w1[j] & 0x0F0F0F0Fu;
                A[rb][j][2] = (w0[j] >> 4) & 0x0F0F0F0Fu;
                A[rb][j][3] = (w1[j] >> 4) & 0x0F0F0F0Fu;
            }
        }
        // this block's metadata (loaded with its first unit, which this warp has already waited for);
        // rows past N were zero-filled by TMA: s = 0 folds them away
        const unsigned char* ms = meta + (mb & 1) * kMetaBytes;
        const int gb = g & (kMetaGroups - 1);
        float sv[KR], zv[KR];
#pragma unroll
        for (int k = 0; k < KR; ++k) {
            const int r = rrow(k);
            sv[k] = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(ms + r * (kMetaGroups * 2) + 2 * gb));
            zv[k] = (float)*reinterpret_cast<const int32_t*>(ms + kScBytes + r * (kMetaGroups * 4) + 4 * gb);
        }
        const float* ext = reinterpret_cast<const float*>(st + C::kXOff + C::kXRows * 128);
        const unsigned char* xr = st + C::kXOff + g8 * 128 + tig * 32;

        // The folds of tokens whose planes sit in tiles t0, t1, t2 (columns 2 tig + j, j < JN):
        //   y[k][q0 + j] += s (65536 P2 + 256 P1 + P0 - z sum) 2^(E - 21)
        auto mma_fold = [&](const int (&tl)[3], int q0, int JN, bool release) {
            uint32_t bx[3][8];
#pragma unroll
            for (int u = 0; u < 3; ++u) {
                if (u == 2 && NT == 4) continue;  // NT = 4: planes 0 and 1 share tile 0
                const uint4* xp = reinterpret_cast<const uint4*>(xr + tl[u] * 8 * 128);
                const uint4 u0 = xp[0], u1 = xp[1];
                bx[u][0] = u0.x; bx[u][1] = u0.y; bx[u][2] = u0.z; bx[u][3] = u0.w;
                bx[u][4] = u1.x; bx[u][5] = u1.y; bx[u][6] = u1.z; bx[u][7] = u1.w;
            }
            float xs[2], xc[2];
#pragma unroll
            for (int j = 0; j < JN; ++j) {
                const int m = mt_token<NT>(tig, q0 + j);
                xs[j] = ext[2 * m];
                xc[j] = ext[2 * m + 1];
            }
            if (release) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            constexpr int NTL = NT == 4 ? 2 : 3;
#pragma unroll
            for (int rb = 0; rb < kRB; ++rb) {
                int d[3][4];
#pragma unroll
                for (int u = 0; u < NTL; ++u) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[u][e] = kPlaneBias;
#pragma unroll
                    for (int j = 0; j < 4; ++j) mma_u8s8(d[u], A[rb][j], bx[u][2 * j], bx[u][2 * j + 1]);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int k = 2 * rb + h;
#pragma unroll
                    for (int j = 0; j < JN; ++j) {
                        int P0, P1, P2;
                        if constexpr (NT == 4) {  // tile 0: (P0, P1) of token tig; tile 1: (P2, -)
                            P0 = d[0][2 * h];
                            P1 = d[0][2 * h + 1];
                            P2 = d[1][2 * h];
                        } else {  // tile u: plane u of tokens 2 tig + j
                            P0 = d[0][2 * h + j];
                            P1 = d[1][2 * h + j];
                            P2 = d[2][2 * h + j];
                        }
                        // each plane sum is biased: its bits read as FP32 are 1.5 2^23 + P, so one exact
                        // subtraction converts it; 256 P1 + P0 is rounded once, by the inner FMA
                        const float F0 = __int_as_float(P0) - 12582912.f, F1 = __int_as_float(P1) - 12582912.f,
                                    F2 = __int_as_float(P2) - 12582912.f;
                        const float qx = fmaf(F2, 65536.f, fmaf(F1, 256.f, F0));
                        y[k][q0 + j] = fmaf(sv[k] * fmaf(-zv[k], xs[j], qx), xc[j], y[k][q0 + j]);
                    }
                }
            }
        };
        if constexpr (NT == 4) {
            const int tl[3] = {0, 1, 1};
            mma_fold(tl, 0, 1, true);
        } else if constexpr (NT == 8) {
            const int tl[3] = {0, 1, 2};
            mma_fold(tl, 0, 2, true);
        } else {
            const int tl0[3] = {0, 2, 4}, tl1[3] = {1, 3, 5};
            mma_fold(tl0, 0, 2, false);
            mma_fold(tl1, 2, 2, true);
        }
    }
    if (cur_tile >= 0) flush(cur_tile);
}

template <int NT>
int mt_occupancy() {
    static PerContext<int> cache;  // the attribute and occupancy belong to a context
    return cache.get([]() -> int {
        if (cudaFuncSetAttribute(decode_mt_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)MtCfg<NT>::kSmem) != cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, decode_mt_kernel<NT>, kThreads, MtCfg<NT>::kSmem) !=
                cudaSuccess ||
            o < 1)
            return 0;
        return o;
    });
}

int mt_occupancy(int nt) { return nt == 4 ? mt_occupancy<4>() : nt == 8 ? mt_occupancy<8>() : mt_occupancy<16>(); }

int mt_x_bytes(int nt) { return nt == 4 ? MtCfg<4>::kXBytes : nt == 8 ? MtCfg<8>::kXBytes : MtCfg<16>::kXBytes; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct MtPlan {
    int nt, grid, units_base, units_rem, max_slots, row_tiles;
};

MtPlan plan_mt(int nt, int64_t N, int64_t K, int num_sms) {
    MtPlan p{};
    p.nt = nt;
    const int64_t G = K / kGroup;
    p.row_tiles = (int)ceil_div(N, kRows);
    const int64_t units = (int64_t)p.row_tiles * G;
    int occ = mt_occupancy(nt);
    if (occ < 1) occ = 1;
    int64_t grid = (int64_t)occ * num_sms;
    if (grid > units) grid = units;
    p.grid = (int)grid;
    p.units_base = (int)(units / grid);
    p.units_rem = (int)(units % grid);
    p.max_slots = (int)((G - 1) / p.units_base + 2);
    return p;
}

// Token tile for the chunk of `tokens` (<= 16) tokens.
int mt_nt_for(int tokens) { return tokens <= 4 ? 4 : tokens <= 8 ? 8 : 16; }

template <int NT>
int launch_mt_kernel(const CUtensorMap& tq, const CUtensorMap& tsc, const CUtensorMap& tze, const MtArgs& args,
                     int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = MtCfg<NT>::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_mt_kernel<NT>, tq, tsc, tze, args) == cudaSuccess ? W4A16_OK
                                                                                            : W4A16_ERR_CUDA;
}

template <int NT>
int launch_prep(const uint16_t* X, const float* xscale, int Mc, int K, uint8_t* out, cudaStream_t stream) {
    const int64_t threads = (int64_t)(K / kGroup) * NT * 32;
    int grid = (int)ceil_div(threads, 256);
    if (grid > num_sms_current() * 8) grid = num_sms_current() * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prep_mt_kernel<NT>, X, xscale, Mc, K, out) == cudaSuccess ? W4A16_OK
                                                                                               : W4A16_ERR_CUDA;
}

}  // namespace

bool mt_supported(int64_t K) { return (K / kGroup) % kMetaGroups == 0; }

size_t mt_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
    const int64_t G = K / kGroup;
    size_t need = 0;
    for (int nt : {4, 8, 16}) {
        if (nt > 4 && mt_nt_for((int)(M < 16 ? M : 16)) < nt) break;
        const MtPlan p = plan_mt(nt, N, K, num_sms);
        const int mc = (int)(M < nt ? M : nt);
        const size_t b = align256((size_t)G * mt_x_bytes(nt)) +
                         align256((size_t)p.row_tiles * p.max_slots * mc * kRows * 4);
        if (b > need) need = b;
    }
    return need;
}

int launch_decode_mt(const uint16_t* X, const float* xscale, int64_t M, int64_t K, const uint32_t* qweight,
                     const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* scratch,
                     cudaStream_t stream) {
    const int G = (int)(K / kGroup);
    CUtensorMap tq, tsc, tze;
    if (!tmap_2d_cached(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)K / 8, (uint64_t)N, (uint64_t)K / 2,
                        kWordsPerGroup, kRows, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !tmap_2d_cached(&tsc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, scales, (uint64_t)G, (uint64_t)N, (uint64_t)G * 2,
                        kMetaGroups, kRows) ||
        !tmap_2d_cached(&tze, CU_TENSOR_MAP_DATA_TYPE_INT32, zeros, (uint64_t)G, (uint64_t)N, (uint64_t)G * 4,
                        kMetaGroups, kRows))
        return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    const int sms = num_sms_current();
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        const int Mc = (int)(M - m0 < 16 ? M - m0 : 16);
        const int nt = mt_nt_for(Mc);
        const MtPlan p = plan_mt(nt, N, K, sms);
        uint8_t* xrows = reinterpret_cast<uint8_t*>(scratch);
        float* partial = reinterpret_cast<float*>(reinterpret_cast<char*>(scratch) +
                                                  align256((size_t)G * mt_x_bytes(nt)));
        const uint16_t* Xc = X + m0 * K;
        int st = nt == 4   ? launch_prep<4>(Xc, xscale, Mc, (int)K, xrows, stream)
                 : nt == 8 ? launch_prep<8>(Xc, xscale, Mc, (int)K, xrows, stream)
                           : launch_prep<16>(Xc, xscale, Mc, (int)K, xrows, stream);
        if (st != W4A16_OK) return st;
        MtArgs args;
        args.xrows = xrows;
        args.scales = scales;
        args.zeros = zeros;
        args.Y = Y + m0 * N;
        args.partial = partial;
        args.fault = fault;
        args.M = Mc;
        args.N = (int)N;
        args.G = G;
        args.units_base = p.units_base;
        args.units_rem = p.units_rem;
        args.max_slots = p.max_slots;
        st = nt == 4   ? launch_mt_kernel<4>(tq, tsc, tze, args, p.grid, stream)
             : nt == 8 ? launch_mt_kernel<8>(tq, tsc, tze, args, p.grid, stream)
                       : launch_mt_kernel<16>(tq, tsc, tze, args, p.grid, stream);
        if (st != W4A16_OK) return st;
        st = launch_decode_reduce(partial, args.Y, N, Mc, G, p.units_base, p.units_rem, p.max_slots, p.row_tiles,
                                  stream);
        if (st != W4A16_OK) return st;
    }
    return W4A16_OK;
}

}  // namespace w4a16
