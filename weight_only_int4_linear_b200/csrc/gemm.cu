// Prefill path of the W4A16 linear layer: a persistent, warp-specialised
// tcgen05 GEMM for large M.
//
// The weights are dequantised tile by tile on chip and never written back:
// packed codes arrive by TMA, dequantiser warps expand them to BF16 operand
// tiles in shared memory, and the 5th-generation tensor cores multiply them
// with BF16 X tiles ("Weight-Only Quantization and Mixed Precision",
// section 7: fused read, unpack, dequantise and matmul, asynchronous copies
// overlapping the math; "Quantization I: int8, int4, the basics", Concept:
// dequantise tile by tile inside the multiply, accumulate in higher precision).
//
// Arithmetic: per group g of 128 weights along K,
//   Y[m][n] += s[n][g] * sum_k (q[n][k] - c) x[m][k]  -  s[n][g] (z[n][g] - c) xsum[m][g]
// The dequantiser forms (128 + q) in BF16 (0x4300 | q, one lop3 per two codes)
// and subtracts (128 + c) with one packed BF16 subtract, exact because both
// are integers of magnitude <= 256: c = z whenever |z| <= 128 (every group
// whose range straddles zero), else c = 0.  The inner sum runs on the tensor
// cores into a per-group FP32 accumulator in tensor memory; the fold is one
// FP32 FMA per element, T += s * D, plus the xsum term for the rare rows with
// c != z.  The BF16 scale never enters a rounded operand; the only rounding
// besides FP32 summation is the final BF16 rounding of Y.
//
// Tile: 256 weight rows (MMA M) x 256 tokens (MMA N, swap-AB so the per-row
// scale is a per-thread constant in the fold), computed by a cluster of two
// CTAs with the pair MMA (tcgen05.mma.cta_group::2): each CTA dequantises its
// own 128 weight rows into its shared memory, holds half of the tile's X rows
// (the MMA exchanges the B halves between the pair), and receives its 128
// rows of the FP32 accumulator in its own tensor memory.  Per CTA this halves
// the X bytes that TMA writes and the MMA reads from shared memory against a
// one-CTA 128 x 256 tile, which leaves room for six stages.  Rank 0 issues
// the MMAs; both CTAs' dequantiser and fold warps arrive on rank 0's barriers
// (mapa + remote mbarrier arrive), and its commits arrive on both CTAs'
// barriers (multicast commit).  No TMA load is multicast.  K advances in
// stages of 64 (half a group).  MMA K order inside each 8-block of K is
// (0,4,1,5,2,6,3,7): that is the order a lop3 pair extraction yields, and X
// is prepared in it.  (Built with W4A16_PF_CTAS=1 the same kernel runs one
// CTA per 128 x 256 tile with cta_group::1.)
//
// Warps (512 threads per CTA with 8 fold warps):
//   0-3   dequantise: thread = weight row; 8 packed words -> one 128-byte
//         row of the 128B-swizzled K-major A tile
//   4-11  fold + epilogue: warp w reads TMEM lane quadrant w % 4, token
//         columns 128 * ((w - 4) / 4) ... + 127; totals live in registers;
//         T += s * D as packed FP32 FMAs (fma.rn.f32x2)
//   12    TMA: this CTA's X half (128 x 64, 128-byte swizzle) and code tile
//         (128 x 8 words, 32-byte swizzle) per stage
//   13    MMA issue (rank 0): four tcgen05.mma (256 x 256 x 16) per stage
//   14-15 idle
// Accumulators: two 256-column TMEM buffers, one per group in flight, so the
// fold of group g overlaps the MMAs of group g + 1.
#include "common.cuh"
#include "sm100.cuh"

#include <mutex>

namespace w4a16 {
namespace {

#ifndef W4A16_PF_CTAS
#define W4A16_PF_CTAS 2
#endif
constexpr int kPCtas = W4A16_PF_CTAS;          // CTAs per MMA: 1 (cta_group::1) or a 2-CTA cluster (cta_group::2)
static_assert(kPCtas == 1 || kPCtas == 2, "CTAs per MMA");
constexpr int kPBM = 128;                      // weight rows per CTA (the MMA covers kPBM * kPCtas)
constexpr int kPBN = 256;                      // tokens per tile
constexpr int kPBNc = kPBN / kPCtas;           // tokens whose X tile this CTA holds (B split along N)
constexpr int kPBK = 64;                       // K per stage
#ifndef W4A16_PF_STAGES
#define W4A16_PF_STAGES (kPCtas == 2 ? 6 : 4)
#endif
constexpr int kPStages = W4A16_PF_STAGES;
constexpr int kPXBytes = kPBNc * kPBK * 2;     // 32 KB (1 CTA) or 16 KB (2 CTAs)
constexpr int kPABytes = kPBM * kPBK * 2;      // 16 KB
constexpr int kPCodeBytes = kPBM * kPBK / 2;   // 4 KB
constexpr int kPStageBytes = kPXBytes + kPABytes + kPCodeBytes;  // 52 KB or 36 KB (1024-aligned)
static_assert(kPStageBytes % 1024 == 0, "stage alignment");
constexpr size_t kPSmem = (size_t)kPStages * kPStageBytes + 1024;  // + alignment slack
static_assert(kPSmem + 512 <= 232448, "shared memory per CTA");
#ifndef W4A16_PF_FOLD_WARPS
#define W4A16_PF_FOLD_WARPS 8
#endif
constexpr int kPFoldWarps = W4A16_PF_FOLD_WARPS;          // 8 or 16 (2 or 4 per TMEM lane quadrant)
constexpr int kPFoldParts = kPFoldWarps / 4;              // token column slices per lane quadrant
constexpr int kPFoldCols = kPBN / kPFoldParts;            // token columns per fold thread: 128 or 64
constexpr int kPThreads = (4 + kPFoldWarps + 4) * 32;     // dequant warpgroup, fold warpgroups, TMA/MMA warpgroup
constexpr int kPTmaWarp = 4 + kPFoldWarps, kPMmaWarp = kPTmaWarp + 1;
// register split: every warp starts with the launch share (65536 / threads, a multiple of 8);
// setmaxnreg moves registers from the dequantisers and the TMA/MMA warpgroup to the fold warps
constexpr int kPRegsLaunch = (65536 / kPThreads) & ~7;
constexpr int kPRegsDequant = 56;
constexpr int kPRegsIssue = kPFoldWarps == 16 ? 40 : 72;
constexpr int kPRegsFold = kPFoldWarps == 16 ? 96 : 192;
static_assert(32 * (4 * kPRegsDequant + 4 * kPRegsIssue + kPFoldWarps * kPRegsFold) <= kPRegsLaunch * kPThreads,
              "setmaxnreg split exceeds the registers the block is launched with");
static_assert(kPFoldWarps == 8 || kPFoldWarps == 16, "fold warps");
constexpr int kPLdCols = kPFoldWarps == 16 ? 8 : 16;    // TMEM columns per fold load
constexpr uint32_t kPIdesc = idesc_bf16_f32(kPBM * kPCtas, kPBN);

struct PrefillArgs {
    const uint16_t* scales;
    const int32_t* zeros;
    const float* xsT;  // [G][Mp]: per-group sums of X, Mp = M rounded up to a multiple of 256 (zero past M)
    uint16_t* Y;
    int* fault;
    int M, N, K, G, Mp;
    int m_tiles, n_tiles;       // tiles of 256 tokens x (128 x CTAs per MMA) weight rows
    int tiles, units;           // MMA unit (CTA or cluster) b runs tiles b, b + units, b + 2 units, ...
};

__device__ __forceinline__ uint32_t magic_pair(uint32_t w) {
    uint32_t r;
    asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(w));  // (w & m) | c
    return r;
}

// (a - b) on BF16 pairs; exact here (integers of magnitude <= 256).
__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint4 permute_block(uint4 v) {
    uint4 o;
    o.x = __byte_perm(v.x, v.z, 0x5410);  // x0, x4
    o.y = __byte_perm(v.x, v.z, 0x7632);  // x1, x5
    o.z = __byte_perm(v.y, v.w, 0x5410);  // x2, x6
    o.w = __byte_perm(v.y, v.w, 0x7632);  // x3, x7
    return o;
}

// X -> Xp (each 8-block reordered (0,4,1,5,2,6,3,7)) and xsT[g][m] = sum of quantisation group g of
// GS weights (row stride Mp, a multiple of the 256-token tile so one bulk copy per group and tile
// reads it).  xscale (nullable): each x is first replaced by bf16(x * xscale[k]) (AWQ).
template <int GS>
__global__ void __launch_bounds__(256) prefill_prep_kernel(const uint16_t* __restrict__ X,
                                                           const float* __restrict__ xscale, int M, int K, int Mp,
                                                           uint16_t* __restrict__ Xp, float* __restrict__ xsT) {
    pdl_launch_dependents();
    const int G = K / kGroup;
    const int64_t units = (int64_t)M * G * 16;  // multiple of 16
    for (int64_t u0 = (int64_t)blockIdx.x * blockDim.x; u0 < units; u0 += (int64_t)gridDim.x * blockDim.x) {
        const int64_t u = u0 + threadIdx.x;
        const bool active = u < units;
        const int64_t mg = u >> 4;  // (m, g) pair, g fastest
        const int blk = (int)(u & 15);
        const int m = (int)(mg / G), g = (int)(mg - (int64_t)m * G);
        float sum = 0.f;
        if (active) {
            const int64_t off = (int64_t)m * K + (int64_t)g * kGroup + blk * 8;
            uint4 v = *reinterpret_cast<const uint4*>(X + off);
            if (xscale) {
                const float4* r = reinterpret_cast<const float4*>(xscale + (int64_t)g * kGroup + blk * 8);
                const float4 r0 = __ldg(r), r1 = __ldg(r + 1);
                v = make_uint4(bf16x2_scaled(v.x, r0.x, r0.y), bf16x2_scaled(v.y, r0.z, r0.w),
                               bf16x2_scaled(v.z, r1.x, r1.y), bf16x2_scaled(v.w, r1.z, r1.w));
            }
            *reinterpret_cast<uint4*>(Xp + off) = permute_block(v);
            sum = (bf16lo(v.x) + bf16hi(v.x)) + (bf16lo(v.y) + bf16hi(v.y)) + (bf16lo(v.z) + bf16hi(v.z)) +
                  (bf16lo(v.w) + bf16hi(v.w));
        }
        constexpr int LPG = GS / 8;  // lanes (8-blocks) per quantisation group, aligned in the block of 16
#pragma unroll
        for (int o = LPG / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (active && blk % LPG == 0) xsT[((int64_t)g * (kGroup / GS) + blk / LPG) * Mp + m] = sum;
    }
}

// (t0, t1) = fma(s, d0, t0), fma(s, d1, t1) as one packed FP32 instruction (each lane a correctly
// rounded fused multiply-add: the same bits as two fmaf calls).
__device__ __forceinline__ void fma2_bcast(float& t0, float& t1, float s, uint32_t d0, uint32_t d1) {
    asm("{\n\t.reg .b64 sa, da, ta;\n\t"
        "mov.b64 sa, {%2, %2};\n\t"
        "mov.b64 da, {%3, %4};\n\t"
        "mov.b64 ta, {%0, %1};\n\t"
        "fma.rn.f32x2 ta, sa, da, ta;\n\t"
        "mov.b64 {%0, %1}, ta;\n\t}"
        : "+f"(t0), "+f"(t1)
        : "f"(s), "r"(d0), "r"(d1));
}

__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[8]) { tmem_ld8(taddr, r); }
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[16]) { tmem_ld16(taddr, r); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Tile t -> (weight row tile nt, token tile mt).  Groups of kPRaster token tiles are walked with
// the token tile fastest, so the tiles in flight at once (consecutive t, one per MMA unit) share a
// few X tiles and a few weight row tiles, and both stay in L2 between their uses.
#ifndef W4A16_PF_RASTER
#define W4A16_PF_RASTER 4
#endif
constexpr int kPRaster = W4A16_PF_RASTER;
__device__ __forceinline__ void tile_coords(int t, const PrefillArgs& a, int& nt, int& mt) {
    const int per_group = kPRaster * a.n_tiles;
    const int grp = t / per_group, r = t - grp * per_group;
    const int gm = min(kPRaster, a.m_tiles - grp * kPRaster);  // token tiles in this group (the last may be short)
    nt = r / gm;
    mt = grp * kPRaster + (r - nt * gm);
}

// Arrive on the MMA-issuing CTA's barrier (rank 0 of the cluster; this CTA with one CTA per MMA).
__device__ __forceinline__ void arrive_issuer(uint64_t* bar) {
    if constexpr (kPCtas == 2)
        mbar_arrive_cluster(bar, 0);
    else
        mbar_arrive(bar);
}


// GS: quantisation group size, 128 (two 64-K stages per group) or 64 (one stage per group).
template <int GS>
__global__ void __launch_bounds__(kPThreads, 1) prefill_kernel(const __grid_constant__ CUtensorMap tx,
                                                               const __grid_constant__ CUtensorMap tq,
                                                               const PrefillArgs a) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kPStages], afull[kPStages], empty[kPStages], mdone[2], dfree[2];
    __shared__ __align__(8) uint64_t drained;
    __shared__ uint32_t s_tmem;
    const uint32_t raw = smem_u32(smem_raw);
    // identical offsets in both CTAs of a cluster: the pair MMA reads the peer's tiles at this CTA's offsets
    unsigned char* ring = smem_raw + ((1024u - (raw & 1023u)) & 1023u);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = kPCtas == 2 ? cluster_ctarank() : 0u;
    const int b = blockIdx.x / kPCtas;  // MMA unit: this CTA or its cluster
    const int ntiles = b < a.tiles ? (a.tiles - 1 - b) / a.units + 1 : 0;  // tiles b, b + units, ...
    constexpr int kSpg = GS / kPBK;  // 64-K stages per quantisation group
    static_assert(kSpg * kPBK == GS && kSpg >= 1, "group size");
    const int G = a.G;               // quantisation groups per row
    const int stages_per_tile = kSpg * G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);  // TMA: X and codes tiles
            mbar_init(&afull[s], 4 * kPCtas);  // the dequantiser warps of every CTA of the MMA
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&mdone[i], 1);
            mbar_init(&dfree[i], kPFoldWarps * kPCtas);  // the fold warps of every CTA of the MMA
        }
        mbar_init(&drained, 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (warp == 0) {
        if constexpr (kPCtas == 2)
            tmem_alloc_pair(&s_tmem, 512);
        else
            tmem_alloc(&s_tmem, 512);
    }
    // barriers initialised and the TMEM base known in every CTA before any (remote) arrival
    if constexpr (kPCtas == 2)
        cluster_sync();
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int wg = warp >> 2;
    // register split (launch: 512 x 128 = 65536): 4 x 32 x (72 + 56 + 192 + 192) = 65536
    if (wg == 1 + kPFoldParts) {  // ------------------------------------------------ TMA + MMA
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPRegsIssue));
        if (warp == kPTmaWarp && lane == 0) {
            prefetch_tmap(&tx);
            prefetch_tmap(&tq);
            pdl_wait_primary();  // X comes from the preparation kernel
            int it = 0;
            for (int tt = 0; tt < ntiles; ++tt) {
                int nt, mt;
                tile_coords(b + tt * a.units, a, nt, mt);
                for (int ks = 0; ks < stages_per_tile; ++ks, ++it) {
                    const int s = it % kPStages;
                    if (it >= kPStages && !mbar_wait(&empty[s], ((it / kPStages) - 1) & 1, a.fault, 61)) goto done_tma;
                    unsigned char* st = ring + s * kPStageBytes;
                    mbar_arrive_expect_tx(&full[s], kPXBytes + kPCodeBytes);
                    tma_load_2d(st, &tx, ks * kPBK, mt * kPBN + (int)rank * kPBNc, &full[s]);
                    tma_load_2d(st + kPXBytes + kPABytes, &tq, ks * (kPBK / 8), (nt * kPCtas + (int)rank) * kPBM,
                                &full[s]);
                }
            }
        done_tma:
            // copies in flight land before the CTA may exit
            for (int i = max(0, it - kPStages); i < it; ++i) mbar_wait(&full[i % kPStages], (i / kPStages) & 1, a.fault, 62);
        } else if (warp == kPMmaWarp && lane == 0 && rank == 0) {
            // afull[s] also stands for full[s]: every dequantiser warp waited on its CTA's copies first
            int it = 0, gc = 0;
            for (int tt = 0; tt < ntiles; ++tt) {
                for (int ks = 0; ks < stages_per_tile; ++ks, ++it) {
                    const int s = it % kPStages;
                    const int half = ks % kSpg;  // stage within the quantisation group
                    const int dbuf = gc & 1;
                    if (half == 0 && gc >= 2 && !mbar_wait(&dfree[dbuf], ((gc >> 1) - 1) & 1, a.fault, 71)) goto done_mma;
                    if (!mbar_wait(&afull[s], (it / kPStages) & 1, a.fault, 73)) goto done_mma;
                    tc_fence_after();
                    const uint32_t xaddr = smem_u32(ring + s * kPStageBytes);
                    const uint32_t aaddr = xaddr + kPXBytes;
#pragma unroll
                    for (int kk = 0; kk < kPBK / 16; ++kk) {
                        const uint64_t ad = sw128_kmajor_desc(aaddr + kk * 32), bd = sw128_kmajor_desc(xaddr + kk * 32);
                        if constexpr (kPCtas == 2)
                            umma_ss_pair(tmem + dbuf * kPBN, ad, bd, kPIdesc, half > 0 || kk > 0);
                        else
                            umma_ss(tmem + dbuf * kPBN, ad, bd, kPIdesc, half > 0 || kk > 0);
                    }
                    if constexpr (kPCtas == 2) {
                        umma_commit_pair(&empty[s], 0x3);
                        if (half == kSpg - 1) umma_commit_pair(&mdone[dbuf], 0x3);
                    } else {
                        umma_commit(&empty[s]);
                        if (half == kSpg - 1) umma_commit(&mdone[dbuf]);
                    }
                    if (half == kSpg - 1) ++gc;
                }
            }
        done_mma:
            // every MMA issued (also on an early exit) completes before the teardown
            if constexpr (kPCtas == 2)
                umma_commit_pair(&drained, 0x1);
            else
                umma_commit(&drained);
            mbar_wait(&drained, 0, a.fault, 74);
        }
    } else if (wg == 0) {  // ------------------------------------ dequantisers
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPRegsDequant));
        const int r = threadIdx.x;  // weight row within this CTA's 128
        // codes tile: 32 bytes per row, 32-byte swizzle: 16-byte chunk c of row r at c ^ ((r >> 2) & 1)
        const int csw = (r >> 2) & 1;
        int it = 0;
        for (int tt = 0; tt < ntiles; ++tt) {
            int nt, mt;
            tile_coords(b + tt * a.units, a, nt, mt);
            const int n = (nt * kPCtas + (int)rank) * kPBM + r;
            uint32_t zc2 = 0x43004300u;  // (128 + c) as a BF16 pair
            for (int ks = 0; ks < stages_per_tile; ++ks, ++it) {
                const bool first_half = ks % kSpg == 0;  // first stage of a quantisation group
                if (first_half) {
                    const int z = n < a.N ? __ldg(a.zeros + (int64_t)n * G + ks / kSpg) : 0;
                    const int c = (z >= -128 && z <= 128) ? z : 0;
                    const uint32_t cb = __float_as_uint(128.f + (float)c) >> 16;  // exact: |128 + c| <= 256
                    zc2 = cb | (cb << 16);
                }
                const int s = it % kPStages;
                if (!mbar_wait(&full[s], (it / kPStages) & 1, a.fault, 81)) goto done_dq;
                unsigned char* st = ring + s * kPStageBytes;
                const unsigned char* codes = st + kPXBytes + kPABytes + r * 32;
                const uint4 c0 = *reinterpret_cast<const uint4*>(codes + 16 * csw);
                const uint4 c1 = *reinterpret_cast<const uint4*>(codes + 16 * (1 - csw));
                const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                // A row r: 128 bytes, 16-byte chunk j (word j) stored at chunk j ^ (r % 8)
                unsigned char* arow = st + kPXBytes + r * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t x = w[j];
                    const uint4 v = make_uint4(sub_bf16x2(magic_pair(x), zc2), sub_bf16x2(magic_pair(x >> 4), zc2),
                                               sub_bf16x2(magic_pair(x >> 8), zc2), sub_bf16x2(magic_pair(x >> 12), zc2));
                    *reinterpret_cast<uint4*>(arow + 16 * (j ^ (r & 7))) = v;
                }
                fence_proxy_async_shared();  // generic-proxy writes -> visible to the tensor core
                __syncwarp();
                if (lane == 0) arrive_issuer(&afull[s]);
            }
        }
    done_dq:;
    } else {  // -------------------------------------------- fold + epilogue (wg 1, 2)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPRegsFold));
        const int quad = warp & 3;
        const int colh = (warp - 4) >> 2;            // token column slice of the tile (kPFoldCols wide)
        const int row = quad * 32 + lane;            // weight row within this CTA's 128 = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        float T[kPFoldCols];
#pragma unroll
        for (int j = 0; j < kPFoldCols; ++j) T[j] = 0.f;
        int gc = 0;
        bool aborted = false;
        // this row's scale and zero point, loaded one group ahead of their use (rows past N: scale 0)
        auto row_of = [&](int tt2) {
            int nt2, mt2;
            tile_coords(b + tt2 * a.units, a, nt2, mt2);
            return (nt2 * kPCtas + (int)rank) * kPBM + row;
        };
        uint32_t s_nx = 0;
        int z_nx = 0;
        if (ntiles > 0) {
            const int n0 = row_of(0);
            s_nx = n0 < a.N ? __ldg(a.scales + (int64_t)n0 * G) : 0u;
            z_nx = n0 < a.N ? __ldg(a.zeros + (int64_t)n0 * G) : 0;
        }
        for (int tt = 0; tt < ntiles; ++tt) {
            int nt, mt;
            tile_coords(b + tt * a.units, a, nt, mt);
            const int n = (nt * kPCtas + (int)rank) * kPBM + row;
            const int n_next = tt + 1 < ntiles ? row_of(tt + 1) : a.N;  // the next tile's row (a.N: none)
            const int m0 = mt * kPBN + colh * kPFoldCols;
            for (int g = 0; g < G; ++g, ++gc) {
                const int dbuf = gc & 1;
                const uint32_t s_cur = s_nx;
                const int z_cur = z_nx;
                const int nn = g + 1 < G ? n : n_next, gn = g + 1 < G ? g + 1 : 0;
                s_nx = nn < a.N ? __ldg(a.scales + (int64_t)nn * G + gn) : 0u;
                z_nx = nn < a.N ? __ldg(a.zeros + (int64_t)nn * G + gn) : 0;
                if (!aborted && !mbar_wait(&mdone[dbuf], (gc >> 1) & 1, a.fault, 91)) aborted = true;
                if (!aborted) {
                    const float sv = bf16_bits_to_float((uint16_t)s_cur), zv = (float)z_cur;
                    // rows whose zero point was not subtracted by the dequantiser (|z| > 128) fold
                    // - s (z - c) xsum with c = 0, the X sums of this thread's tokens read from global memory
                    const float zr = (z_cur >= -128 && z_cur <= 128) ? 0.f : zv;
                    const bool need_xs = __any_sync(0xFFFFFFFFu, zr != 0.f);
                    const float* xs = a.xsT + (int64_t)g * a.Mp + m0;
                    tc_fence_after();
#pragma unroll
                    for (int cc = 0; cc < kPFoldCols / kPLdCols; ++cc) {
                        const int j0 = cc * kPLdCols;
                        uint32_t d[kPLdCols];
                        tmem_ldn(tl + dbuf * kPBN + colh * kPFoldCols + j0, d);
                        tmem_wait_ld();
                        if (!need_xs) {
#pragma unroll
                            for (int e = 0; e < kPLdCols; e += 2) fma2_bcast(T[j0 + e], T[j0 + e + 1], sv, d[e], d[e + 1]);
                        } else {
#pragma unroll
                            for (int j4 = 0; j4 < kPLdCols / 4; ++j4) {
                                const float4 xv = __ldg(reinterpret_cast<const float4*>(xs + j0 + 4 * j4));
                                const float xq[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int j = j0 + 4 * j4 + e;
                                    T[j] = fmaf(sv, fmaf(-zr, xq[e], __uint_as_float(d[4 * j4 + e])), T[j]);
                                }
                            }
                        }
                    }
                    tc_fence_before();
                }
                __syncwarp();
                if (lane == 0 && !aborted) arrive_issuer(&dfree[dbuf]);
            }
            // epilogue: this thread's row n, tokens m0 .. m0 + kPFoldCols - 1
            if (n < a.N) {
#pragma unroll
                for (int j = 0; j < kPFoldCols; ++j) {
                    const int m = m0 + j;
                    if (m < a.M) a.Y[(int64_t)m * a.N + n] = float_to_bf16_bits(T[j]);
                }
            }
#pragma unroll
            for (int j = 0; j < kPFoldCols; ++j) T[j] = 0.f;
        }
    }
    // teardown: every role done, every MMA complete (drained), no arrival still bound for the peer
    __syncwarp();
    if constexpr (kPCtas == 2)
        cluster_sync();
    else
        __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        if constexpr (kPCtas == 2)
            tmem_dealloc_pair(tmem, 512);
        else
            tmem_dealloc(tmem, 512);
    }
}

std::mutex g_ptmap_mu;
struct PTmap {
    const void* ptr;
    int64_t rows, cols;
    int kind;
    CUtensorMap map;
};
PTmap g_ptmaps[64];
int g_ptmap_next = 0;

bool prefill_tmap(int kind, const void* ptr, int64_t rows, int64_t cols, CUtensorMap* out) {
    std::lock_guard<std::mutex> lk(g_ptmap_mu);
    for (auto& e : g_ptmaps)
        if (e.ptr == ptr && e.rows == rows && e.cols == cols && e.kind == kind) {
            *out = e.map;
            return true;
        }
    PTmap& e = g_ptmaps[g_ptmap_next];
    bool ok;
    if (kind == 0)  // prepared X: bf16 [M][K], box 64 x (this CTA's tokens), 128-byte swizzle
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 2, kPBK, kPBNc, CU_TENSOR_MAP_SWIZZLE_128B);
    else  // packed weights: uint32 [N][K/8], box 8 words x 128 rows, 32-byte swizzle
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT32, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 4, kPBK / 8, kPBM, CU_TENSOR_MAP_SWIZZLE_32B);
    if (!ok) return false;
    e.ptr = ptr;
    e.rows = rows;
    e.cols = cols;
    e.kind = kind;
    g_ptmap_next = (g_ptmap_next + 1) % 64;
    *out = e.map;
    return true;
}

size_t align256p(size_t x) { return (x + 255) & ~(size_t)255; }

// MMA units of the prefill kernel that fit on the current device at once (cached per context).
template <class Kern>
int prefill_resident_units(const cudaLaunchConfig_t& cfg, Kern kernel) {
    static PerContext<int> cache;  // the same for both group sizes: same resources
    return cache.get([&]() -> int {
        int units = 0;
        if constexpr (kPCtas == 1) {
            units = num_sms_current();
        } else {
            cudaLaunchConfig_t q = cfg;
            q.gridDim = dim3((unsigned)(kPCtas * num_sms_current()));
            if (cudaOccupancyMaxActiveClusters(&units, kernel, &q) != cudaSuccess) {
                cudaGetLastError();
                return 0;
            }
        }
        return units;
    });
}

}  // namespace

size_t prefill_workspace_bytes(int64_t M, int64_t K, int group) {
    const int64_t Mp = (M + kPBN - 1) / kPBN * kPBN;
    // the decode path's counter area stays untouched at the front (shared workspaces)
    return kCounterBytes + align256p((size_t)M * K * 2) + align256p((size_t)(K / group) * Mp * 4);
}

namespace {
template <int GS>
int launch_prefill_gs(const uint16_t* X, const float* xscale, int64_t M, int64_t K, const uint32_t* qweight,
                      const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                      cudaStream_t stream) {
    static PerContext<int> attr;  // the attribute belongs to a context
    if (!attr.get([]() -> int {
            return cudaFuncSetAttribute(prefill_kernel<GS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kPSmem) == cudaSuccess;
        }))
        return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    char* ws = reinterpret_cast<char*>(workspace) + kCounterBytes;
    uint16_t* Xp = reinterpret_cast<uint16_t*>(ws);
    float* xsT = reinterpret_cast<float*>(ws + align256p((size_t)M * K * 2));
    CUtensorMap tx, tq;
    if (!prefill_tmap(0, Xp, M, K, &tx) || !prefill_tmap(1, qweight, N, K / 8, &tq)) return W4A16_ERR_CUDA;

    const int G = (int)(K / GS);  // quantisation groups per row
    const int64_t units = M * (K / kGroup) * 16;
    int pgrid = (int)ceil_div(units, 256);
    if (pgrid > num_sms_current() * 16) pgrid = num_sms_current() * 16;
    const int Mp = (int)((M + kPBN - 1) / kPBN * kPBN);
    if (Mp > M && cudaMemsetAsync(xsT, 0, (size_t)G * Mp * 4, stream) != cudaSuccess) return W4A16_ERR_CUDA;
    prefill_prep_kernel<GS><<<pgrid, 256, 0, stream>>>(X, xscale, (int)M, (int)K, Mp, Xp, xsT);
    if (cudaGetLastError() != cudaSuccess) return W4A16_ERR_CUDA;

    PrefillArgs args;
    args.scales = scales;
    args.zeros = zeros;
    args.xsT = xsT;
    args.Y = Y;
    args.fault = fault;
    args.M = (int)M;
    args.N = (int)N;
    args.K = (int)K;
    args.G = G;
    args.Mp = Mp;
    args.m_tiles = (int)ceil_div(M, kPBN);
    args.n_tiles = (int)ceil_div(N, kPBM * kPCtas);
    const int tiles = args.m_tiles * args.n_tiles;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = kPSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = kPCtas;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 2;
    // persistent: one MMA unit (CTA or 2-CTA cluster) per resident slot, so that every unit runs
    // in the first wave (a cluster needs two free SMs of one GPC, which not every SM count allows)
    int mma_units = prefill_resident_units(cfg, prefill_kernel<GS>);
    if (mma_units <= 0) return W4A16_ERR_CUDA;
    if (mma_units > tiles) mma_units = tiles;
    args.tiles = tiles;
    args.units = mma_units;
    cfg.gridDim = dim3((unsigned)(mma_units * kPCtas));
    return cudaLaunchKernelEx(&cfg, prefill_kernel<GS>, tx, tq, args) == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}
}  // namespace

int launch_prefill(const uint16_t* X, const float* xscale, int64_t M, int64_t K, int group, const uint32_t* qweight,
                   const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                   cudaStream_t stream) {
    if (group == 64)
        return launch_prefill_gs<64>(X, xscale, M, K, qweight, scales, zeros, N, Y, workspace, stream);
    return launch_prefill_gs<128>(X, xscale, M, K, qweight, scales, zeros, N, Y, workspace, stream);
}

}  // namespace w4a16
