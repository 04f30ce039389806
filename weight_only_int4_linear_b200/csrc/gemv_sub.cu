// Integer GEMV for quantisation groups of 32 or 64 weights, one token per launch
// ("Quantization I: int8, int4, the basics", Concept: groups of 32-128 values;
// "Weight-Only Quantization and Mixed Precision", section 8).  The same unit
// (128 rows x 128 K of packed codes), ring, split-K protocol and A operand as the
// group-128 integer GEMV for one token in gemv.cu, whose constants it repeats;
// what differs is how the X operand keeps the sub-groups of a 128-K unit apart,
// the per-lane folds and the 4-unit metadata blocks (described at SubCfg).
#include "common.cuh"
#include "decode_units.cuh"
#include "sm100.cuh"

#include <mutex>

namespace w4a16 {
namespace {

// The one-token integer GEMV's geometry (gemv.cu).
constexpr int kRowsPerCta = 128;
constexpr int kCcWarps = 4;                          // compute warps
constexpr int kCcTmaWarp = kCcWarps;                 // warp 4
constexpr int kCcXWarp = kCcWarps + 1;               // warp 5
constexpr int kCcThreads = (kCcWarps + 2) * 32;
constexpr int kCcStages = 4;
constexpr int kCcCodeBytes = kRowsPerCta * kWordsPerGroup * 4;  // 8 KB, 64-byte swizzle
constexpr int kCcXOff = kCcCodeBytes;                // X digit rows after the codes
constexpr int kChunkMax = 4;                         // units per chunk (a metadata block holds 4 units)

struct SubArgs {
    const uint16_t* Xp;  // [K] BF16, this launch's token
    float* partial;      // [row_tiles][cpt][128]: one slot of sums per chunk
    int* counters;       // counters[0]: the chunk counter
    int* fault;
    int N, G;            // G = 128-K units per row (a multiple of 4)
    int U;               // units per chunk: 2 or 4 (4 for groups of 32)
    int cpt, chunks;     // chunks per row tile, chunks in all
};

// This lane's four BF16 values of 128-K unit g: lane 2w + h holds values 4h..4h+3 of word w.
__device__ __forceinline__ uint2 load_group_x(const uint16_t* __restrict__ X, int g, int lane) {
    return __ldg(reinterpret_cast<const uint2*>(X + (int64_t)g * kGroup + lane * 4));
}

// mma.sync m16n8k32, A 16 x 32 unsigned bytes, B 32 x 8 signed bytes, D (+)= int32.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Tensor maps keyed by base pointer and shape: packed codes (box = one 128-K unit x 128 rows,
// 64-byte swizzle) and the metadata blocks (box = kMetaGroups groups x 128 rows).
struct SubTmap {
    const void* ptr;
    int64_t rows, cols;
    int kind;
    CUtensorMap map;
};
std::mutex g_sub_mu;
SubTmap g_sub_maps[64];
int g_sub_next = 0;

bool sub_tmap(int kind, const void* ptr, int64_t rows, int64_t cols, int box_groups, CUtensorMap* out) {
    std::lock_guard<std::mutex> lk(g_sub_mu);
    for (auto& e : g_sub_maps)
        if (e.ptr == ptr && e.rows == rows && e.cols == cols && e.kind == kind) {
            *out = e.map;
            return true;
        }
    SubTmap& e = g_sub_maps[g_sub_next];
    bool ok;
    if (kind == 0)  // codes: uint32 [rows = N][cols = K/8]
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT32, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 4, kWordsPerGroup, kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_64B);
    else if (kind == 1)  // scales: bf16 [rows = N][cols = K/GS]
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 2, (uint32_t)box_groups, kRowsPerCta);
    else  // zeros: int32 [rows = N][cols = K/GS]
        ok = encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_INT32, ptr, (uint64_t)cols, (uint64_t)rows,
                            (uint64_t)cols * 4, (uint32_t)box_groups, kRowsPerCta);
    if (!ok) return false;
    e.ptr = ptr;
    e.rows = rows;
    e.cols = cols;
    e.kind = kind;
    g_sub_next = (g_sub_next + 1) % 64;
    *out = e.map;
    return true;
}

// A 128-K unit holds SUB = 128 / GS groups; the X operand keeps them
// apart: digit row p SUB + j holds digit plane p of x for the K positions of sub-group j and
// zero elsewhere, so D column p SUB + j is sum_{k in j} q_k d_p(x_k).  SUB = 2 fits the 8 MMA
// columns (6 rows); SUB = 4 takes a second MMA per K step for plane 2 (rows 8-11).  Lane
// tig = j folds sub-group j with its own scale and zero point; the row's total is the sum of
// the quad's lanes, added in a fixed order where the output is written.  Metadata comes per
// block of 4 units (4 SUB groups: 16-byte scale rows for GS = 64, 32-byte for GS = 32).
template <int GS>
struct SubCfg {
    static constexpr int kSub = 128 / GS;
    static constexpr int kRows = 3 * kSub;                       // digit rows
    static constexpr int kExt = kRows * 128;                     // 2^(E-21), then kSub integer sums
    static constexpr int kStageBytes = (kCcCodeBytes + kExt + 4 * (1 + kSub) + 511) / 512 * 512;
    static constexpr int kMetaGroups = 4 * kSub;                 // groups per metadata block (4 units)
    static constexpr int kScBytes = kRowsPerCta * kMetaGroups * 2;
    static constexpr int kMetaBytes = kRowsPerCta * kMetaGroups * 6;
    static constexpr int kMetaOff = kCcStages * kStageBytes;
    // chunks of 2 (GS = 64 only) or 4 units; a chunk's block overwrites the slot of the chunk kMetaSlots
    // chunks earlier, whose last unit is then (kMetaSlots - 1) Umin + 1 units back
    static constexpr int kUnitsMin = GS == 64 ? 2 : 4;
    static constexpr int kMetaSlots = GS == 64 ? 3 : 2;
    static constexpr size_t kSmem = (size_t)kMetaOff + kMetaSlots * kMetaBytes + 512;
    static constexpr int kMinBlocks = GS == 64 ? 4 : 3;
    static_assert((kMetaSlots - 1) * kUnitsMin + 1 >= kCcStages, "metadata slot reuse");
};

// One warp writes the digits of one 128-K unit for groups of GS (layout above).  Within a row,
// word w's eight digit bytes are stored in the order the codes come out of a packed word
// ((w & 0x0F0F0F0F) gives codes 0, 2, 4, 6, (w >> 4) & 0x0F0F0F0F codes 1, 3, 5, 7), so the
// byte of code k lines up with it in the MMA: the lane pair (w, h = 0/1) holding codes 4h..4h+3
// assembles [h0.c0, h0.c2, h1.c0, h1.c2] (h = 0) and [h0.c1, h0.c3, h1.c1, h1.c3] (h = 1).
template <int GS>
__device__ __forceinline__ void prep_unit_x8_sub(const uint2 v, unsigned char* dst, int lane) {
    using C = SubCfg<GS>;
    constexpr int kLanes = GS / 4;  // lanes per sub-group (lane l holds k = 4l .. 4l + 3)
    const uint32_t bits[4] = {v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16};
    uint32_t amax = max(max(bits[0] & 0x7FFFu, bits[1] & 0x7FFFu), max(bits[2] & 0x7FFFu, bits[3] & 0x7FFFu));
    amax = __reduce_max_sync(0xFFFFFFFFu, amax);
    const int ef = (int)(amax >> 7);
    const int E = ef == 0 ? -127 : ef - 127;
    const int kx = 21 - E;
    const int k1 = min(kx, 127);
    const float s1 = pow2f(k1), s2 = pow2f(kx - k1);
    int xi[4];
    uint32_t dg[3] = {0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xi[i] = __float2int_rn(__uint_as_float(bits[i] << 16) * s1 * s2);
        const int d0 = ((xi[i] + 128) & 255) - 128;
        const int t = (xi[i] - d0) >> 8;
        const int d1 = ((t + 128) & 255) - 128;
        const int d2 = (t - d1) >> 8;
        const int pos = (i & 1) ? 16 + 8 * (i >> 1) : 8 * (i >> 1);
        dg[0] |= (uint32_t)(d0 & 255) << pos;
        dg[1] |= (uint32_t)(d1 & 255) << pos;
        dg[2] |= (uint32_t)(d2 & 255) << pos;
    }
    const int h = lane & 1, w = lane >> 1, j = lane / kLanes;
#pragma unroll
    for (int p = 0; p < 3; ++p) {
        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, dg[p], 1);
        const uint32_t lo = h ? other : dg[p], hi = h ? dg[p] : other;
        const uint32_t out = h ? __byte_perm(lo, hi, 0x7632) : __byte_perm(lo, hi, 0x5410);
#pragma unroll
        for (int jj = 0; jj < C::kSub; ++jj)
            *reinterpret_cast<uint32_t*>(dst + (p * C::kSub + jj) * 128 + 8 * w + 4 * h) = jj == j ? out : 0u;
    }
    const unsigned seg = ((1u << kLanes) - 1u) << (lane & ~(kLanes - 1));
    const int sum = __reduce_add_sync(seg, (xi[0] + xi[1]) + (xi[2] + xi[3]));  // |sum| < 2^28
    float* ext = reinterpret_cast<float*>(dst + C::kExt);
    if ((lane & (kLanes - 1)) == 0) ext[1 + j] = (float)sum;
    if (lane == 0) ext[0] = pow2f(E - 21);
}

template <int GS>
__global__ void __launch_bounds__(kCcThreads, SubCfg<GS>::kMinBlocks) decode_sub_kernel(
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tsc,
    const __grid_constant__ CUtensorMap tze, const SubArgs a) {
    using C = SubCfg<GS>;
    constexpr int kSub = C::kSub;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kCcStages], empty[kCcStages], dready[kCcStages];
    __shared__ int4 s_desc[kCcStages];  // (row tile, unit, chunk slot, flags) of the unit in each stage
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((512u - (raw & 511u)) & 511u);
    unsigned char* meta = ring + C::kMetaOff;
    constexpr int kFirst = 1, kLast = 2, kEnd = 4, kSlotShift = 4;

    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    int* const next_chunk = a.counters;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kCcStages; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], kCcWarps);
            mbar_init(&dready[s], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kCcTmaWarp) {  // ------------------------------------------- TMA
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tsc);
            prefetch_tmap(&tze);
            int i = 0, nchunks = 0;
            bool ok = true;
            // the units of chunk c (a chunk lies inside one 4-unit metadata block, loaded with its first unit)
            auto issue_chunk = [&](int c) {
                const int tile = c / a.cpt, k = c - tile * a.cpt;
                const int mslot = nchunks++ % C::kMetaSlots;
                for (int u = 0; u < a.U; ++u, ++i) {
                    const int s = i % kCcStages;
                    if (i >= kCcStages && !mbar_wait(&empty[s], ((i / kCcStages) - 1) & 1, a.fault, 111)) {
                        ok = false;
                        return;
                    }
                    const int g = k * a.U + u;
                    s_desc[s] = make_int4(tile, g, k,
                                          (u == 0 ? kFirst : 0) | (u + 1 == a.U ? kLast : 0) | (mslot << kSlotShift));
                    mbar_arrive(&dready[s]);
                    unsigned char* st = ring + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], kCcCodeBytes + (u == 0 ? C::kMetaBytes : 0));
                    tma_load_2d(st, &tq, g * kWordsPerGroup, tile * kRowsPerCta, &full[s]);
                    if (u == 0) {
                        unsigned char* ms = meta + mslot * C::kMetaBytes;
                        const int g0 = (g & ~3) * kSub;
                        tma_load_2d(ms, &tsc, g0, tile * kRowsPerCta, &full[s]);
                        tma_load_2d(ms + C::kScBytes, &tze, g0, tile * kRowsPerCta, &full[s]);
                    }
                }
            };
            issue_chunk(b);  // gridDim.x <= chunks; the weights need nothing from the preceding kernel
            pdl_wait_primary();  // the chunk counter is this launch's once the preceding one has completed
            // a launch draws exactly `chunks` values: the CTA drawing the last one resets the counter
            int v = ok ? atomicAdd(next_chunk, 1) : 0;
            while (ok && (int)gridDim.x + v < a.chunks) {
                const int c = (int)gridDim.x + v;
                v = atomicAdd(next_chunk, 1);  // in flight while chunk c is issued
                issue_chunk(c);
            }
            if (ok && v == a.chunks - 1) *next_chunk = 0;
            for (int j = max(0, i - kCcStages); j < i; ++j)
                mbar_wait(&full[j % kCcStages], (j / kCcStages) & 1, a.fault, 112);
            if (ok) {  // the end of the unit stream, in the stage after the last unit
                const int s = i % kCcStages;
                if (i < kCcStages || mbar_wait(&empty[s], ((i / kCcStages) - 1) & 1, a.fault, 111)) {
                    s_desc[s] = make_int4(-1, 0, 0, kEnd);
                    mbar_arrive(&dready[s]);
                    mbar_arrive(&full[s]);
                }
            }
        }
        return;
    }

    if (warp == kCcXWarp) {  // ------------------------------------------ X warp
        pdl_wait_primary();
        uint2 xq[kChunkMax];  // the chunk's units, loaded together at its first unit
        for (int i = 0;; ++i) {
            const int s = i % kCcStages;
            if (!warp_wait(&dready[s], (i / kCcStages) & 1, a.fault, 114)) break;
            const int4 d = s_desc[s];
            if (!(d.w & kEnd)) {
                if (d.w & kFirst) {
#pragma unroll
                    for (int j = 0; j < kChunkMax; ++j)
                        if (j < a.U) xq[j] = load_group_x(a.Xp, d.y + j, lane);
                }
                const int u = d.y & (a.U - 1);
                uint2 v = xq[0];
#pragma unroll
                for (int j = 1; j < kChunkMax; ++j)
                    if (u == j) v = xq[j];
                prep_unit_x8_sub<GS>(v, ring + s * C::kStageBytes + kCcXOff, lane);  // the stage is free
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
            if (d.w & kEnd) break;
        }
        return;
    }

    // ---------------------------------------------------- compute warps 0-3
    const int g8 = lane >> 2, tig = lane & 3;
    const bool folder = tig < kSub;               // lane tig folds sub-group tig
    const int jsub = folder ? tig : 0;
    auto rrow = [&](int k) { return 32 * warp + 16 * (k >> 1) + g8 + 8 * (k & 1); };
    float y[4] = {0.f, 0.f, 0.f, 0.f};

    for (int i = 0;; ++i) {
        const int s = i % kCcStages;
        if (!warp_wait(&full[s], (i / kCcStages) & 1, a.fault, 113)) break;
        const int4 d = s_desc[s];
        if (d.w & kEnd) break;
        const int g = d.y;
        const unsigned char* st = ring + s * C::kStageBytes;
        uint4 cw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = rrow(k);
            cw[k] = *reinterpret_cast<const uint4*>(st + r * 64 + 16 * (tig ^ ((r >> 1) & 3)));
        }
        uint32_t bx[8], bz[8];  // digit rows g8 (planes 0-1, or all three for kSub = 2) and 8 + g8 (plane 2, kSub = 4)
        {
            const bool has = g8 < (C::kRows < 8 ? C::kRows : 8);
            const uint4* xp = reinterpret_cast<const uint4*>(st + kCcXOff + g8 * 128 + tig * 32);
            const uint4 u0 = has ? xp[0] : make_uint4(0, 0, 0, 0), u1 = has ? xp[1] : make_uint4(0, 0, 0, 0);
            bx[0] = u0.x; bx[1] = u0.y; bx[2] = u0.z; bx[3] = u0.w;
            bx[4] = u1.x; bx[5] = u1.y; bx[6] = u1.z; bx[7] = u1.w;
            if constexpr (kSub == 4) {
                const bool hz = g8 < C::kRows - 8;
                const uint4* zp = reinterpret_cast<const uint4*>(st + kCcXOff + (8 + g8) * 128 + tig * 32);
                const uint4 v0 = hz ? zp[0] : make_uint4(0, 0, 0, 0), v1 = hz ? zp[1] : make_uint4(0, 0, 0, 0);
                bz[0] = v0.x; bz[1] = v0.y; bz[2] = v0.z; bz[3] = v0.w;
                bz[4] = v1.x; bz[5] = v1.y; bz[6] = v1.z; bz[7] = v1.w;
            }
        }
        const float* ext = reinterpret_cast<const float*>(st + kCcXOff + C::kExt);
        const float xscale = ext[0], xsum = ext[1 + jsub];
        const unsigned char* ms = meta + ((d.w >> kSlotShift) & 3) * C::kMetaBytes;
        const int gi = (g & 3) * kSub + jsub;  // this lane's group inside the metadata block
        float sv[4], zv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = rrow(k);
            sv[k] = bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(ms + r * (C::kMetaGroups * 2) + 2 * gi));
            zv[k] = (float)*reinterpret_cast<const int32_t*>(ms + C::kScBytes + r * (C::kMetaGroups * 4) + 4 * gi);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
            const uint32_t w0[4] = {cw[2 * rb].x, cw[2 * rb].y, cw[2 * rb].z, cw[2 * rb].w};
            const uint32_t w1[4] = {cw[2 * rb + 1].x, cw[2 * rb + 1].y, cw[2 * rb + 1].z, cw[2 * rb + 1].w};
            int dd[4] = {0, 0, 0, 0}, e[4] = {0, 0, 0, 0};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t a0 = w0[j] & 0x0F0F0F0Fu, a1 = w1[j] & 0x0F0F0F0Fu;
                const uint32_t a2 = (w0[j] >> 4) & 0x0F0F0F0Fu, a3 = (w1[j] >> 4) & 0x0F0F0F0Fu;
                mma_u8s8(dd, a0, a1, a2, a3, bx[2 * j], bx[2 * j + 1]);
                if constexpr (kSub == 4) mma_u8s8(e, a0, a1, a2, a3, bz[2 * j], bz[2 * j + 1]);
            }
            // lane tig holds D columns 2 tig, 2 tig + 1 of rows g8 (d0, d1) and g8 + 8 (d2, d3); folder j
            // gathers column p kSub + j of every plane p (plane 2 of kSub = 4 from the second MMA)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                int P[3];
#pragma unroll
                for (int p = 0; p < 3; ++p) {
                    const bool second = kSub == 4 && p == 2;
                    const int col = (p * kSub + jsub) & 7;
                    const int src = (lane & ~3) | (col >> 1);
                    const int va = __shfl_sync(0xFFFFFFFFu, second ? e[2 * hh] : dd[2 * hh], src);
                    const int vb = __shfl_sync(0xFFFFFFFFu, second ? e[2 * hh + 1] : dd[2 * hh + 1], src);
                    P[p] = (col & 1) ? vb : va;
                }
                const float qx = fmaf((float)P[2], 65536.f, (float)(P[1] * 256 + P[0]));
                const int k = 2 * rb + hh;
                if (folder) y[k] = fmaf(sv[k] * fmaf(-zv[k], xsum, qx), xscale, y[k]);  // power of two last
            }
        }
        if (d.w & kLast) {  // the chunk's row sums (the quad's sub-groups, in a fixed order) into its slot
            float* part = a.partial + ((int64_t)d.x * a.cpt + d.z) * kRowsPerCta;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float tot = y[k] + __shfl_xor_sync(0xFFFFFFFFu, y[k], 1);
                if constexpr (kSub == 4) tot += __shfl_xor_sync(0xFFFFFFFFu, tot, 2);
                if (tig == 0) part[rrow(k)] = tot;
                y[k] = 0.f;
            }
        }
    }
}

template <int GS>
int occupancy_sub() {
    static PerContext<int> cache;  // the attribute and occupancy belong to a context
    return cache.get([]() -> int {
        if (cudaFuncSetAttribute(decode_sub_kernel<GS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SubCfg<GS>::kSmem) != cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, decode_sub_kernel<GS>, kCcThreads, SubCfg<GS>::kSmem) !=
                cudaSuccess ||
            o < 1)
            return 0;
        return o;
    });
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }


// Chunk deal and workspace of the small-group kernel (one token per launch).
DecodePlan plan_decode_sub(int64_t N, int64_t K, int group, int num_sms) {
    DecodePlan p{};
    const int64_t G = K / kGroup;  // 128-K units per row (a multiple of 4)
    p.cc_tokens = 1;
    p.nt = 1;
    p.row_tiles = (int)ceil_div(N, kRowsPerCta);
    int occ = group == 64 ? occupancy_sub<64>() : occupancy_sub<32>();
    if (occ < 1) occ = 1;
    const int64_t grid = (int64_t)occ * num_sms;
    // chunks of 4 units where every CTA streams 12 or more units, else of 2 (groups of 32: always 4)
    p.cc_units = (group == 32 || (int64_t)p.row_tiles * G >= 12 * grid) ? 4 : 2;
    p.cc_cpt = (int)(G / p.cc_units);
    p.cc_chunks = p.row_tiles * p.cc_cpt;
    p.grid = (int)(grid < p.cc_chunks ? grid : p.cc_chunks);
    p.ws_xp_bytes = 0;
    p.ws_xs_bytes = 0;
    p.ws_partial_bytes = align256((size_t)p.cc_chunks * kRowsPerCta * 4);
    p.ws_counter_bytes = kCounterBytes;  // counters[0] is the chunk counter
    return p;
}

template <int GS>
int launch_sub(const CUtensorMap& tq, const CUtensorMap& tsc, const CUtensorMap& tze, const SubArgs& args, int grid,
               cudaStream_t stream) {
    if (occupancy_sub<GS>() < 1) return W4A16_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kCcThreads);
    cfg.dynamicSmemBytes = SubCfg<GS>::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_sub_kernel<GS>, tq, tsc, tze, args) == cudaSuccess ? W4A16_OK
                                                                                               : W4A16_ERR_CUDA;
}

}  // namespace

size_t decode_sub_workspace_bytes(int64_t N, int64_t K, int group) {
    return plan_decode_sub(N, K, group, num_sms_current()).workspace_bytes();
}

int launch_decode_sub(const uint16_t* X, int64_t M, int64_t K, int group, const uint32_t* qweight,
                      const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                      cudaStream_t stream) {
    const DecodePlan plan = plan_decode_sub(N, K, group, num_sms_current());
    const int ng = (int)(K / group);
    CUtensorMap tq, tsc, tze;
    const int box = 4 * (128 / group);  // SubCfg<group>::kMetaGroups
    if (!sub_tmap(0, qweight, N, K / 8, 0, &tq) || !sub_tmap(1, scales, N, ng, box, &tsc) ||
        !sub_tmap(2, zeros, N, ng, box, &tze))
        return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    char* ws = reinterpret_cast<char*>(workspace);
    SubArgs args{};
    args.partial = reinterpret_cast<float*>(ws + plan.ws_counter_bytes);
    args.counters = reinterpret_cast<int*>(ws);
    args.fault = fault;
    args.N = (int)N;
    args.G = (int)(K / kGroup);
    args.U = plan.cc_units;
    args.cpt = plan.cc_cpt;
    args.chunks = plan.cc_chunks;
    for (int64_t m = 0; m < M; ++m) {  // one token per launch, then its chunk sums
        args.Xp = X + m * K;
        int st = group == 64 ? launch_sub<64>(tq, tsc, tze, args, plan.grid, stream)
                             : launch_sub<32>(tq, tsc, tze, args, plan.grid, stream);
        if (st != W4A16_OK) return st;
        st = launch_cc_reduce(args.partial, Y + m * N, N, plan.cc_cpt, plan.row_tiles, stream);
        if (st != W4A16_OK) return st;
    }
    return W4A16_OK;
}

}  // namespace w4a16
