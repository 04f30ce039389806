// W8A16 linear layer: INT8 weights with one BF16 scale per output row, BF16
// activations, FP32 accumulation ("Weight-Only Quantization and Mixed
// Precision", section 5: INT8 weights against 16-bit activations, half the
// weight bytes of BF16; section 8: INT8 needs no grouping).  Quantisation is
// symmetric per row: s_n = bf16(max_k |w[n][k]| / 127), q = clamp(rint(w / s_n),
// -127, 127), w_hat = q s_n.
//
// The product is the decode kernel of the INT4 layer with one-byte codes:
// persistent split-K over units of 128 rows x 128 K (16 KB of codes by TMA,
// 128-byte swizzle), X of each 128-K block written by an X warp as three
// signed base-256 digit planes of x_int = x 2^(21 - E), and the dot products
// as mma.sync m16n8k32 s8 x s8 (codes x digits), exact in int32:
//   sum_k q x  =  sum_blocks 2^(E - 21) (P0 + 256 P1 + 65536 P2),
// folded in FP32 once per block; the row scale multiplies the row's sum once,
// where the output is written.  Up to two tokens per launch (NT = 1, 2);
// larger M runs as consecutive launches of two tokens.
#include "common.cuh"
#include "decode_units.cuh"
#include "sm100.cuh"
#include "w8a16.h"

#include <mutex>


namespace w4a16 {
namespace {

constexpr int kW8Rows = 128;                     // weight rows per unit (and per row tile)
constexpr int kW8K = 128;                        // K per unit: one X digit block
constexpr int kW8Warps = 4;                      // compute warps, 32 rows each
constexpr int kW8TmaWarp = kW8Warps;             // warp 4
constexpr int kW8XWarp = kW8Warps + 1;           // warp 5
constexpr int kW8Threads = (kW8Warps + 2) * 32;
constexpr int kW8CodeBytes = kW8Rows * kW8K;     // 16 KB, 128-byte swizzle
constexpr int kW8XOff = kW8CodeBytes;            // X digit rows of the unit's block, after the codes
constexpr int kW8XAhead = 6;                     // X warp: loads in flight, in units
// Ring depth and CTAs per SM: one token, 3 stages x 4 CTAs; two tokens (more registers), 4 x 3.
// Either way 12 units of codes (192 KB) in flight per SM.
template <int NT>
__host__ __device__ constexpr int w8_stages() { return NT == 1 ? 3 : 4; }
template <int NT>
__host__ __device__ constexpr int w8_min_blocks() { return NT == 1 ? 4 : 3; }
template <int NT>
__host__ __device__ constexpr int w8_x_bytes() { return 3 * NT * 128 + 4 * NT; }  // digit rows + 2^(E-21) per token
template <int NT>
__host__ __device__ constexpr int w8_stage_bytes() { return (kW8CodeBytes + w8_x_bytes<NT>() + 1023) / 1024 * 1024; }
template <int NT>
__host__ __device__ constexpr size_t w8_smem() { return (size_t)w8_stages<NT>() * w8_stage_bytes<NT>() + 1024; }

struct W8Args {
    const uint16_t* X;       // [M][K] BF16, this launch's tokens
    const uint16_t* scales;  // [N] BF16
    uint16_t* Y;             // [M][N]
    float* partial;          // [row_tiles][max_slots][M][128]
    int* counters;           // [row_tiles]
    int* fault;
    int M, N, K, G;
    int units_base, units_rem;
    int max_slots;
};

// One warp writes token m's digits of one 128-K block in natural K order: lane l holds x at
// k = 4l .. 4l + 3, digit plane p of x_k is byte k of row p NT + m; the block's 2^(E - 21)
// follows the 3 NT rows.
template <int NT>
__device__ __forceinline__ void w8_prep_block(const uint2 v, unsigned char* dst, int lane, int m) {
    const uint32_t bits[4] = {v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16};
    uint32_t amax = max(max(bits[0] & 0x7FFFu, bits[1] & 0x7FFFu), max(bits[2] & 0x7FFFu, bits[3] & 0x7FFFu));
    amax = __reduce_max_sync(0xFFFFFFFFu, amax);
    const int ef = (int)(amax >> 7);
    const int E = ef == 0 ? -127 : ef - 127;  // every |x| of the block is below 2^(E + 1)
    const int kx = 21 - E;                    // in [-106, 148]
    const int k1 = min(kx, 127);
    const float s1 = pow2f(k1), s2 = pow2f(kx - k1);  // exact scalings, |x * 2^kx| < 2^22
    uint32_t dg[3] = {0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int xi = __float2int_rn(__uint_as_float(bits[i] << 16) * s1 * s2);
        const int d0 = ((xi + 128) & 255) - 128;
        const int t = (xi - d0) >> 8;
        const int d1 = ((t + 128) & 255) - 128;
        const int d2 = (t - d1) >> 8;
        dg[0] |= (uint32_t)(d0 & 255) << (8 * i);
        dg[1] |= (uint32_t)(d1 & 255) << (8 * i);
        dg[2] |= (uint32_t)(d2 & 255) << (8 * i);
    }
#pragma unroll
    for (int p = 0; p < 3; ++p) *reinterpret_cast<uint32_t*>(dst + (p * NT + m) * 128 + 4 * lane) = dg[p];
    if (lane == 0) reinterpret_cast<float*>(dst + 3 * NT * 128)[m] = pow2f(E - 21);
}

// mma.sync m16n8k32, A 16 x 32 signed bytes (row-major fragments), B 32 x 8 signed bytes
// (column-major fragments), D (+)= int32: exact integer dot products.
__device__ __forceinline__ void mma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT>
__global__ void __launch_bounds__(kW8Threads, w8_min_blocks<NT>()) w8_decode_kernel(const __grid_constant__ CUtensorMap tq,
                                                                                    const W8Args a) {
    constexpr int kW8Stages = w8_stages<NT>();
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kW8Stages], empty[kW8Stages];
    __shared__ int s_last;
    const uint32_t raw = smem_u32(smem_raw);
    unsigned char* ring = smem_raw + ((1024u - (raw & 1023u)) & 1023u);  // 1024-aligned (128-byte swizzle)
    constexpr int kStageBytes = w8_stage_bytes<NT>();

    pdl_launch_dependents();  // the next call may start its weight loads as this grid's CTAs retire
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int64_t u_first = (int64_t)b * a.units_base + min(b, a.units_rem);
    const int nunits = a.units_base + (b < a.units_rem ? 1 : 0);
    const int G = a.G, N = a.N;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kW8Stages; ++s) {
            mbar_init(&full[s], 2);  // TMA thread (with the transaction bytes) + X warp
            mbar_init(&empty[s], kW8Warps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kW8TmaWarp) {  // ------------------------------------------- TMA
        if (lane == 0) {
            prefetch_tmap(&tq);
            // the weights need nothing from the preceding kernel: no PDL wait here
            UnitCursor cur(u_first, G);
            int issued = 0;
            for (int i = 0; i < nunits; ++i, cur.next(G)) {
                const int s = i % kW8Stages;
                if (i >= kW8Stages && !mbar_wait(&empty[s], ((i / kW8Stages) - 1) & 1, a.fault, 101)) break;
                mbar_arrive_expect_tx(&full[s], kW8CodeBytes);
                tma_load_2d(ring + s * kStageBytes, &tq, cur.g * kW8K, cur.tile * kW8Rows, &full[s]);
                ++issued;
            }
            // no copy may still be in flight when the CTA exits
            for (int i = max(0, issued - kW8Stages); i < issued; ++i)
                mbar_wait(&full[i % kW8Stages], (i / kW8Stages) & 1, a.fault, 102);
        }
        return;
    }

    if (warp == kW8XWarp) {  // ------------------------------------------ X warp
        pdl_wait_primary();  // X may come from the preceding kernel
        // loads run kW8XAhead units ahead of the preparation, so L2 latency is paid once, not per unit
        uint2 q[kW8XAhead][NT];
        UnitCursor cl(u_first, G);
#pragma unroll
        for (int j = 0; j < kW8XAhead; ++j, cl.next(G))
#pragma unroll
            for (int m = 0; m < NT; ++m)
                q[j][m] = j < nunits && m < a.M
                              ? __ldg(reinterpret_cast<const uint2*>(a.X + (int64_t)m * a.K + (int64_t)cl.g * kW8K + 4 * lane))
                              : make_uint2(0, 0);
        for (int i = 0; i < nunits; ++i, cl.next(G)) {
            uint2 v[NT];
#pragma unroll
            for (int m = 0; m < NT; ++m) {
                v[m] = q[0][m];
#pragma unroll
                for (int j = 0; j + 1 < kW8XAhead; ++j) q[j][m] = q[j + 1][m];
                q[kW8XAhead - 1][m] =
                    i + kW8XAhead < nunits && m < a.M
                        ? __ldg(reinterpret_cast<const uint2*>(a.X + (int64_t)m * a.K + (int64_t)cl.g * kW8K + 4 * lane))
                        : make_uint2(0, 0);
            }
            const int s = i % kW8Stages;
            if (i >= kW8Stages && !warp_wait(&empty[s], ((i / kW8Stages) - 1) & 1, a.fault, 103)) break;
#pragma unroll
            for (int m = 0; m < NT; ++m) w8_prep_block<NT>(v[m], ring + s * kStageBytes + kW8XOff, lane, m);
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
        }
        return;
    }

    // ---------------------------------------------------- compute warps 0-3
    const int t = threadIdx.x;
    // Warp w takes rows 32 w .. 32 w + 31 as two 16-row MMA blocks.  Lane (g8, tig) = (lane / 4,
    // lane % 4) holds, per block, rows g8 and g8 + 8, bytes 32 tig .. 32 tig + 31 of each (words
    // 0-3 and 4-7).  MMA j takes words j (A columns 4 tig ..) and 4 + j (A columns 16 + 4 tig ..)
    // of every lane, so its K = 32 values are k = 32 tig + 4 j + {0..3} and 32 tig + 16 + 4 j +
    // {0..3} over the lanes; the B fragments are the same words of digit row n = g8.  After a
    // unit, D column n = p NT + m of a row is sum_k q_k d_p(x_k) of token m.
    const int g8 = lane >> 2, tig = lane & 3;
    const int mt = tig < NT ? tig : NT - 1;  // the token this lane folds (lanes tig < NT)
    const bool owner = tig < NT && tig < a.M;
    auto rrow = [&](int k) { return 32 * warp + 16 * (k >> 1) + g8 + 8 * (k & 1); };
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    int cur_tile = -1;
    bool aborted = false;

    // the row scale enters every block's fold (s P, then the power of two), so that no partial sum
    // leaves the FP32 range unless the result does; rows past N fold with s = 0
    float sn[4] = {0.f, 0.f, 0.f, 0.f};
    auto load_row_scales = [&](int tile) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int n = tile * kW8Rows + rrow(k);
            sn[k] = n < N ? bf16_bits_to_float(a.scales[n]) : 0.f;
        }
    };
    auto flush = [&](int tile) {
        const int first = cta_of_unit((int64_t)tile * G, a.units_base, a.units_rem);
        const int last = cta_of_unit((int64_t)tile * G + G - 1, a.units_base, a.units_rem);
        if (first == last) {
            if (owner) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int n = tile * kW8Rows + rrow(k);
                    if (n < N) a.Y[(int64_t)mt * N + n] = float_to_bf16_bits(y[k]);
                }
            }
        } else {
            const int slot = b - first, nseg = last - first + 1;
            float* part = a.partial + ((int64_t)tile * a.max_slots + slot) * a.M * kW8Rows;
            if (owner) {
#pragma unroll
                for (int k = 0; k < 4; ++k) part[mt * kW8Rows + rrow(k)] = y[k];
            }
            named_barrier_sync(1, kW8Warps * 32);
            if (t == 0) s_last = (arrive_acq_rel_gpu(&a.counters[tile]) == nseg - 1);
            named_barrier_sync(1, kW8Warps * 32);
            if (s_last) {
                const int rows = min(kW8Rows, N - tile * kW8Rows);
                const float* pb = a.partial + (int64_t)tile * a.max_slots * a.M * kW8Rows;
#pragma unroll
                for (int m = 0; m < NT; ++m) {
                    if (m >= a.M) break;
                    for (int rl = t; rl < rows; rl += kW8Warps * 32) {
                        const float sum = sum_slots(pb + (int64_t)m * kW8Rows + rl, (int64_t)a.M * kW8Rows, nseg);
                        const int n = tile * kW8Rows + rl;
                        a.Y[(int64_t)m * N + n] = float_to_bf16_bits(sum);
                    }
                }
                if (t == 0) a.counters[tile] = 0;
            }
            named_barrier_sync(1, kW8Warps * 32);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) y[k] = 0.f;
    };

    UnitCursor uc(u_first, G);
    for (int i = 0; i < nunits; ++i, uc.next(G)) {
        const int tile = uc.tile;
        if (tile != cur_tile) {
            if (cur_tile >= 0) flush(cur_tile);
            cur_tile = tile;
            load_row_scales(tile);
        }
        if (aborted) continue;
        const int s = i % kW8Stages;
        if (!warp_wait(&full[s], (i / kW8Stages) & 1, a.fault, 104)) {
            aborted = true;
            continue;
        }
        const unsigned char* st = ring + s * kStageBytes;
        // codes: chunks 2 tig and 2 tig + 1 of each row, 128-byte swizzle (chunk c of row r at c ^ (r & 7))
        uint4 cw[4][2];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = rrow(k);
#pragma unroll
            for (int c = 0; c < 2; ++c)
                cw[k][c] = *reinterpret_cast<const uint4*>(st + r * 128 + 16 * ((2 * tig + c) ^ (r & 7)));
        }
        uint32_t bx[8];
        if (g8 < 3 * NT) {
            const uint4* xp = reinterpret_cast<const uint4*>(st + kW8XOff + g8 * 128 + tig * 32);
            const uint4 u0 = xp[0], u1 = xp[1];
            bx[0] = u0.x; bx[1] = u0.y; bx[2] = u0.z; bx[3] = u0.w;
            bx[4] = u1.x; bx[5] = u1.y; bx[6] = u1.z; bx[7] = u1.w;
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) bx[j] = 0u;
        }
        const float xscale = reinterpret_cast<const float*>(st + kW8XOff + 3 * NT * 128)[mt];
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
            const uint32_t w0[8] = {cw[2 * rb][0].x, cw[2 * rb][0].y, cw[2 * rb][0].z, cw[2 * rb][0].w,
                                    cw[2 * rb][1].x, cw[2 * rb][1].y, cw[2 * rb][1].z, cw[2 * rb][1].w};
            const uint32_t w1[8] = {cw[2 * rb + 1][0].x, cw[2 * rb + 1][0].y, cw[2 * rb + 1][0].z,
                                    cw[2 * rb + 1][0].w, cw[2 * rb + 1][1].x, cw[2 * rb + 1][1].y,
                                    cw[2 * rb + 1][1].z, cw[2 * rb + 1][1].w};
            int d[4] = {0, 0, 0, 0};
#pragma unroll
            for (int j = 0; j < 4; ++j) mma_s8s8(d, w0[j], w1[j], w0[4 + j], w1[4 + j], bx[j], bx[4 + j]);
            // lane tig holds columns 2 tig, 2 tig + 1 of rows g8 (d0, d1) and g8 + 8 (d2, d3)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                int P0, P1, P2;
                if constexpr (NT == 1) {  // planes 0, 1 at lane tig 0, plane 2 at lane tig 1
                    P0 = d[2 * h];
                    P1 = d[2 * h + 1];
                    P2 = __shfl_sync(0xFFFFFFFFu, d[2 * h], lane | 1);
                } else {  // column p NT + m: token 0 planes at (0,0), (1,0), (2,0); token 1 at (0,1), (1,1), (2,1)
                    const int own = tig == 0 ? d[2 * h] : d[2 * h + 1];
                    const int x = __shfl_xor_sync(0xFFFFFFFFu, tig == 0 ? d[2 * h + 1] : d[2 * h], 1);
                    const int t0 = __shfl_sync(0xFFFFFFFFu, d[2 * h], (lane & ~3) | 2);
                    const int t1 = __shfl_sync(0xFFFFFFFFu, d[2 * h + 1], (lane & ~3) | 2);
                    P0 = tig == 0 ? own : x;
                    P1 = tig == 0 ? x : own;
                    P2 = tig == 0 ? t0 : t1;
                }
                // |P| <= 128 * 127 * 128 < 2^21: 256 P1 + P0 is exact in int32, the rest FP32
                const float qx = fmaf((float)P2, 65536.f, (float)(P1 * 256 + P0));
                y[2 * rb + h] = fmaf(sn[2 * rb + h] * qx, xscale, y[2 * rb + h]);
            }
        }
    }
    if (cur_tile >= 0) flush(cur_tile);
}

template <int NT>
int w8_occupancy() {
    static PerContext<int> cache;  // the attribute and occupancy belong to a context
    return cache.get([]() -> int {
        if (cudaFuncSetAttribute(w8_decode_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)w8_smem<NT>()) != cudaSuccess)
            return 0;
        int o = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, w8_decode_kernel<NT>, kW8Threads, w8_smem<NT>()) !=
                cudaSuccess ||
            o < 1)
            return 0;
        return o;
    });
}

struct W8Plan {
    int row_tiles, grid, units_base, units_rem, max_slots;
    size_t ws_counter_bytes, ws_partial_bytes;
};

size_t align256w(size_t x) { return (x + 255) / 256 * 256; }

W8Plan plan_w8(int64_t M, int64_t N, int64_t K, int num_sms) {
    W8Plan p{};
    const int64_t G = K / kW8K;
    const int Mc = (int)(M < 2 ? M : 2);
    p.row_tiles = (int)ceil_div(N, kW8Rows);
    const int64_t units = (int64_t)p.row_tiles * G;
    int occ = Mc == 1 ? w8_occupancy<1>() : w8_occupancy<2>();
    if (occ < 1) occ = 1;
    int64_t grid = (int64_t)occ * num_sms;
    if (grid > units) grid = units;
    p.grid = (int)grid;
    p.units_base = (int)(units / grid);
    p.units_rem = (int)(units % grid);
    p.max_slots = (int)((G - 1) / p.units_base + 2);
    p.ws_partial_bytes = align256w((size_t)p.row_tiles * p.max_slots * Mc * kW8Rows * 4);
    p.ws_counter_bytes =
        align256w((size_t)(p.row_tiles > kSharedCounterTiles ? p.row_tiles : kSharedCounterTiles) * 4);
    return p;
}

// Tensor maps of INT8 weight matrices keyed by base pointer and shape.
struct W8Tmap {
    const void* ptr;
    int64_t rows, cols;
    CUtensorMap map;
};
std::mutex g_w8_mu;
W8Tmap g_w8_maps[32];
int g_w8_next = 0;

bool w8_tmap(const int8_t* q, int64_t N, int64_t K, CUtensorMap* out) {
    std::lock_guard<std::mutex> lk(g_w8_mu);
    for (auto& e : g_w8_maps)
        if (e.ptr == q && e.rows == N && e.cols == K) {
            *out = e.map;
            return true;
        }
    W8Tmap& e = g_w8_maps[g_w8_next];
    // int8 [rows = N][cols = K], box = 128 K x 128 rows, 128-byte swizzle
    if (!encode_tmap_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)N, (uint64_t)K, kW8K, kW8Rows,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    e.ptr = q;
    e.rows = N;
    e.cols = K;
    g_w8_next = (g_w8_next + 1) % 32;
    *out = e.map;
    return true;
}

template <int NT>
int launch_w8_nt(const CUtensorMap& tq, const W8Args& args, int grid, cudaStream_t stream) {
    if (w8_occupancy<NT>() < 1) return W4A16_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kW8Threads);
    cfg.dynamicSmemBytes = w8_smem<NT>();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w8_decode_kernel<NT>, tq, args) == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

// One CTA per row: max |w| (FP32 compares), the BF16 scale and the codes, every decision in
// binary64 as the scheme's definition states.
__global__ void __launch_bounds__(256) w8_quantize_kernel(const float* __restrict__ W, int64_t K,
                                                          int8_t* __restrict__ q, uint16_t* __restrict__ scales,
                                                          int32_t* status) {
    __shared__ float s_max[8];
    __shared__ int s_bad[8];
    const int64_t n = blockIdx.x;
    const float* w = W + n * K;
    float m = 0.f;
    int bad = 0;
    for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
        const float v = w[k];
        if (!isfinite(v)) bad = 1;
        else m = fmaxf(m, fabsf(v));
    }
    m = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m)));  // m >= 0: bit order = value order
    bad = __any_sync(0xFFFFFFFFu, bad);
    if ((threadIdx.x & 31) == 0) {
        s_max[threadIdx.x >> 5] = m;
        s_bad[threadIdx.x >> 5] = bad;
    }
    __syncthreads();
    m = 0.f;
    bad = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
        m = fmaxf(m, s_max[i]);
        bad |= s_bad[i];
    }
    if (bad) {
        if (threadIdx.x == 0) {
            atomicCAS(status, 0, (int)W4A16_ERR_NONFINITE);
            scales[n] = 0;
        }
        for (int64_t k = threadIdx.x; k < K; k += blockDim.x) q[n * K + k] = 0;
        return;
    }
    uint16_t sb = double_to_bf16_bits(__ddiv_rn((double)m, 127.0));
    if ((sb & 0x7FFFu) == 0) {
        sb = double_to_bf16_bits((double)m);
        if ((sb & 0x7FFFu) == 0) sb = 0x3F80u;  // 1.0
    }
    const double s = (double)bf16_bits_to_float(sb);
    for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
        const double t = fmin(fmax(rint(__ddiv_rn((double)w[k], s)), -127.0), 127.0);
        q[n * K + k] = (int8_t)(int)t;
    }
    if (threadIdx.x == 0) scales[n] = sb;
}

// W_hat = q s rounded to BF16 (q s is exact in FP32: a 7-bit integer times an 8-bit significand).
__global__ void w8_dequant_kernel(const int8_t* __restrict__ q, const uint16_t* __restrict__ scales, int64_t N,
                                  int64_t K, uint16_t* __restrict__ out) {
    const int64_t total = N * K;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = float_to_bf16_bits((float)q[i] * bf16_bits_to_float(scales[i / K]));
}

}  // namespace

size_t w8_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    const W8Plan p = plan_w8(M, N, K, num_sms_current());
    return p.ws_counter_bytes + p.ws_partial_bytes;
}

int launch_w8(const uint16_t* X, int64_t M, int64_t K, const int8_t* q, const uint16_t* scales, int64_t N,
              uint16_t* Y, void* workspace, cudaStream_t stream) {
    const W8Plan plan = plan_w8(M, N, K, num_sms_current());
    CUtensorMap tq;
    if (!w8_tmap(q, N, K, &tq)) return W4A16_ERR_CUDA;
    int* fault = fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    char* ws = reinterpret_cast<char*>(workspace);
    W8Args args;
    args.scales = scales;
    args.partial = reinterpret_cast<float*>(ws + plan.ws_counter_bytes);
    args.counters = reinterpret_cast<int*>(ws);
    args.fault = fault;
    args.N = (int)N;
    args.K = (int)K;
    args.G = (int)(K / kW8K);
    args.units_base = plan.units_base;
    args.units_rem = plan.units_rem;
    args.max_slots = plan.max_slots;
    for (int64_t m0 = 0; m0 < M; m0 += 2) {
        const int Mc = (int)((M - m0) < 2 ? (M - m0) : 2);
        args.X = X + m0 * K;
        args.Y = Y + m0 * N;
        args.M = Mc;
        // a one-token tail of an even plan reuses its unit deal; partial slots are sized for two tokens
        const int st = Mc == 1 ? launch_w8_nt<1>(tq, args, plan.grid, stream) : launch_w8_nt<2>(tq, args, plan.grid, stream);
        if (st != W4A16_OK) return st;
    }
    return W4A16_OK;
}

int launch_w8_quantize(const float* W, int64_t N, int64_t K, int8_t* q, uint16_t* scales, int32_t* status,
                       cudaStream_t stream) {
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), stream) != cudaSuccess) return W4A16_ERR_CUDA;
    w8_quantize_kernel<<<(unsigned)N, 256, 0, stream>>>(W, K, q, scales, status);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

int launch_w8_dequant(const int8_t* q, const uint16_t* scales, int64_t N, int64_t K, uint16_t* out,
                      cudaStream_t stream) {
    int64_t blocks = ceil_div(N * K, 256);
    if (blocks > (int64_t)num_sms_current() * 32) blocks = (int64_t)num_sms_current() * 32;
    w8_dequant_kernel<<<(unsigned)blocks, 256, 0, stream>>>(q, scales, N, K, out);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

}  // namespace w4a16
