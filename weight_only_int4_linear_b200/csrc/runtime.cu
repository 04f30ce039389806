// Host-side runtime helpers: tensor-map encoding through the driver entry
// point (no link-time dependency on libcuda), and the per-device fault word
// that bounded device waits report to.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace w4a16 {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void resolve_encode() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
        cudaGetLastError();
}

__device__ int g_fault;  // bounded-wait fault word: 0 = none, else the site that gave up
PerContext<int*> g_fault_addr;

typedef CUresult (*PFN_ctx_get_current)(CUcontext*);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long*);
PFN_ctx_get_current g_ctx_current = nullptr;
PFN_ctx_get_id g_ctx_id = nullptr;
std::once_flag g_ctx_once;

void resolve_ctx() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_current = reinterpret_cast<PFN_ctx_get_current>(fn);
    else
        cudaGetLastError();
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_id = reinterpret_cast<PFN_ctx_get_id>(fn);
    else
        cudaGetLastError();
}
}  // namespace

uint64_t context_key() {
    std::call_once(g_ctx_once, resolve_ctx);
    if (!g_ctx_current || !g_ctx_id) return 0;
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return (uint64_t)id + 1;  // context IDs are unique over the process; 0 stays "none"
}

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    std::call_once(g_encode_once, resolve_encode);
    if (!g_encode) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {
struct TmapKey {
    const void* base;
    uint64_t inner, outer, row_bytes;
    uint32_t box_inner, box_outer;
    int dtype, swizzle;
    bool operator==(const TmapKey& o) const {
        return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
               box_inner == o.box_inner && box_outer == o.box_outer && dtype == o.dtype && swizzle == o.swizzle;
    }
};
constexpr int kTmapSlots = 256;
TmapKey g_tkeys[kTmapSlots];
CUtensorMap g_tmaps[kTmapSlots];
int g_tnext = 0, g_tused = 0;
std::mutex g_tmu;
}  // namespace

bool tmap_2d_cached(CUtensorMap* out, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    const TmapKey key{base, inner, outer, row_bytes, box_inner, box_outer, (int)dtype, (int)swizzle};
    std::lock_guard<std::mutex> lk(g_tmu);
    for (int i = 0; i < g_tused; ++i)
        if (g_tkeys[i] == key) {
            *out = g_tmaps[i];
            return true;
        }
    CUtensorMap m;
    if (!encode_tmap_2d(&m, dtype, base, inner, outer, row_bytes, box_inner, box_outer, swizzle)) return false;
    g_tkeys[g_tnext] = key;
    g_tmaps[g_tnext] = m;
    g_tnext = (g_tnext + 1) % kTmapSlots;
    if (g_tused < kTmapSlots) ++g_tused;
    *out = m;
    return true;
}

int* fault_word() {
    return g_fault_addr.get([]() -> int* {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fault) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return static_cast<int*>(p);
    });
}

}  // namespace w4a16

namespace w4a16 {
namespace {
// One CTA waits on a phase of an mbarrier that nothing will complete (no copy, no MMA and no other
// thread is ever attached to it), with the caller's limit: the bounded wait runs out, records
// kSelftestSite and the kernel returns, as every pipeline wait of the library does on a timeout.
__global__ void __launch_bounds__(32) selftest_wait_kernel(long long limit, int* fault) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, fault, W4A16_SELFTEST_SITE, limit);
}
}  // namespace
}  // namespace w4a16

extern "C" W4A16_API int w4a16_selftest_wait(int64_t limit_cycles, void* stream) {
    if (limit_cycles < 1 || limit_cycles > W4A16_SELFTEST_MAX_CYCLES) return W4A16_ERR_ARG;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
        cudaGetLastError();
        return W4A16_ERR_DEVICE;
    }
    int* fault = w4a16::fault_word();
    if (!fault) return W4A16_ERR_CUDA;
    w4a16::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((long long)limit_cycles, fault);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

extern "C" W4A16_API int w4a16_device_fault(void) {
    int* p = w4a16::fault_word();
    if (!p) return -1;
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
    if (v != 0) cudaMemset(p, 0, sizeof(int));
    return v;
}
