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
constexpr int kMaxDev = 64;
int* g_fault_addr[kMaxDev];
std::mutex g_fault_mu;
}  // namespace

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

int* fault_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
    std::lock_guard<std::mutex> lk(g_fault_mu);
    if (!g_fault_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fault) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_fault_addr[dev] = static_cast<int*>(p);
    }
    return g_fault_addr[dev];
}

}  // namespace w4a16

extern "C" W4A16_API int w4a16_device_fault(void) {
    int* p = w4a16::fault_word();
    if (!p) return -1;
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
    if (v != 0) cudaMemset(p, 0, sizeof(int));
    return v;
}
