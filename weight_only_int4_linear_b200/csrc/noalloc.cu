// w4a16_linear_noalloc: the decode-path linear layer with its scratch memory
// in a fixed, file-scope device array instead of a caller-provided workspace.
//
// Who needs it: callers that must not allocate device memory once they are
// running -- a serving loop that reserves all of HBM at start-up, a host
// framework whose own allocator owns the device, or code that cannot call
// cudaMalloc from where it calls us -- can use this entry point without first
// sizing and allocating a workspace.
//
// The price: every process that loads the library holds kNoAllocScratchBytes
// of device memory on each GPU it touches, from module load until exit, and
// all calls on a device share that one buffer (see include/w4a16.h).
#include <mutex>

#include "common.cuh"

namespace w4a16 {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;  // 16 MiB

// Device-side scratch: X preparation, split-K partial sums and arrival counters.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_addr[kMaxDev];  // device address of g_noalloc_scratch, per device
std::mutex g_scratch_mu;

// Set-up, once per device, with that device current: the name
// g_noalloc_scratch is only a host-side stand-in, so the device address must
// be queried before a kernel may be given it.
void* scratch_address(int* status) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        cudaGetLastError();
        *status = W4A16_ERR_DEVICE;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t rc = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (rc != cudaSuccess || !p) {
            cudaGetLastError();
            *status = W4A16_ERR_CUDA;
            return nullptr;
        }
        g_scratch_addr[dev] = p;
    }
    *status = W4A16_OK;
    return g_scratch_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The current device must be sm_100; returns its SM count, or 0.
int device_sms() {
    int dev = 0, major = 0, minor = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return (major == 10 && minor == 0) ? sms : 0;
}

}  // namespace
}  // namespace w4a16

using namespace w4a16;

extern "C" size_t w4a16_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" int w4a16_linear_noalloc(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight,
                                    const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y,
                                    void* stream) {
    if (!X || !qweight || !scales || !zeros || !Y) return W4A16_ERR_ARG;
    if (M < 1 || N < 1 || K < 1) return W4A16_ERR_ARG;
    if (K % kGroup != 0) return W4A16_ERR_SHAPE;
    constexpr int64_t kMaxDim = (int64_t)1 << 30;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return W4A16_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(Y))
        return W4A16_ERR_ALIGN;
    const int sms = device_sms();
    if (sms == 0) return W4A16_ERR_DEVICE;
    const DecodePlan plan = plan_decode(M, N, K, sms);
    // a problem that needs more scratch than the built-in buffer holds is refused
    if (plan.workspace_bytes() > kNoAllocScratchBytes) return W4A16_ERR_WORKSPACE;
    int st = W4A16_OK;
    void* scratch = scratch_address(&st);
    if (!scratch) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // the buffer keeps the previous call's contents: the arrival counters must start at zero
    // counters lead the layout; only this call's row tiles need clearing
    if (cudaMemsetAsync(scratch, 0, (size_t)plan.row_tiles * 4, s) != cudaSuccess) return W4A16_ERR_CUDA;
    return launch_decode(X, nullptr, M, K, qweight, scales, zeros, N, Y, scratch, plan, s);
}
