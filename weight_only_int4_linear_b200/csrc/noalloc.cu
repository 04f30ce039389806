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
#include "common.cuh"

namespace w4a16 {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;  // 16 MiB

// Device-side scratch: X preparation, split-K partial sums and arrival counters.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

PerContext<void*> g_scratch_addr;  // device address of g_noalloc_scratch, per device and context

// Set-up, once per device (and again after a cudaDeviceReset), with that device current: the name
// g_noalloc_scratch is only a host-side stand-in, so the device address must be queried before a
// kernel may be given it.
void* scratch_address() {
    return g_scratch_addr.get([]() -> void* {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return p;
    });
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
    if (check_device() != W4A16_OK) return W4A16_ERR_DEVICE;
    // the same SM count the launch sizes its grids with
    const DecodePlan plan = plan_decode(M, N, K, num_sms_current());
    // a problem whose decode-path scratch exceeds the built-in buffer is refused
    if (plan.workspace_bytes() > kNoAllocScratchBytes) return W4A16_ERR_WORKSPACE;
    void* scratch = scratch_address();
    if (!scratch) return W4A16_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    // the buffer keeps the previous call's contents: the arrival counters must start at zero
    // counters lead the layout; only this call's row tiles need clearing
    if (cudaMemsetAsync(scratch, 0, (size_t)plan.row_tiles * 4, s) != cudaSuccess) return W4A16_ERR_CUDA;
    return launch_decode(X, nullptr, M, K, qweight, scales, zeros, N, Y, scratch, plan, s);
}
