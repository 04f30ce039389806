// C-ABI entry points of the w4a16 library: host-side validation, device
// checks and kernel dispatch.  No entry point allocates device memory or
// synchronises the host.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "w8a16.h"

namespace w4a16 {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_device_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 rejected
std::atomic<int> g_num_sms[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

int check_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return W4A16_ERR_DEVICE;
    }
    if (dev >= kMaxDevices) return W4A16_ERR_DEVICE;
    int state = g_device_ok[dev].load(std::memory_order_acquire);
    if (state == 0) {
        int major = 0, minor = 0, sms = 0;
        bool ok = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
                  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
                  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
        ok = ok && major == 10 && minor == 0;
        if (ok) g_num_sms[dev].store(sms, std::memory_order_relaxed);
        state = ok ? 1 : 2;
        g_device_ok[dev].store(state, std::memory_order_release);
    }
    return state == 1 ? W4A16_OK : W4A16_ERR_DEVICE;
}

namespace {
// Shape limits: indices inside the kernels are 32-bit for M, N, K and 64-bit
// for element offsets.
constexpr int64_t kMaxDim = (int64_t)1 << 30;

int check_shape(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || N < 1 || K < 1) return W4A16_ERR_ARG;
    if (K % kGroup != 0) return W4A16_ERR_SHAPE;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return W4A16_ERR_SHAPE;
    return W4A16_OK;
}
}  // namespace

int num_sms_current() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    const int s = g_num_sms[dev].load(std::memory_order_relaxed);
    return s > 0 ? s : 148;
}

}  // namespace w4a16

using namespace w4a16;

extern "C" {

const char* w4a16_status_string(int status) {
    switch (status) {
        case W4A16_OK: return "ok";
        case W4A16_ERR_ARG: return "invalid argument (null pointer, non-positive size or unknown option)";
        case W4A16_ERR_ALIGN: return "a base pointer is not 16-byte aligned";
        case W4A16_ERR_SHAPE: return "unsupported shape (K must be a multiple of 128; sizes up to 2^30)";
        case W4A16_ERR_DEVICE: return "no usable device: the current CUDA device must be sm_100 (B200)";
        case W4A16_ERR_WORKSPACE: return "workspace missing or smaller than w4a16_workspace_bytes()";
        case W4A16_ERR_CUDA: return "the CUDA runtime reported an error at launch";
        case W4A16_ERR_NONFINITE: return "a weight group holds NaN or Inf";
        case W4A16_ERR_ZERO_RANGE: return "a zero point does not fit in int32";
        default: return "unknown status";
    }
}

int w4a16_version(void) { return 100; }

static int quantize_pack_entry(const float* W, const float* col_scale, int64_t N, int64_t K, uint32_t* qweight,
                               uint16_t* scales, int32_t* zeros, int32_t* dev_status, bool symmetric, void* stream) {
    if (!W || !qweight || !scales || !zeros || !dev_status) return W4A16_ERR_ARG;
    int st = check_shape(1, N, K);
    if (st != W4A16_OK) return st;
    if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
        (col_scale && !aligned16(col_scale)) || (reinterpret_cast<uintptr_t>(dev_status) & 3u))
        return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    return launch_quantize_pack(W, col_scale, N, K, qweight, scales, zeros, dev_status, symmetric,
                                (cudaStream_t)stream);
}

int w4a16_quantize_pack(const float* W, int64_t N, int64_t K, uint32_t* qweight, uint16_t* scales, int32_t* zeros,
                        int32_t* dev_status, void* stream) {
    return quantize_pack_entry(W, nullptr, N, K, qweight, scales, zeros, dev_status, false, stream);
}

int w4a16_quantize_pack_sym(const float* W, int64_t N, int64_t K, uint32_t* qweight, uint16_t* scales,
                            int32_t* zeros, int32_t* dev_status, void* stream) {
    return quantize_pack_entry(W, nullptr, N, K, qweight, scales, zeros, dev_status, true, stream);
}

int w4a16_quantize_pack_awq(const float* W, const float* s, int64_t N, int64_t K, uint32_t* qweight,
                            uint16_t* scales, int32_t* zeros, int32_t* dev_status, void* stream) {
    if (!s) return W4A16_ERR_ARG;
    return quantize_pack_entry(W, s, N, K, qweight, scales, zeros, dev_status, false, stream);
}

size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (check_shape(M, N, K) != W4A16_OK) return 0;
    check_device();  // caches the SM count the plan depends on
    // enough for every kernel family (the decode need is independent of M beyond 32 tokens)
    const size_t dec = plan_decode(M, N, K, num_sms_current()).workspace_bytes();
    const size_t pre = prefill_workspace_bytes(M, K);
    return dec > pre ? dec : pre;
}

int w4a16_workspace_init(void* workspace, size_t bytes, void* stream) {
    if (bytes == 0) return W4A16_OK;
    if (!workspace) return W4A16_ERR_ARG;
    if (check_device() != W4A16_OK) return W4A16_ERR_DEVICE;
    return cudaMemsetAsync(workspace, 0, bytes, (cudaStream_t)stream) == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

static int linear_entry(const uint16_t* X, const float* xscale, int64_t M, int64_t K, const uint32_t* qweight,
                        const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                        size_t workspace_bytes, int path, void* stream) {
    if (!X || !qweight || !scales || !zeros || !Y) return W4A16_ERR_ARG;
    if (path < W4A16_PATH_AUTO || path > W4A16_PATH_PREFILL) return W4A16_ERR_ARG;
    int st = check_shape(M, N, K);
    if (st != W4A16_OK) return st;
    if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(Y) ||
        (xscale && !aligned16(xscale)))
        return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    const bool prefill = path == W4A16_PATH_PREFILL || (path == W4A16_PATH_AUTO && M >= kPrefillMinM);
    const DecodePlan plan = plan_decode(M, N, K, num_sms_current());
    const size_t need = prefill ? prefill_workspace_bytes(M, K) : plan.workspace_bytes();
    if (need > 0 && (!workspace || workspace_bytes < need)) return W4A16_ERR_WORKSPACE;
    if (need > 0 && !aligned16(workspace)) return W4A16_ERR_ALIGN;
    if (prefill)
        return launch_prefill(X, xscale, M, K, kGroup, qweight, scales, zeros, N, Y, workspace, (cudaStream_t)stream);
    return launch_decode(X, xscale, M, K, qweight, scales, zeros, N, Y, workspace, plan, (cudaStream_t)stream);
}

int w4a16_linear_path(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                      const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace, size_t workspace_bytes,
                      int path, void* stream) {
    return linear_entry(X, nullptr, M, K, qweight, scales, zeros, N, Y, workspace, workspace_bytes, path, stream);
}

int w4a16_linear_awq(const uint16_t* X, const float* inv_s, int64_t M, int64_t K, const uint32_t* qweight,
                     const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                     size_t workspace_bytes, int path, void* stream) {
    if (!inv_s) return W4A16_ERR_ARG;
    return linear_entry(X, inv_s, M, K, qweight, scales, zeros, N, Y, workspace, workspace_bytes, path, stream);
}

int w4a16_linear(const uint16_t* X, int64_t M, int64_t K, const uint32_t* qweight, const uint16_t* scales,
                 const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace, size_t workspace_bytes,
                 void* stream) {
    return w4a16_linear_path(X, M, K, qweight, scales, zeros, N, Y, workspace, workspace_bytes, W4A16_PATH_AUTO,
                             stream);
}

int w4a16_linear_host(const uint16_t* X_host, uint16_t* X_dev, int64_t M, int64_t K, const uint32_t* qweight,
                      const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y_dev, uint16_t* Y_host,
                      void* workspace, size_t workspace_bytes, void* stream) {
    if (!X_host || !Y_host || !X_dev || !Y_dev) return W4A16_ERR_ARG;
    int st = check_shape(M, N, K);
    if (st != W4A16_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // One token on the decode path: both transfers as part of the kernels' launch chain (the host buffers
    // accessed through their mapped device addresses), so that consecutive calls keep overlapping
    if (M == 1) {
        void *xh = nullptr, *yh = nullptr;
        const bool mapped = cudaHostGetDevicePointer(&xh, const_cast<uint16_t*>(X_host), 0) == cudaSuccess &&
                            cudaHostGetDevicePointer(&yh, Y_host, 0) == cudaSuccess && aligned16(xh);
        if (!mapped) cudaGetLastError();  // not mapped: the copy-engine transfers below
        if ((st = check_device()) != W4A16_OK) return st;
        const DecodePlan plan = plan_decode(M, N, K, num_sms_current());
        if (mapped && plan.cc_tokens) {
            if (!qweight || !scales || !zeros) return W4A16_ERR_ARG;
            if (!aligned16(X_dev) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
                !aligned16(Y_dev))
                return W4A16_ERR_ALIGN;
            const size_t need = plan.workspace_bytes();
            if (need > 0 && (!workspace || workspace_bytes < need)) return W4A16_ERR_WORKSPACE;
            if (need > 0 && !aligned16(workspace)) return W4A16_ERR_ALIGN;
            return launch_decode(X_dev, nullptr, M, K, qweight, scales, zeros, N, Y_dev, workspace, plan, s,
                                 static_cast<const uint16_t*>(xh), static_cast<uint16_t*>(yh));
        }
    }
    if (cudaMemcpyAsync(X_dev, X_host, (size_t)M * K * 2, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return W4A16_ERR_CUDA;
    st = w4a16_linear_path(X_dev, M, K, qweight, scales, zeros, N, Y_dev, workspace, workspace_bytes, W4A16_PATH_AUTO,
                           stream);
    if (st != W4A16_OK) return st;
    return cudaMemcpyAsync(Y_host, Y_dev, (size_t)M * N * 2, cudaMemcpyDeviceToHost, s) == cudaSuccess ? W4A16_OK
                                                                                                        : W4A16_ERR_CUDA;
}

int w4a16_unpack(const uint32_t* qweight, int64_t N, int64_t K, uint8_t* codes, void* stream) {
    if (!qweight || !codes) return W4A16_ERR_ARG;
    int st = check_shape(1, N, K);
    if (st != W4A16_OK) return st;
    if (!aligned16(qweight) || !aligned16(codes)) return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    return launch_unpack(qweight, N, K, codes, (cudaStream_t)stream);
}

int w4a16_dequant(const uint32_t* qweight, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                  uint16_t* W_hat, void* stream) {
    if (!qweight || !scales || !zeros || !W_hat) return W4A16_ERR_ARG;
    int st = check_shape(1, N, K);
    if (st != W4A16_OK) return st;
    if (!aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(W_hat)) return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    return launch_dequant(qweight, scales, zeros, N, K, W_hat, (cudaStream_t)stream);
}

int w4a16_dequant_codes(const uint8_t* codes, const uint16_t* scales, const int32_t* zeros, int64_t N, int64_t K,
                        uint16_t* W_hat, void* stream) {
    if (!codes || !scales || !zeros || !W_hat) return W4A16_ERR_ARG;
    int st = check_shape(1, N, K);
    if (st != W4A16_OK) return st;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(zeros) || !aligned16(W_hat)) return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    return launch_dequant_codes(codes, scales, zeros, N, K, W_hat, (cudaStream_t)stream);
}

int w4a16_renorm_rows(const uint16_t* y, int64_t M, int64_t N, uint16_t* out, void* stream) {
    if (!y || !out) return W4A16_ERR_ARG;
    if (M < 1 || N < 1) return W4A16_ERR_ARG;
    if (M > kMaxDim || N > kMaxDim) return W4A16_ERR_SHAPE;
    int st = check_device();
    if (st != W4A16_OK) return st;
    return launch_renorm(y, M, N, out, (cudaStream_t)stream);
}

int w4a16_quantize_pack_g(const float* W, int64_t N, int64_t K, int group, int symmetric, uint32_t* qweight,
                          uint16_t* scales, int32_t* zeros, int32_t* dev_status, void* stream) {
    if (group == 128) return quantize_pack_entry(W, nullptr, N, K, qweight, scales, zeros, dev_status, symmetric != 0,
                                                 stream);
    if (group != 32 && group != 64) return W4A16_ERR_ARG;
    if (!W || !qweight || !scales || !zeros || !dev_status) return W4A16_ERR_ARG;
    int st = check_shape(1, N, K);
    if (st != W4A16_OK) return st;
    if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
        (reinterpret_cast<uintptr_t>(dev_status) & 3u))
        return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    return launch_quantize_pack_small(W, N, K, group, symmetric != 0, qweight, scales, zeros, dev_status,
                                      (cudaStream_t)stream);
}

size_t w4a16_workspace_bytes_g(int64_t M, int64_t N, int64_t K, int group) {
    if (group == 128) return w4a16_workspace_bytes(M, N, K);
    if ((group != 32 && group != 64) || check_shape(M, N, K) != W4A16_OK || K % 512 != 0) return 0;
    check_device();
    // one token: the integer GEMV with per-sub-group digit rows; more: the BF16 tensor-core GEMV (its
    // scratch after the shared counter area, which it leaves untouched)
    if (M == 1) return decode_sub_workspace_bytes(N, K, group);
    if (group == 64 && M >= kPrefillMinM) return prefill_workspace_bytes(M, K, group);  // the GEMM
    return kCounterBytes + bf_workspace_bytes(M, N, K, group, num_sms_current());
}

int w4a16_linear_g(const uint16_t* X, int64_t M, int64_t K, int group, const uint32_t* qweight,
                   const uint16_t* scales, const int32_t* zeros, int64_t N, uint16_t* Y, void* workspace,
                   size_t workspace_bytes, void* stream) {
    if (group == 128)
        return linear_entry(X, nullptr, M, K, qweight, scales, zeros, N, Y, workspace, workspace_bytes,
                            W4A16_PATH_AUTO, stream);
    if (group != 32 && group != 64) return W4A16_ERR_ARG;
    if (!X || !qweight || !scales || !zeros || !Y) return W4A16_ERR_ARG;
    int st = check_shape(M, N, K);
    if (st != W4A16_OK) return st;
    if (K % 512 != 0) return W4A16_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(Y))
        return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    const size_t need = w4a16_workspace_bytes_g(M, N, K, group);
    if (!workspace || workspace_bytes < need) return W4A16_ERR_WORKSPACE;
    if (!aligned16(workspace)) return W4A16_ERR_ALIGN;
    if (M == 1) return launch_decode_sub(X, M, K, group, qweight, scales, zeros, N, Y, workspace, (cudaStream_t)stream);
    if (group == 64 && M >= kPrefillMinM)
        return launch_prefill(X, nullptr, M, K, group, qweight, scales, zeros, N, Y, workspace, (cudaStream_t)stream);
    return launch_decode_bf(X, nullptr, M, K, group, qweight, scales, zeros, N, Y,
                            reinterpret_cast<char*>(workspace) + kCounterBytes, (cudaStream_t)stream);
}

int w8a16_quantize(const float* W, int64_t N, int64_t K, int8_t* qweight, uint16_t* scales, int32_t* dev_status,
                   void* stream) {
    if (!W || !qweight || !scales || !dev_status) return W4A16_ERR_ARG;
    if (N < 1 || K < 1) return W4A16_ERR_ARG;
    if (N > kMaxDim || K > kMaxDim) return W4A16_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(dev_status) & 3u))
        return W4A16_ERR_ALIGN;
    int st = check_device();
    if (st != W4A16_OK) return st;
    return launch_w8_quantize(W, N, K, qweight, scales, dev_status, (cudaStream_t)stream);
}

int w8a16_dequant(const int8_t* qweight, const uint16_t* scales, int64_t N, int64_t K, uint16_t* W_hat,
                  void* stream) {
    if (!qweight || !scales || !W_hat) return W4A16_ERR_ARG;
    if (N < 1 || K < 1) return W4A16_ERR_ARG;
    if (N > kMaxDim || K > kMaxDim) return W4A16_ERR_SHAPE;
    if (!aligned16(qweight) || !aligned16(scales) || !aligned16(W_hat)) return W4A16_ERR_ALIGN;
    int st = check_device();
    if (st != W4A16_OK) return st;
    return launch_w8_dequant(qweight, scales, N, K, W_hat, (cudaStream_t)stream);
}

size_t w8a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (check_shape(M, N, K) != W4A16_OK) return 0;
    check_device();  // caches the SM count the plan depends on
    return w8_workspace_bytes(M, N, K);
}

int w8a16_linear(const uint16_t* X, int64_t M, int64_t K, const int8_t* qweight, const uint16_t* scales, int64_t N,
                 uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream) {
    if (!X || !qweight || !scales || !Y) return W4A16_ERR_ARG;
    int st = check_shape(M, N, K);
    if (st != W4A16_OK) return st;
    if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(Y)) return W4A16_ERR_ALIGN;
    if ((st = check_device()) != W4A16_OK) return st;
    const size_t need = w8_workspace_bytes(M, N, K);
    if (!workspace || workspace_bytes < need) return W4A16_ERR_WORKSPACE;
    if (!aligned16(workspace)) return W4A16_ERR_ALIGN;
    return launch_w8(X, M, K, qweight, scales, N, Y, workspace, (cudaStream_t)stream);
}

}  // extern "C"
