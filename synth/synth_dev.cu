// Device-side filler for the seeded synthetic weights: the same counter-based
// generator as synth.c (definition in synth_core.h), evaluated on the GPU so
// that large weight sets (tens of GB) need not cross PCIe.  Input generation
// only.  Build with -fmad=false so that no multiply-add is fused and the bits
// match the host generator.
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth_core.h"

__global__ void synth_fill_normal_kernel(uint64_t key, uint64_t offset, int64_t count, double sigma,
                                         float* __restrict__ out) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
        out[i] = __double2float_rn(sigma * syn_normal(key, offset + (uint64_t)i));
}

extern "C" int synth_dev_fill_normal_f32(uint64_t seed, uint64_t tag, uint64_t offset, int64_t count,
                                         double sigma, float* out, void* stream) {
    if (count < 0 || (count > 0 && out == nullptr)) return 1;
    if (count == 0) return 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 2;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 2;
    int64_t blocks = (count + 255) / 256;
    int64_t cap = (int64_t)sms * 16;
    if (blocks > cap) blocks = cap;
    synth_fill_normal_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(syn_key(seed, tag), offset,
                                                                                count, sigma, out);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
