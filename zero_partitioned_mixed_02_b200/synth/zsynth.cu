// Synthetic input generator: host and device entry points (see zsynth.h).
// Input infrastructure only; none of the optimizer's arithmetic lives here.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "zsynth.h"

extern "C" uint64_t zsynth_key(uint64_t seed, uint64_t stream, uint64_t step, uint64_t rank)
{
    return zs_mix(zs_mix(zs_mix(zs_mix(seed) ^ stream) ^ step) ^ rank);
}

extern "C" void zsynth_host_f32(float* out, int64_t n, int64_t index0, uint64_t key,
                                const zsynth_dist* d)
{
    for (int64_t k = 0; k < n; ++k) out[k] = zs_value(key, index0 + k, d);
}

extern "C" void zsynth_host_f32_at(float* out, const int64_t* idx, int64_t n, uint64_t key,
                                   const zsynth_dist* d)
{
    for (int64_t k = 0; k < n; ++k) out[k] = zs_value(key, idx[k], d);
}

namespace {

template <bool HALF>
__global__ void fill_kernel(void* out, int64_t n, int64_t index0, uint64_t key, zsynth_dist d)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
        const float x = zs_value(key, index0 + k, &d);
        if (HALF)
            static_cast<__half*>(out)[k] = __float2half_rn(x);
        else
            static_cast<float*>(out)[k] = x;
    }
}

int launch(bool half, void* out, int64_t n, int64_t index0, uint64_t key, const zsynth_dist* d,
           void* stream)
{
    if (n <= 0) return 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)sms * 8;
    if (blocks > cap) blocks = cap;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (half)
        fill_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(out, n, index0, key, *d);
    else
        fill_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(out, n, index0, key, *d);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

extern "C" int zsynth_fill_f16(uint16_t* out, int64_t n, int64_t index0, uint64_t key,
                               const zsynth_dist* d, void* stream)
{
    return launch(true, out, n, index0, key, d, stream);
}

extern "C" int zsynth_fill_f32(float* out, int64_t n, int64_t index0, uint64_t key,
                               const zsynth_dist* d, void* stream)
{
    return launch(false, out, n, index0, key, d, stream);
}
