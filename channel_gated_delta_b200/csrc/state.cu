// State initialisation: S <- 0 or S <- S_src, 128-bit grid-stride copy.
#include "common.cuh"

namespace gdelta {

__global__ void __launch_bounds__(256) state_init_kernel(float4 *__restrict__ S,
                                                         const float4 *__restrict__ src, size_t n4) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride)
        S[i] = src ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
}

cudaError_t launch_state_init(float *S, const float *src, size_t n, cudaStream_t stream) {
    if (n == 0 || S == src) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t n4 = n / 4;                       // n is a multiple of 64*64
    size_t blocks = (n4 + 255) / 256;
    const size_t cap = (size_t)sms * 8;
    if (blocks > cap) blocks = cap;
    state_init_kernel<<<(unsigned)blocks, 256, 0, stream>>>((float4 *)S, (const float4 *)src, n4);
    return cudaGetLastError();
}

}  // namespace gdelta
