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

// S_out = A S_in + D per head: A [d_k, d_k], S_in / D / S_out [d_k, d_v], fp32.
// A block owns 16 rows of one head's S_out; a thread owns d_v / 16 adjacent
// columns of one row and walks k, reading a 16-row slab of A from shared
// memory and S_in rows from global (each row serves the block's 16 rows).
template <int DV>
__global__ void __launch_bounds__(256) state_affine_kernel(float *S_out, const float *__restrict__ A,
                                                           const float *__restrict__ S_in, const float *D, int dk) {
    constexpr int CPT = DV / 16;
    __shared__ float sA[16][128 + 1];
    const int head = blockIdx.x, r0 = 16 * blockIdx.y;
    const int tid = threadIdx.x, r = tid / 16, cg = tid % 16;
    const float *Ah = A + (size_t)head * dk * dk + (size_t)r0 * dk;
    for (int e = tid; e < 16 * dk; e += 256) sA[e / dk][e % dk] = Ah[e];
    __syncthreads();
    const size_t off = (size_t)head * dk * DV + (size_t)(r0 + r) * DV + cg * CPT;
    float acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; c += 4) {
        const float4 d = D ? *reinterpret_cast<const float4 *>(D + off + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        acc[c] = d.x; acc[c + 1] = d.y; acc[c + 2] = d.z; acc[c + 3] = d.w;
    }
    if (S_in) {
        const float *Sh = S_in + (size_t)head * dk * DV + cg * CPT;
        for (int k = 0; k < dk; ++k) {
            const float a = sA[r][k];
#pragma unroll
            for (int c = 0; c < CPT; c += 4) {
                const float4 s4 = __ldg(reinterpret_cast<const float4 *>(Sh + (size_t)k * DV + c));
                acc[c] = fmaf(a, s4.x, acc[c]);
                acc[c + 1] = fmaf(a, s4.y, acc[c + 1]);
                acc[c + 2] = fmaf(a, s4.z, acc[c + 2]);
                acc[c + 3] = fmaf(a, s4.w, acc[c + 3]);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < CPT; c += 4)
        *reinterpret_cast<float4 *>(S_out + off + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
}

cudaError_t launch_state_affine(float *S_out, const float *A, const float *S_in, const float *D, int BH, int dk,
                                int dv, cudaStream_t stream) {
    const dim3 grid((unsigned)BH, (unsigned)(dk / 16));
    if (dv == 128)
        state_affine_kernel<128><<<grid, 256, 0, stream>>>(S_out, A, S_in, D, dk);
    else
        state_affine_kernel<64><<<grid, 256, 0, stream>>>(S_out, A, S_in, D, dk);
    return cudaGetLastError();
}

}  // namespace gdelta
