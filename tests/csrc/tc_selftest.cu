// Single-CTA tcgen05 GEMM used by the tests to check the operand views of the
// tensor-core forward kernel: D[M,N] = (a_neg ? -1 : 1) * A[M,K] * B[K,N] with
// fp16 operands staged in 128-byte-swizzled row tiles and fp32 accumulation
// in TMEM.  Test infrastructure; not part of the library.
#include <cuda_fp16.h>
#include <stdint.h>

#include "tc_common.cuh"

using namespace gdelta::tc;

struct SelftestParams {
    const float *A, *B;
    float *D;
    int M, N, K;
    int a_mn, b_mn, a_neg;
    int RA, a_row0, RB, b_row0;
    int *err;
    int d_lane;          // M = 64 only: lane offset of the accumulator (0 or 16)
};

__global__ void __launch_bounds__(128) tc_selftest_kernel(SelftestParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int colsA = p.a_mn ? p.M : p.K, colsB = p.b_mn ? p.N : p.K;
    const int bytesA = p.RA * 128 * ((colsA + 63) / 64), bytesB = p.RB * 128 * ((colsB + 63) / 64);
    uint8_t *tA = base, *tB = base + bytesA;
    uint64_t *mbar = (uint64_t *)(tB + bytesB);
    uint32_t *slot = (uint32_t *)(mbar + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int i = tid; i < (bytesA + bytesB) / 4; i += 128) ((uint32_t *)base)[i] = 0u;
    __syncthreads();
    for (int e = tid; e < p.M * p.K; e += 128) {
        const int m = e / p.K, k = e % p.K;
        const int r = p.a_row0 + (p.a_mn ? k : m), c = p.a_mn ? m : k;
        *(__half *)(tA + tile_off(p.RA, r, c)) = __float2half_rn(p.A[e]);
    }
    for (int e = tid; e < p.K * p.N; e += 128) {
        const int k = e / p.N, n = e % p.N;
        const int r = p.b_row0 + (p.b_mn ? k : n), c = p.b_mn ? n : k;
        *(__half *)(tB + tile_off(p.RB, r, c)) = __float2half_rn(p.B[e]);
    }
    fence_proxy_async();
    if (warp == 0) {
        tmem_alloc(smem_u32(slot), 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(smem_u32(mbar), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t taddr = *slot;
    if (tid == 0) {
        const uint32_t id = idesc_f16(p.M, p.N, p.a_mn, p.b_mn, p.a_neg);
        const uint32_t a0 = smem_u32(tA), b0 = smem_u32(tB);
        for (int ks = 0; ks < p.K / 16; ++ks) {
            const uint64_t ad = p.a_mn ? desc_mnmajor(a0, p.RA, p.a_row0, ks) : desc_kmajor(a0, p.RA, p.a_row0, ks);
            const uint64_t bd = p.b_mn ? desc_mnmajor(b0, p.RB, p.b_row0, ks) : desc_kmajor(b0, p.RB, p.b_row0, ks);
            mma_f16(taddr + ((uint32_t)p.d_lane << 16), ad, bd, id, ks > 0);
        }
        mma_commit(smem_u32(mbar));
    }
    const bool ok = mbar_wait(smem_u32(mbar), 0);
    if (!ok && tid == 0) atomicExch(p.err, 1);
    fence_after_sync();
    if (ok) {
        for (int c = 0; c < p.N; c += 32) {
            float v[32];
            tmem_ld32(taddr + ((uint32_t)(32 * warp) << 16) + (uint32_t)c, v);
            int row = -1;
            if (p.M == 128) row = 32 * warp + lane;
            else if (lane >= p.d_lane && lane < p.d_lane + 16) row = 16 * warp + lane - p.d_lane;
            if (row >= 0)
                for (int i = 0; i < 32 && c + i < p.N; ++i) p.D[row * p.N + c + i] = v[i];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(taddr, 256);
}

extern "C" int tc_selftest(const float *A, const float *B, float *D, int M, int N, int K, int a_mn, int b_mn,
                           int a_neg, int RA, int a_row0, int RB, int b_row0, int d_lane, int *err, void *stream) {
    SelftestParams p{A, B, D, M, N, K, a_mn, b_mn, a_neg, RA, a_row0, RB, b_row0, err, d_lane};
    if (d_lane != 0 && !(M == 64 && d_lane == 16)) return 2;
    const int colsA = a_mn ? M : K, colsB = b_mn ? N : K;
    // bounds of every access, checked on the host before the launch
    if ((M != 64 && M != 128) || N % 32 || N < 32 || N > 256 || K % 16 || K < 16) return 2;
    if (a_row0 % 8 || b_row0 % 8 || colsA % 64 || colsB % 64) return 2;
    if (a_row0 + (a_mn ? K : M) > RA || b_row0 + (b_mn ? K : N) > RB) return 2;
    const size_t smem = 1024 + (size_t)RA * 128 * (colsA / 64) + (size_t)RB * 128 * (colsB / 64) + 64;
    if (smem > 227 * 1024) return 2;
    cudaFuncSetAttribute(tc_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    tc_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? 0 : 1;
}
