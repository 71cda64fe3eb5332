// Five-gate low-rank projection (Muir review §2.3, the fused prologue of the
// mixer): the decay f, erase b, output g, write w and query-gain q gates of a
// layer share one down-projection of the layer input x (width R = the sum of
// the gates' ranks, 64 + 64 + 128 + 128 + 128 = 512 in the review's main
// model); each gate has its own up-projection back to the model width d and a
// per-channel bias, which give its logits.  The logits are activated into the
// form the mixer reads: log alpha = log sigmoid(f) (fp32), b = 2 sigmoid,
// g = sigmoid, w = sigmoid, z = the q logit (the mixer applies 2 sigmoid).
//
// Two launches of one persistent tcgen05 GEMM kernel (bf16 operands, fp32
// accumulation in TMEM):
//   down:  c = x[N, d] w_down[d, R], kept as two bf16 parts c = hi + lo
//          (codes[:, 0:R] = hi, codes[:, R:2R] = lo)
//   up:    gate i:  act_i((hi + lo)[:, R_i] w_up[R_i, :] + bias_i)   (grouped: K = 2 r_i)
// The codes are the A operand of the second product and the tensor core takes
// 16-bit operands; one bf16 part alone would round them to 8 bits, which the
// log-decay's sensitivity to its logit shows (about 4 % of its rms on the
// workload), while the two parts carry about 16 bits.
// A CTA runs one SM: warp 0 stages A and B tiles with TMA into a ring of
// stages (128-byte swizzle, the layout the MMA descriptors read), warp 1 issues
// the MMAs (M = 128 tokens, N = 256 columns, K = 64 per stage) into one of two
// TMEM accumulators, warps 2-9 drain the other accumulator meanwhile: two warps
// per 32-lane TMEM quadrant, one per half of the tile's columns.  The down
// launch stores the code halves directly; the up launch adds the bias, applies
// the activation and writes the gates through shared memory with TMA stores
// (one instruction per 4 KB box instead of 16-byte stores to 32 rows).
#include <cuda.h>
#include <cstring>
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace gdelta {

namespace {

constexpr int kPM = 128;                          // tokens per tile
constexpr int kPN = 256;                          // output columns per tile
constexpr int kPK = 64;                           // contraction per stage (128 bytes of bf16)
constexpr int kPATile = kPM * kPK * 2;            // 16 KiB
constexpr int kPBTile = kPK * kPN * 2;            // 32 KiB: 4 column blocks of 64 x 64
constexpr int kPStage = kPATile + kPBTile;
// warp 0 TMA, warp 1 MMA, then the epilogue warps: 8 for down (two per TMEM lane
// quadrant, 128 columns each), 16 for up (four per quadrant, 64 columns each:
// its epilogue, with the bias and the activations, is what bounds it)
template <bool kUp>
constexpr int epi_warps() { return kUp ? 16 : 8; }
template <bool kUp>
constexpr int proj_threads() { return 64 + 32 * epi_warps<kUp>(); }
constexpr int kPBox = 32 * 128;                   // one staged output box: 32 rows of 128 bytes
constexpr uint32_t kPDrainPolls = 1u << 22;

// Shared memory.  down: a 4-deep operand ring.  up: a 3-deep ring, two staged
// output boxes per epilogue warp (1024-byte aligned, as the 128-byte swizzle
// wants) and each epilogue warp's slice of the bias (128 floats).
template <bool kUp>
struct ProjSmem {
    static constexpr int kStages = kUp ? 3 : 4;
    static constexpr int STAGES = 0;
    static constexpr int OUT = kStages * kPStage;
    static constexpr int BIAS = OUT + (kUp ? epi_warps<kUp>() * kPBox : 0);        // one staged box per warp
    static constexpr int BAR = BIAS + (kUp ? epi_warps<kUp>() * 64 * 4 : 0);    // full, empty, acc_full[2], acc_empty[2], stall
    static constexpr int MISC = BAR + 8 * (2 * kStages + 5);              // TMEM slot, abort flag
    static constexpr int TOTAL = MISC + 64;
    static_assert(OUT % 1024 == 0, "staged boxes start on a 1024-byte boundary");
};

struct ProjParams {
    int M;                 // tokens
    int d;                 // model width
    int R;                 // total rank
    int jobs;              // output tiles
    int nn;                // column tiles per (token tile, gate)
    int rk[5], roff[5];    // ranks and their offsets in the code
    __nv_bfloat16 *codes;  // [M, 2R]: hi | lo (written by the down launch)
    const float *bias;     // [5, d]
    int *status;
    uint32_t spin;
    int stall;             // failure-path test: wait first on a barrier nothing completes
};

// The up launch's outputs as TMA store maps (128-byte swizzle): log alpha
// [M, d] fp32 in boxes of 32 columns x 32 rows, b, g, w, z [M, d] bf16 in boxes
// of 64 columns x 32 rows.
struct OutMaps {
    CUtensorMap la, gb, gg, gw, gz;
};

struct Job {
    int m0, n0, k0, nk, gate;
};

template <bool kUp>
__device__ __forceinline__ Job job_of(const ProjParams &p, int j) {
    Job t;
    if (!kUp) {
        t.m0 = kPM * (j / p.nn);
        t.n0 = kPN * (j % p.nn);
        t.k0 = 0;
        t.nk = p.d / kPK;
        t.gate = 0;
    } else {
        const int per_m = 5 * p.nn, r = j % per_m;
        t.m0 = kPM * (j / per_m);
        t.gate = r / p.nn;
        t.n0 = kPN * (r % p.nn);
        t.k0 = p.roff[t.gate];
        t.nk = 2 * (p.rk[t.gate] / kPK);          // the hi part's stages, then the lo part's
    }
    return t;
}

__device__ __forceinline__ float pex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float plg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float ptanh(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// sigmoid(v) = (1 + tanh(v / 2)) / 2: one special-function instruction (its
// relative error, about 2^-11, is below the bf16 rounding of the output)
__device__ __forceinline__ float psigmoid(float v) { return fmaf(0.5f, ptanh(0.5f * v), 0.5f); }
// log sigmoid(v) = -(max(-v, 0) + ln(1 + e^-|v|)), both logs through the
// special-function unit (base 2); for large |v| the sum 1 + e^-|v| rounds, an
// absolute error below 1e-7 in the fp32 log-decay
__device__ __forceinline__ float plogsigmoid(float v) {
    const float e = pex2(-fabsf(v) * 1.4426950408889634f);
    return -(fmaxf(-v, 0.f) + 0.6931471805599453f * plg2(1.f + e));
}

__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

}  // namespace

template <bool kUp>
__global__ void __launch_bounds__(proj_threads<kUp>(), 1)
    gate_proj_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ OutMaps om, const __grid_constant__ ProjParams p) {
    using L = ProjSmem<kUp>;
    constexpr int kPStages = L::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_full = tc::smem_u32(sm + L::BAR), s_empty = s_full + 8 * kPStages;
    const uint32_t s_accf = s_empty + 8 * kPStages, s_acce = s_accf + 16, s_stall = s_acce + 16;
    uint32_t *tslot = (uint32_t *)(sm + L::MISC);
    volatile int *abort_flag = (volatile int *)(sm + L::MISC + 8);
    if (!kUp) tc::grid_launch_dependents();       // the up launch may start once every down CTA has started

    if (tid == 0) {
        for (int s = 0; s < kPStages; ++s) {
            tc::mbar_init(s_full + 8 * s, 1);
            tc::mbar_init(s_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(s_accf + 8 * b, 1);
            tc::mbar_init(s_acce + 8 * b, epi_warps<kUp>());
        }
        tc::mbar_init(s_stall, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *abort_flag = 0;
        // failure-path test: a wait that nothing completes runs out before any copy or MMA
        if (p.stall && !tc::mbar_wait(s_stall, 0, p.spin)) *abort_flag = 1;
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(tslot), 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // the up launch is a programmatic dependent of the down launch: the codes are
    // read only after this (hardware) wait for the whole down grid
    if (kUp) tc::grid_dependency_wait();
    const uint32_t tmem = *tslot;
    bool timed_out = false;

    if (warp == 0 && lane == 0) {
        // ---- TMA producer
        uint32_t it = 0;
        for (int j = blockIdx.x; j < p.jobs && !timed_out; j += gridDim.x) {
            const Job t = job_of<kUp>(p, j);
            for (int kk = 0; kk < t.nk; ++kk, ++it) {
                const uint32_t s = it % kPStages, u = it / kPStages;
                if (*abort_flag || (u > 0 && !tc::mbar_wait(s_empty + 8 * s, (u - 1) & 1u, p.spin))) {
                    timed_out = true;
                    break;
                }
                // up: the second half of the stages reads the lo part of the codes
                // against the same rows of w_up
                const int half = kUp ? t.nk / 2 : t.nk;
                const int kr = kk % half, ka = t.k0 + kPK * kr + (kk >= half ? p.R : 0);
                const uint32_t a = tc::smem_u32(sm + L::STAGES + s * kPStage), b = a + kPATile;
                tc::mbar_arrive_expect_tx(s_full + 8 * s, kPStage);
                tc::tma_load_2d(a, &tmA, ka, t.m0, s_full + 8 * s);
#pragma unroll
                for (int c = 0; c < kPN / 64; ++c)
                    tc::tma_load_2d(b + c * (kPK * 128), &tmB, t.n0 + 64 * c, t.k0 + kPK * kr, s_full + 8 * s);
            }
        }
        if (timed_out) {
            *abort_flag = 1;
            // the loads already issued land before the CTA's shared memory goes away
            const uint32_t first = it > (uint32_t)kPStages ? it - kPStages : 0u;
            for (uint32_t i = first; i < it; ++i)
                tc::mbar_wait(s_full + 8 * (i % kPStages), (i / kPStages) & 1u, kPDrainPolls);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer
        const uint32_t idesc = tc::idesc_bf16(kPM, kPN, false, true);
        uint32_t it = 0, t = 0;
        bool issued = false;
        for (int j = blockIdx.x; j < p.jobs && !timed_out; j += gridDim.x, ++t) {
            const Job jb = job_of<kUp>(p, j);
            const uint32_t b = t & 1u, v = t >> 1;
            if (*abort_flag || (v > 0 && !tc::mbar_wait(s_acce + 8 * b, (v - 1) & 1u, p.spin))) {
                timed_out = true;
                break;
            }
            tc::fence_after_sync();
            const uint32_t acc = tmem + b * kPN;
            for (int kk = 0; kk < jb.nk; ++kk, ++it) {
                const uint32_t s = it % kPStages, u = it / kPStages;
                if (!tc::mbar_wait(s_full + 8 * s, u & 1u, p.spin)) {
                    timed_out = true;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t a = tc::smem_u32(sm + L::STAGES + s * kPStage), bt = a + kPATile;
#pragma unroll
                for (int ks = 0; ks < kPK / 16; ++ks)
                    tc::mma_f16(acc, tc::desc_kmajor_step(tc::desc_kmajor(a, kPM, 0, 0), kPM, ks), tc::desc_mnmajor_step(tc::desc_mnmajor(bt, kPK, 0, 0), ks), idesc,
                                kk > 0 || ks > 0);
                tc::mma_commit(s_empty + 8 * s);              // the stage is free once these MMAs are done
                issued = true;
            }
            if (timed_out) break;
            tc::mma_commit(s_accf + 8 * b);                   // the accumulator is final
        }
        if (timed_out) {
            *abort_flag = 1;
            // every MMA issued so far completes before TMEM is freed
            if (issued) {
                const uint32_t last = it - 1;
                tc::mbar_wait(s_empty + 8 * (last % kPStages), (last / kPStages) & 1u, kPDrainPolls);
            }
        }
    } else if (warp >= 2 && !kUp) {
        // ---- down epilogue: TMEM lanes 32 (warp % 4) .. +31 are the tile's rows;
        // warps 2-5 take columns 0-127 of the tile, warps 6-9 columns 128-255
        const int qd = warp & 3, row = 32 * qd + lane, cbase = warp < 6 ? 0 : kPN / 2;
        uint32_t t = 0;
        for (int j = blockIdx.x; j < p.jobs; j += gridDim.x, ++t) {
            const Job jb = job_of<kUp>(p, j);
            const uint32_t b = t & 1u, v = t >> 1;
            bool ok = true;
            if (lane == 0) ok = !*abort_flag && tc::mbar_wait(s_accf + 8 * b, v & 1u, p.spin);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                timed_out = true;
                break;
            }
            tc::fence_after_sync();
            const uint32_t acc = tmem + ((uint32_t)(32 * qd) << 16) + b * kPN;
            const int m = jb.m0 + row;
            for (int c = 0; c < kPN / 64; ++c) {
                float x[32];
                tc::tmem_ld32(acc + cbase + 32 * c, x);
                const int n = jb.n0 + cbase + 32 * c;
                if (m < p.M) {
                    // c = hi + lo: hi its bf16 rounding, lo the bf16 rounding of the rest
                    float lo[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) lo[i] = x[i] - __bfloat162float(__float2bfloat16_rn(x[i]));
                    uint4 *dh = reinterpret_cast<uint4 *>(p.codes + (size_t)m * 2 * p.R + n);
                    uint4 *dl = reinterpret_cast<uint4 *>(p.codes + (size_t)m * 2 * p.R + p.R + n);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        dh[q] = make_uint4(pack_bf2(x[8 * q], x[8 * q + 1]), pack_bf2(x[8 * q + 2], x[8 * q + 3]),
                                           pack_bf2(x[8 * q + 4], x[8 * q + 5]), pack_bf2(x[8 * q + 6], x[8 * q + 7]));
                        dl[q] = make_uint4(pack_bf2(lo[8 * q], lo[8 * q + 1]), pack_bf2(lo[8 * q + 2], lo[8 * q + 3]),
                                           pack_bf2(lo[8 * q + 4], lo[8 * q + 5]), pack_bf2(lo[8 * q + 6], lo[8 * q + 7]));
                    }
                }
            }
            // this warp's reads of the accumulator are complete: hand it back
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_local(s_acce + 8 * b);
        }
        if (timed_out && lane == 0) *abort_flag = 1;
    } else if (warp >= 2) {
        // ---- up epilogue.  The warp owns TMEM lanes 32 (warp % 4) .. +31 (the
        // tile's rows) and 64 of its columns (warps 2-5 the first quarter, 6-9 the
        // second, ...).  Activated values are staged in shared memory as boxes of
        // 32 rows x 128 bytes (32 fp32 or 64 bf16 columns), each row's 16-byte
        // chunks in the 128-byte-swizzled order (chunk q at q ^ (row % 8): the
        // eight rows a store phase covers hit eight different bank groups), and
        // lane 0 writes each box with one TMA store; the warp's one box buffer is
        // refilled once the previous store has read it.
        const int ew = warp - 2, qd = warp & 3, cbase = 64 * (ew >> 2);
        const uint32_t obuf = tc::smem_u32(sm + L::OUT + ew * kPBox);
        float *sbias = reinterpret_cast<float *>(sm + L::BIAS + ew * 64 * 4);
        const uint32_t rowoff = (uint32_t)lane * 128u, sw = (uint32_t)(lane & 7);
        uint32_t t = 0;
        for (int j = blockIdx.x; j < p.jobs; j += gridDim.x, ++t) {
            const Job jb = job_of<kUp>(p, j);
            const uint32_t b = t & 1u, v = t >> 1;
            // this warp's 64 bias values, fetched before the accumulator wait
            const float4 bv = lane < 16 ? __ldg(reinterpret_cast<const float4 *>(p.bias + (size_t)jb.gate * p.d +
                                                                                 jb.n0 + cbase) + lane)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            bool ok = true;
            if (lane == 0) ok = !*abort_flag && tc::mbar_wait(s_accf + 8 * b, v & 1u, p.spin);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                timed_out = true;
                break;
            }
            tc::fence_after_sync();
            const uint32_t acc = tmem + ((uint32_t)(32 * qd) << 16) + b * kPN + cbase;
            const int y = jb.m0 + 32 * qd;                 // the boxes' first row
            auto release = [&]() {
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive_local(s_acce + 8 * b);
            };
            if (y >= p.M) {                                // rows past the last token: nothing to store
                release();
                continue;
            }
            if (lane < 16) reinterpret_cast<float4 *>(sbias)[lane] = bv;
            __syncwarp();
            const CUtensorMap *map = jb.gate == 0 ? &om.la : jb.gate == 1 ? &om.gb : jb.gate == 2 ? &om.gg
                                     : jb.gate == 3 ? &om.gw : &om.gz;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float x[32];
                tc::tmem_ld32(acc + 32 * hh, x);
                if (hh == 1) release();
                const float4 *bb = reinterpret_cast<const float4 *>(sbias + 32 * hh);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 c4 = bb[q];
                    x[4 * q] += c4.x; x[4 * q + 1] += c4.y; x[4 * q + 2] += c4.z; x[4 * q + 3] += c4.w;
                }
                if (jb.gate == 0) {
                    // log alpha: a box of 32 fp32 columns per half
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = plogsigmoid(x[i]);
                    if (lane == 0) tc::bulk_wait_read_n<0>();
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        st_shared_v4(obuf + rowoff + (((uint32_t)q ^ sw) << 4), __float_as_uint(x[4 * q]),
                                     __float_as_uint(x[4 * q + 1]), __float_as_uint(x[4 * q + 2]),
                                     __float_as_uint(x[4 * q + 3]));
                    tc::fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) {
                        tc::tma_store_2d(map, obuf, jb.n0 + cbase + 32 * hh, y);
                        tc::bulk_commit();
                    }
                } else {
                    // a bf16 gate: both halves fill one box of 64 columns (chunks 4 hh .. 4 hh + 3)
                    if (jb.gate == 1) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) x[i] = 2.f * psigmoid(x[i]);
                    } else if (jb.gate != 4) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) x[i] = psigmoid(x[i]);
                    }
                    if (hh == 0) {
                        if (lane == 0) tc::bulk_wait_read_n<0>();
                        __syncwarp();
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_shared_v4(obuf + rowoff + (((uint32_t)(4 * hh + q) ^ sw) << 4), pack_bf2(x[8 * q], x[8 * q + 1]),
                                     pack_bf2(x[8 * q + 2], x[8 * q + 3]), pack_bf2(x[8 * q + 4], x[8 * q + 5]),
                                     pack_bf2(x[8 * q + 6], x[8 * q + 7]));
                    if (hh == 1) {
                        tc::fence_proxy_async();
                        __syncwarp();
                        if (lane == 0) {
                            tc::tma_store_2d(map, obuf, jb.n0 + cbase, y);
                            tc::bulk_commit();
                        }
                    }
                }
            }
        }
        // the boxes' stores are complete before the CTA's shared memory goes away
        if (lane == 0) tc::bulk_wait_all();
        if (timed_out && lane == 0) *abort_flag = 1;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && *abort_flag && p.status) atomicCAS(p.status, 0, (int)kDevTimeout);
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps (128-byte swizzle boxes: 64 x 128 for A, 64 x 64 for B)
// and the two launches.
// ---------------------------------------------------------------------------
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// A row-major [rows, cols] matrix of `esize`-byte elements, boxes of box_cols x
// box_rows with the 128-byte swizzle (box_cols * esize = 128).
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t esize, uint64_t rows, uint64_t cols,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapL2promotion l2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * esize};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An operand: bf16, boxes of 64 columns x box_rows rows.
bool operand_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, 64, box_rows,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// An output of the up launch: 32 rows of 128 bytes per box.
bool output_map(CUtensorMap *m, void *base, bool fp32, uint64_t rows, uint64_t cols) {
    return fp32 ? make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, cols, 32, 32,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE)
                : make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, 64, 32,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

}  // namespace

size_t gate_proj_workspace_bytes(int N, int R) { return ((size_t)N * 2 * R * 2 + 255) & ~(size_t)255; }

cudaError_t launch_gate_proj(const GateProjParams &gp, cudaStream_t stream) {
    static int sms[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!sms[dev]) {
        e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    const int smem_down = ProjSmem<false>::TOTAL + 1024, smem_up = ProjSmem<true>::TOTAL + 1024;
    e = cudaFuncSetAttribute(gate_proj_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_down);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gate_proj_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_up);
    if (e != cudaSuccess) return e;

    ProjParams p{};
    p.M = gp.N;
    p.d = gp.d;
    p.R = 0;
    for (int i = 0; i < 5; ++i) {
        p.rk[i] = gp.ranks[i];
        p.roff[i] = p.R;
        p.R += gp.ranks[i];
    }
    p.codes = (__nv_bfloat16 *)gp.codes;
    p.bias = gp.bias;
    p.status = gp.status;
    p.spin = gp.wait_limit;
    p.stall = gp.stall;
    const int mt = (gp.N + kPM - 1) / kPM;

    CUtensorMap ta, tb;
    OutMaps om;
    memset(&om, 0, sizeof(om));                      // the down launch stores directly
    // down: A = x [N, d], B = w_down [d, R]
    if (!operand_map(&ta, gp.x, (uint64_t)gp.N, (uint64_t)gp.d, kPM) ||
        !operand_map(&tb, gp.w_down, (uint64_t)gp.d, (uint64_t)p.R, kPK))
        return cudaErrorInvalidValue;
    p.nn = p.R / kPN;
    p.jobs = mt * p.nn;
    gate_proj_kernel<false><<<min(sms[dev], p.jobs), proj_threads<false>(), smem_down, stream>>>(ta, tb, om, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // up: A = codes [N, 2R] (hi | lo), B = w_up [R, d]; the five outputs
    const uint64_t N = (uint64_t)gp.N, d = (uint64_t)gp.d;
    if (!operand_map(&ta, gp.codes, N, (uint64_t)(2 * p.R), kPM) ||
        !operand_map(&tb, gp.w_up, (uint64_t)p.R, d, kPK) || !output_map(&om.la, gp.log_alpha, true, N, d) ||
        !output_map(&om.gb, gp.b, false, N, d) || !output_map(&om.gg, gp.g, false, N, d) ||
        !output_map(&om.gw, gp.w, false, N, d) || !output_map(&om.gz, gp.z, false, N, d))
        return cudaErrorInvalidValue;
    p.nn = gp.d / kPN;
    p.jobs = mt * 5 * p.nn;
    return tc::launch_dependent(gate_proj_kernel<true>, dim3(min(sms[dev], p.jobs)), dim3(proj_threads<true>()),
                                smem_up, stream, ta, tb, om, p);
}

}  // namespace gdelta
