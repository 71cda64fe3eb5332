// Tensor-core chunked forward (tcgen05, fp16 operands, fp32 accumulation in
// TMEM).  One CTA per (batch, head) walks the sequence chunk by chunk; the
// fp32 state lives in TMEM for the whole sequence.
//
// Notation (row-vector convention; one chunk of n <= 64 tokens, token t,
// key channel i; Lambda_t = cumulative log-decay inside the chunk, inclusive;
// k^ = b*k, v^ = w*v, q~ = q * gamma_stat * 2 sigmoid(z)):
//
//   c_i   = (Lambda_{0,i} + Lambda_{n-1,i}) / 2      per-channel pivot
//   Kp    = k  * e^{Lambda_t - c}     Kc  = k  * e^{c - Lambda_t}
//   Qp    = q~ * e^{Lambda_t - c}     K^c = k^ * e^{c - Lambda_t}
//
// so Kp_t . Kc_s = sum_i k_ti e^{Lambda_ti - Lambda_si} k_si exactly, with
// every factor inside e^{+-span/2}: the decay-relative products are plain
// matrix products and nothing is divided by a cumulative decay.  This is the
// boundary-pivot idea of the Muir review (§2.4) with the pivot at the middle
// of the chunk; when a chunk's decay span (max_i Lambda_{0,i} - Lambda_{n-1,i})
// exceeds kSpanMax the chunk is shortened (64 -> 32 -> ... -> 1 tokens, the
// rest padded with identity tokens) until the factors fit fp16.
//
// Per chunk (MMA shapes M x N x K):
//   P    = [Kp; Qp] [Kc; K^c]^T                      128x128x128 -> M, L, Aq, Bq
//   T^-1 = (I + L)^-1                                fp32, divide and conquer on CUDA cores
//   W'   = T^-1 Kp,  N = T^-1 M                      64x128x64, 64x64x64
//   S_c  = Diag(e^c) S                               (state operand, fp16)
//   [R; O] = [W'; Qp] S_c + [N; Aq] V^               128xDVx(128+64)
//   O   -= Bq R                                      (negated A)
//   X    = S_c + Kc^T V^ - K^c^T R                   accumulated in TMEM (fp32)
//   S_next = Diag(e^{Lambda_{n-1} - c}) X
// which is the unrolled recurrence S_t = Diag(alpha_t)S - k^_t^T(k_t Diag(alpha_t) S)
// + k_t^T v^_t, o_t = q~_t S_t of the Muir review §2.1 (R holds the erase
// projections r_t = k_t Diag(alpha_t) S_{t-1}).  y = g * O / rms(O).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace gdelta {

namespace {

constexpr int kC = 64;        // tokens per chunk
constexpr int kDK = 128;      // key channels
constexpr int kDV = 128;      // value channels of a head
constexpr float kSpanMax = 12.f;
constexpr int kThreads = 256;
constexpr int kLW = 68;       // row stride (floats) of the fp32 L / T^-1 matrix
constexpr int kYS = 36;       // row stride (floats) of the merge buffer
constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (PTX ex2.approx, flush-to-zero).  With
// log-decays pre-scaled by log2(e), e^x = 2^(x log2 e) costs one instruction.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2 sigmoid(z) = 2 / (1 + e^-z); the exponent is clamped so that the sum stays finite.
__device__ __forceinline__ float two_sigmoid_fast(float z) {
    return __fdividef(2.f, 1.f + ex2(fminf(-z * kLog2e, 126.f)));
}

// Warp reduce-scatter of 16 per-lane partial sums: afterwards lane l holds the
// sum over all 32 lanes of value 8 b4 + 4 b3 + 2 b2 + b1 (b_i = bit i of l),
// in 16 shuffles instead of the 80 of sixteen separate butterflies.
__device__ __forceinline__ float reduce_scatter16(const float (&v)[16], int lane) {
    float w8[8], w4[4], w2[2];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float keep = b4 ? v[8 + j] : v[j], send = b4 ? v[j] : v[8 + j];
        w8[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float keep = b3 ? w8[4 + j] : w8[j], send = b3 ? w8[j] : w8[4 + j];
        w4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float keep = b2 ? w4[2 + j] : w4[j], send = b2 ? w4[j] : w4[2 + j];
        w2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    float w1;
    {
        const float keep = b1 ? w2[1] : w2[0], send = b1 ? w2[0] : w2[1];
        w1 = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    return w1 + __shfl_xor_sync(0xffffffffu, w1, 1);
}

// shared-memory map (bytes); tiles are 1024-byte aligned
template <int DVC>
struct Smem {
    static constexpr int AP = 0;                          // [Kp | W' ; Qp]  128 x 128 fp16
    static constexpr int BP = AP + 128 * 256;             // [Kc ; K^c]      128 x 128
    static constexpr int TI = BP + 128 * 256;             // T^-1             64 x 64
    static constexpr int MM = TI + 64 * 128;              // M                64 x 64
    static constexpr int ANAB = MM + 64 * 128;            // [N ; Aq ; Bq]   192 x 64
    static constexpr int VH = ANAB + 192 * 128;           // V^               64 x DVC
    static constexpr int SC = VH + 64 * 2 * DVC;          // S_c             128 x DVC
    static constexpr int RR = SC + 128 * 2 * DVC;         // R                64 x DVC
    static constexpr int GS = RR + 64 * 2 * DVC;          // output gate g (bf16 [64][DVC])
    static constexpr int LW = GS + 64 * 2 * DVC;          // fp32 L, then T^-1   [64][kLW]
    static constexpr int YB = LW + 64 * kLW * 4;          // fp32 merge buffer  [32][kYS]
    static constexpr int WT = YB + 32 * kYS * 4;          // fp32 per-warp log-decay totals [8][128]
    static constexpr int PR = WT + 8 * 128 * 4;           // fp32 Lambda at the probe tokens [7][128]
    static constexpr int VEC = PR + 8 * 128 * 4;          // fp32 vectors
    static constexpr int nvec = 8 * 128;
    static constexpr int PART = VEC + nvec * 4;           // fp32 [64][2] RMS partial sums
    static constexpr int MISC = PART + 64 * 2 * 4;        // mbarrier, TMEM slot, flags
    static constexpr int TOTAL = MISC + 64;
};

// Per-window record written by the intra kernel: the chunk's operand tiles in
// the exact shared-memory byte layout the chain kernel uses, then the pivot
// vectors e^c and e^{Lambda_{n-1} - c} (fp32, 128 each).
constexpr int kWinAP = 0;                     // [W' ; Qp]       128 x 128 fp16
constexpr int kWinBP = kWinAP + 128 * 256;    // [Kc ; K^c]      128 x 128
constexpr int kWinANAB = kWinBP + 128 * 256;  // [N ; Aq ; Bq]   192 x 64
constexpr int kWinVH = kWinANAB + 192 * 128;  // V^               64 x 128
constexpr int kWinVEC = kWinVH + 64 * 256;    // e^c, e^{Lambda_{n-1} - c}
constexpr int kWinPad = 1024 - 2 * 128 * 4;   // padding to a 1 KB multiple
constexpr int kWinBytes = kWinVEC + 1024;

// TMEM columns
constexpr uint32_t kTmP = 0;       // P (128 x 128), later [R; O] (128 x DVC)
constexpr uint32_t kTmW = 128;     // W' (M=64, 128 columns)
constexpr uint32_t kTmN = 256;     // N  (M=64, 64 columns)
constexpr uint32_t kTmX = 384;     // state accumulator X (128 x DVC)

struct TcParams {
    int B, T, H;
    const __nv_bfloat16 *q, *k, *z, *b, *v, *w, *g;
    const float *la, *gs, *S_in;
    float *S_out;
    __nv_bfloat16 *y;
    float *o_raw;
    float eps;
    int *status;
    const uint8_t *ws;       // per-window chunk tiles from the intra kernel, or null
    const int *wflags;       // per-window flag: 0 = tiles valid, 1 = process here
    int NW;                  // windows of 64 tokens per head
};

__device__ __forceinline__ void bf16x8_to_f(const uint4 &u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float *f) {
    return make_uint4(tc::pack_half2(f[0], f[1]), tc::pack_half2(f[2], f[3]), tc::pack_half2(f[4], f[5]),
                      tc::pack_half2(f[6], f[7]));
}

__device__ __forceinline__ float maxabs(const float *f, int n) {
    float m = 0.f;
    for (int i = 0; i < n; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

// 32 columns of one accumulator row -> four 16-byte fp16 chunks of a row tile.
__device__ __forceinline__ void store_row32(uint8_t *tile, int R, int r, int col, const float (&v)[32]) {
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
        *(uint4 *)(tile + tc::tile_chunk_off(R, r, col / 8 + q4)) = pack8(v + 8 * q4);
}

// One merge level of the divide-and-conquer inverse, block size BS (pairs of
// BS x BS blocks along the diagonal of the 64 x 64 matrix in lw).
template <int BS>
__device__ __forceinline__ void merge_level(float *lw, float *yb, int tid) {
    constexpr int QPR = BS / 4, PER = BS * QPR, NTASK = (32 / BS) * PER;
    const int pr = tid / PER, rem = tid % PER, i = rem / QPR, j0 = 4 * (rem % QPR);
    const int oo = 2 * BS * pr;
    if (tid < NTASK) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *crow = lw + (oo + BS + i) * kLW + oo;
#pragma unroll
        for (int s = 0; s < BS; ++s) {
            const float c = crow[s];
            const float4 a = *reinterpret_cast<const float4 *>(lw + (oo + s) * kLW + oo + j0);
            acc.x += c * a.x; acc.y += c * a.y; acc.z += c * a.z; acc.w += c * a.w;
        }
        *reinterpret_cast<float4 *>(yb + (pr * BS + i) * kYS + j0) = acc;
    }
    __syncthreads();
    if (tid < NTASK) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *drow = lw + (oo + BS + i) * kLW + oo + BS;
#pragma unroll
        for (int s = 0; s < BS; ++s) {
            const float d = drow[s];
            const float4 y = *reinterpret_cast<const float4 *>(yb + (pr * BS + s) * kYS + j0);
            acc.x += d * y.x; acc.y += d * y.y; acc.z += d * y.z; acc.w += d * y.w;
        }
        *reinterpret_cast<float4 *>(lw + (oo + BS + i) * kLW + oo + j0) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    __syncthreads();
}

}  // namespace

template <int DVC>
__global__ void __launch_bounds__(kThreads, 1) gdn2_fwd_tc_kernel(TcParams p) {
    using L = Smem<DVC>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x;                 // b * H + h
    const int bb = head / p.H, h = head % p.H;
    const int T = p.T, H = p.H;
    const int dv0 = 0;                            // first value column of this CTA

    float *lw = (float *)(sm + L::LW);
    float *yb = (float *)(sm + L::YB);
    float *wtot = (float *)(sm + L::WT);
    float *probe = (float *)(sm + L::PR);
    float *vec = (float *)(sm + L::VEC);
    float *ecv = vec + 128, *fcv = vec + 256, *fprev = vec + 384, *gsv = vec + 512;
    float *spanred = vec + 640;                   // [8 warps][8]
    float *diagq = vec + 768, *diagb = vec + 896; // exact q~_t.k_t and q~_t.(b*k)_t
    float *part = (float *)(sm + L::PART);
    __nv_bfloat16 *gsm = (__nv_bfloat16 *)(sm + L::GS);
    uint64_t *mbar = (uint64_t *)(sm + L::MISC);
    uint32_t *tslot = (uint32_t *)(sm + L::MISC + 8);
    int *flags = (int *)(sm + L::MISC + 16);      // [0] abort, [1] chosen n, [2] log2 of the chunk
    uint64_t *tbar = (uint64_t *)(sm + L::MISC + 32);
    const uint32_t s_ap = tc::smem_u32(sm + L::AP), s_bp = tc::smem_u32(sm + L::BP);
    const uint32_t s_ti = tc::smem_u32(sm + L::TI), s_mm = tc::smem_u32(sm + L::MM);
    const uint32_t s_anab = tc::smem_u32(sm + L::ANAB), s_vh = tc::smem_u32(sm + L::VH);
    const uint32_t s_sc = tc::smem_u32(sm + L::SC), s_rr = tc::smem_u32(sm + L::RR);
    const uint32_t s_mbar = tc::smem_u32(mbar), s_tbar = tc::smem_u32(tbar);

    // ---- set-up: TMEM, mbarrier, per-head vectors
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_u32(tslot), 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(s_mbar, 1);
        tc::mbar_init(s_tbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
    }
    if (tid < kDK) {
        gsv[tid] = p.gs ? p.gs[(size_t)h * kDK + tid] : 1.f;
        fprev[tid] = 1.f;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;
    uint32_t phase = 0, tphase = 0;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's TMEM lanes
    const int row = 32 * (warp & 3) + lane;                         // accumulator row (M = 128)
    const int colhalf = warp >> 2;                                  // 0: warps 0-3, 1: warps 4-7
    float range_max = 0.f;

    // Wait for the MMAs committed so far; uniform abort on a timeout.
    auto wait_mma = [&]() -> bool {
        const bool ok = tc::mbar_wait(s_mbar, phase);
        if (!ok) flags[0] = 1;
        phase ^= 1u;
        __syncthreads();
        tc::fence_after_sync();
        return flags[0] == 0;
    };

    const size_t sbase = (size_t)head * kDK * kDV;
    bool first = true;
    bool prefetched = false;                      // the current window's record is already in flight
    for (int w = 0; w < p.NW && flags[0] == 0; ++w) {
    const int wend = min(T, kC * (w + 1));
    // windows with precomputed chunk tiles (intra kernel) take the fast path;
    // a flagged window (decay span too large for one 64-token chunk) is
    // processed here in shorter chunks
    const bool fast = p.ws != nullptr && p.wflags[(size_t)head * p.NW + w] == 0;
    for (int t0 = kC * w; t0 < wend;) {
        int n;
        if (fast) {
            const uint8_t *rec = p.ws + ((size_t)head * p.NW + w) * kWinBytes;
            if (tid == 0 && !prefetched) {
                tc::fence_proxy_async();
                tc::mbar_arrive_expect_tx(s_tbar, kWinBytes - kWinPad);
                tc::bulk_g2s(s_ap, rec + kWinAP, 128 * 256, s_tbar);
                tc::bulk_g2s(s_bp, rec + kWinBP, 128 * 256, s_tbar);
                tc::bulk_g2s(s_anab, rec + kWinANAB, 192 * 128, s_tbar);
                tc::bulk_g2s(s_vh, rec + kWinVH, 64 * 2 * kDV, s_tbar);
                tc::bulk_g2s(tc::smem_u32(ecv), rec + kWinVEC, 2 * 128 * 4, s_tbar);
            }
            // output gate of the window -> GS
            {
                const int tb = 8 * warp, c4 = 4 * lane;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int t = tb + u;
                    const size_t gv = (((size_t)bb * T + t0 + t) * H + h) * kDV + dv0 + c4;
                    uint2 gg = make_uint2(0, 0);
                    if (t0 + t < wend) gg = __ldg(reinterpret_cast<const uint2 *>(p.g + gv));
                    *reinterpret_cast<uint2 *>(gsm + t * DVC + c4) = gg;
                }
            }
            if (!tc::mbar_wait(s_tbar, tphase)) flags[0] = 1;
            tphase ^= 1u;
            __syncthreads();
            if (flags[0]) break;
            n = wend - t0;
            prefetched = false;
        } else {
            // ---- A: loads, cumulative log-decay, span, chunk length.
            // Warp w owns tokens [8w, 8w+8); lane l owns key channels [4l, 4l+4)
            // and value channels [4l, 4l+4), so every load instruction reads whole
            // 256-byte token rows.
            const int tb = 8 * warp, c4 = 4 * lane;
            float la[8][4];
            uint2 kq[8][4];                           // [token][k, q, z, b]: 4 bf16 each
    #pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = tb + u;
                const bool in = t0 + t < wend;
                const size_t gk = (((size_t)bb * T + t0 + t) * H + h) * kDK + c4;
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (in) x = __ldg(reinterpret_cast<const float4 *>(p.la + gk));
                la[u][0] = x.x; la[u][1] = x.y; la[u][2] = x.z; la[u][3] = x.w;
                kq[u][0] = in ? __ldg(reinterpret_cast<const uint2 *>(p.k + gk)) : make_uint2(0, 0);
                kq[u][1] = in ? __ldg(reinterpret_cast<const uint2 *>(p.q + gk)) : make_uint2(0, 0);
                kq[u][2] = in ? __ldg(reinterpret_cast<const uint2 *>(p.z + gk)) : make_uint2(0, 0);
                kq[u][3] = in ? __ldg(reinterpret_cast<const uint2 *>(p.b + gk)) : make_uint2(0, 0);
            }
            // inclusive scan over tokens: within this warp's 8 tokens, then across warps
    #pragma unroll
            for (int u = 1; u < 8; ++u)
    #pragma unroll
                for (int c = 0; c < 4; ++c) la[u][c] += la[u - 1][c];
            *reinterpret_cast<float4 *>(wtot + warp * kDK + c4) = make_float4(la[7][0], la[7][1], la[7][2], la[7][3]);
            __syncthreads();
            {
                float off[4] = {0.f, 0.f, 0.f, 0.f};
                for (int ww = 0; ww < warp; ++ww) {
                    const float4 o4 = *reinterpret_cast<const float4 *>(wtot + ww * kDK + c4);
                    off[0] += o4.x; off[1] += o4.y; off[2] += o4.z; off[3] += o4.w;
                }
    #pragma unroll
                for (int u = 0; u < 8; ++u)
    #pragma unroll
                    for (int c = 0; c < 4; ++c) la[u][c] += off[c];        // la now holds Lambda_t
            }
            // Lambda at tokens 0, 1, 3, 7, 15, 31, 63 (the last token of a chunk of 2^j)
    #pragma unroll
            for (int j = 0; j < 7; ++j) {
                const int pt = (1 << j) - 1;
                if (pt >= tb && pt < tb + 8) {
    #pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (tb + u == pt)
                            *reinterpret_cast<float4 *>(probe + j * kDK + c4) =
                                make_float4(la[u][0], la[u][1], la[u][2], la[u][3]);
                }
            }
            __syncthreads();
            {
                // span of a chunk of 2^j tokens: max over this thread's 4 channels, then the CTA
                const float4 l0 = *reinterpret_cast<const float4 *>(probe + c4);
                float sp[7];
    #pragma unroll
                for (int j = 0; j < 7; ++j) {
                    const float4 lj = *reinterpret_cast<const float4 *>(probe + j * kDK + c4);
                    float m = fmaxf(fmaxf(l0.x - lj.x, l0.y - lj.y), fmaxf(l0.z - lj.z, l0.w - lj.w));
    #pragma unroll
                    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    sp[j] = m;
                }
                if (lane == 0)
    #pragma unroll
                    for (int j = 0; j < 7; ++j) spanred[warp * 8 + j] = sp[j];
            }
            __syncthreads();
            if (tid == 0) {
                int nj = 0;
                for (int j = 6; j >= 0; --j) {
                    float m = 0.f;
                    for (int ww = 0; ww < 8; ++ww) m = fmaxf(m, spanred[ww * 8 + j]);
                    if (m <= kSpanMax) { nj = j; break; }
                }
                flags[1] = min(1 << nj, wend - t0);
                flags[2] = nj;
            }
            // value-side loads (their latency overlaps the operand computation)
            uint2 vw[8][3];                           // [token][v, w, g]
    #pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = tb + u;
                const bool in = t0 + t < wend;
                const size_t gv = (((size_t)bb * T + t0 + t) * H + h) * kDV + dv0 + c4;
                vw[u][0] = in ? __ldg(reinterpret_cast<const uint2 *>(p.v + gv)) : make_uint2(0, 0);
                vw[u][1] = in ? __ldg(reinterpret_cast<const uint2 *>(p.w + gv)) : make_uint2(0, 0);
                vw[u][2] = in ? __ldg(reinterpret_cast<const uint2 *>(p.g + gv)) : make_uint2(0, 0);
            }
            __syncthreads();
            n = flags[1];

            // ---- B: operand tiles (fp16, swizzled), pivot vectors, exact diagonals
            {
                // Lambda_{n-1} is the probe of the chosen power-of-two chunk: past the
                // end of the sequence the log-decay is zero-padded, so a shorter tail
                // has the same cumulative value there.
                const int jn = flags[2];
                const float4 l0 = *reinterpret_cast<const float4 *>(probe + c4);
                const float4 ln4 = *reinterpret_cast<const float4 *>(probe + jn * kDK + c4);
                const float l0v[4] = {l0.x, l0.y, l0.z, l0.w};
                const float lnv[4] = {ln4.x, ln4.y, ln4.z, ln4.w};
                float cpiv[4], gq[4];
    #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    cpiv[c] = 0.5f * (l0v[c] + lnv[c]);
                    gq[c] = gsv[c4 + c];
                    if (warp == 0) {
                        ecv[c4 + c] = __expf(cpiv[c]);
                        fcv[c4 + c] = __expf(lnv[c] - cpiv[c]);
                    }
                }
    #pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int t = tb + u;
                    const bool live = t < n;
                    float kk[4], qq[4], zz[4], bv[4];
                    {
                        const __nv_bfloat162 *hk = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][0]);
                        const __nv_bfloat162 *hq = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][1]);
                        const __nv_bfloat162 *hz = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][2]);
                        const __nv_bfloat162 *hb = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][3]);
    #pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            float2 f;
                            f = __bfloat1622float2(hk[e]); kk[2 * e] = f.x; kk[2 * e + 1] = f.y;
                            f = __bfloat1622float2(hq[e]); qq[2 * e] = f.x; qq[2 * e + 1] = f.y;
                            f = __bfloat1622float2(hz[e]); zz[2 * e] = f.x; zz[2 * e + 1] = f.y;
                            f = __bfloat1622float2(hb[e]); bv[2 * e] = f.x; bv[2 * e + 1] = f.y;
                        }
                    }
                    float kp[4], kc[4], khc[4], qp[4];
                    float dq = 0.f, db = 0.f;
    #pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float lam = live ? la[u][c] : lnv[c];     // identity padding past n
                        const float d = lam - cpiv[c];
                        const float ep = __expf(d), em = __expf(-d);
                        const float kv = live ? kk[c] : 0.f;
                        const float qt = live ? qq[c] * gq[c] * (2.f / (1.f + __expf(-zz[c]))) : 0.f;
                        const float kh = bv[c] * kv;
                        dq += qt * kv;
                        db += qt * kh;
                        kp[c] = kv * ep;
                        kc[c] = kv * em;
                        khc[c] = kh * em;
                        qp[c] = qt * ep;
                    }
                    range_max = fmaxf(range_max, fmaxf(fmaxf(maxabs(kp, 4), maxabs(kc, 4)),
                                                       fmaxf(maxabs(khc, 4), maxabs(qp, 4))));
                    // the diagonal of Aq / Bq carries no decay: it is summed exactly in
                    // fp32 (a readout whose q~.k nearly cancels, e.g. the first token of a
                    // sequence, is then free of fp16 operand rounding)
    #pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        dq += __shfl_xor_sync(0xffffffffu, dq, o);
                        db += __shfl_xor_sync(0xffffffffu, db, o);
                    }
                    if (lane == 0) {
                        diagq[t] = dq;
                        diagb[t] = db;
                    }
                    const uint32_t off_t = tc::tile_off(128, t, c4), off_b = tc::tile_off(128, 64 + t, c4);
                    *(uint2 *)(sm + L::AP + off_t) = make_uint2(tc::pack_half2(kp[0], kp[1]), tc::pack_half2(kp[2], kp[3]));
                    *(uint2 *)(sm + L::AP + off_b) = make_uint2(tc::pack_half2(qp[0], qp[1]), tc::pack_half2(qp[2], qp[3]));
                    *(uint2 *)(sm + L::BP + off_t) = make_uint2(tc::pack_half2(kc[0], kc[1]), tc::pack_half2(kc[2], kc[3]));
                    *(uint2 *)(sm + L::BP + off_b) =
                        make_uint2(tc::pack_half2(khc[0], khc[1]), tc::pack_half2(khc[2], khc[3]));
                }
                if (c4 < DVC) {
    #pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int t = tb + u;
                        const bool live = t < n;
                        const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&vw[u][0]);
                        const __nv_bfloat162 *hw = reinterpret_cast<const __nv_bfloat162 *>(&vw[u][1]);
                        float vh[4];
    #pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float2 fv = __bfloat1622float2(hv[e]), fw = __bfloat1622float2(hw[e]);
                            vh[2 * e] = live ? fv.x * fw.x : 0.f;
                            vh[2 * e + 1] = live ? fv.y * fw.y : 0.f;
                        }
                        *(uint2 *)(sm + L::VH + tc::tile_off(64, t, c4)) =
                            make_uint2(tc::pack_half2(vh[0], vh[1]), tc::pack_half2(vh[2], vh[3]));
                        *reinterpret_cast<uint2 *>(gsm + t * DVC + c4) = vw[u][2];
                    }
                }
            }
            tc::fence_proxy_async();
            __syncthreads();

            // ---- C: decay-relative products P = [Kp; Qp] [Kc; K^c]^T
            if (tid == 0) {
                tc::fence_after_sync();
                const uint32_t id = tc::idesc_f16(128, 128, false, false, false);
                for (int ks = 0; ks < kDK / 16; ++ks)
                    tc::mma_f16(tmem + kTmP, tc::desc_kmajor(s_ap, 128, 0, ks), tc::desc_kmajor(s_bp, 128, 0, ks), id,
                                ks > 0);
                tc::mma_commit(s_mbar);
            }
            if (!wait_mma()) break;

            // ---- D: masks; M -> MM, L -> fp32, Aq/Bq -> ANAB
            {
                // rows 0-63: warps 0,1 (M, cols 0-63) and warps 4,5 (L, cols 64-127)
                // rows 64-127: warps 2,3 (Aq) and warps 6,7 (Bq)
                const int t = row & 63;
                const bool upper = row < 64;
                float v[2][32];
                tc::tmem_ld32x2(tmem + lane_base + kTmP + 64 * colhalf, tmem + lane_base + kTmP + 64 * colhalf + 32,
                                v[0], v[1]);
    #pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
    #pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int s = 32 * hf + i;
                        const bool keep = upper ? (s < t) : (s <= t);
                        if (!keep) v[hf][i] = 0.f;
                        if (!upper && s == t) v[hf][i] = colhalf == 0 ? diagq[t] : diagb[t];
                    }
                    if (upper && colhalf == 1) {
                        float4 *dst = reinterpret_cast<float4 *>(lw + t * kLW + 32 * hf);
    #pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(v[hf][4 * q], v[hf][4 * q + 1], v[hf][4 * q + 2], v[hf][4 * q + 3]);
                    } else {
                        uint8_t *tile = upper ? sm + L::MM : sm + L::ANAB;
                        const int R = upper ? 64 : 192;
                        const int r = upper ? t : (colhalf == 0 ? 64 + t : 128 + t);
                        store_row32(tile, R, r, 32 * hf, v[hf]);
                    }
                }
            }
            tc::fence_before_sync();
            __syncthreads();

            // ---- E: T^-1 = (I + L)^-1 in place, divide and conquer (fp32)
            {
                // leaves of 8: forward substitution per column, in registers
                if (tid < 64) {
                    const int o = 8 * (tid >> 3), j = tid & 7;
                    float Lr[8][8];
    #pragma unroll
                    for (int i = 1; i < 8; ++i)
    #pragma unroll
                        for (int s = 0; s < i; ++s) Lr[i][s] = lw[(o + i) * kLW + o + s];
                    float x[8];
    #pragma unroll
                    for (int i = 0; i < 8; ++i) x[i] = (i == j) ? 1.f : 0.f;
    #pragma unroll
                    for (int i = 1; i < 8; ++i) {
                        float acc = 0.f;
    #pragma unroll
                        for (int s = 0; s < i; ++s) acc += Lr[i][s] * x[s];
                        if (i > j) x[i] = -acc;
                    }
                    __syncwarp();
                    asm volatile("bar.sync 1, 64;" ::: "memory");     // the 64 leaf threads only
    #pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (i >= j) lw[(o + i) * kLW + o + j] = x[i];
                }
                __syncthreads();
                // merges: [[A, 0], [C, D]]^-1 = [[A^-1, 0], [-D^-1 C A^-1, D^-1]],
                // four output columns per task; the upper triangles are zero, so the
                // sums run over whole blocks without masks
                merge_level<8>(lw, yb, tid);
                merge_level<16>(lw, yb, tid);
                merge_level<32>(lw, yb, tid);
                // T^-1 -> fp16 tile (row t, column s; the upper part of lw is zero)
                for (int u = tid; u < 64 * 8; u += kThreads) {
                    const int t = u >> 3, g8 = u & 7;
                    const float4 a = *reinterpret_cast<const float4 *>(lw + t * kLW + 8 * g8);
                    const float4 b4 = *reinterpret_cast<const float4 *>(lw + t * kLW + 8 * g8 + 4);
                    const float f[8] = {a.x, a.y, a.z, a.w, b4.x, b4.y, b4.z, b4.w};
                    *(uint4 *)(sm + L::TI + tc::tile_chunk_off(64, t, g8)) = pack8(f);
                }
            }
            tc::fence_proxy_async();
            __syncthreads();

            // ---- F: W' = T^-1 Kp, N = T^-1 M
            if (tid == 0) {
                tc::fence_after_sync();
                const uint32_t idw = tc::idesc_f16(64, 128, false, true, false);
                const uint32_t idn = tc::idesc_f16(64, 64, false, true, false);
                for (int ks = 0; ks < kC / 16; ++ks)
                    tc::mma_f16(tmem + kTmW, tc::desc_kmajor(s_ti, 64, 0, ks), tc::desc_mnmajor(s_ap, 128, 0, ks), idw,
                                ks > 0);
                for (int ks = 0; ks < kC / 16; ++ks)
                    tc::mma_f16(tmem + kTmN, tc::desc_kmajor(s_ti, 64, 0, ks), tc::desc_mnmajor(s_mm, 64, 0, ks), idn,
                                ks > 0);
                tc::mma_commit(s_mbar);
            }
            if (!wait_mma()) break;

            // ---- G: W' -> rows 0-63 of AP (over Kp), N -> rows 0-63 of ANAB.
            // M = 64 accumulators sit in lanes 0-15 of each 32-lane group.
            {
                const int t = 16 * (warp & 3) + lane;
                const bool valid = lane < 16;
                float v[2][32];
                // warps 0-3: W' columns 0-63; warps 4-7: W' columns 64-127
                tc::tmem_ld32x2(tmem + lane_base + kTmW + 64 * colhalf, tmem + lane_base + kTmW + 64 * colhalf + 32, v[0],
                                v[1]);
                if (valid) {
    #pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        range_max = fmaxf(range_max, maxabs(v[hf], 32));
                        store_row32(sm + L::AP, 128, t, 64 * colhalf + 32 * hf, v[hf]);
                    }
                }
                // warps 0-3: N columns 0-31; warps 4-7: N columns 32-63
                float nv[32];
                tc::tmem_ld32(tmem + lane_base + kTmN + 32 * colhalf, nv);
                if (valid) {
                    range_max = fmaxf(range_max, maxabs(nv, 32));
                    store_row32(sm + L::ANAB, 192, t, 32 * colhalf, nv);
                }
            }

        }
        // ---- H: state operand S_c = Diag(e^c) S, X <- S_c (fp32, TMEM)
        {
            const int i = row;                                   // key channel
            const float scale = ecv[i] * fprev[i];
            for (int cblk = 0; cblk < DVC / 64; ++cblk) {
                const int col = (DVC / 2) * colhalf + 32 * cblk;
                float v[32];
                if (first) {
                    if (p.S_in) {
                        const float4 *src = reinterpret_cast<const float4 *>(p.S_in + sbase + (size_t)i * kDV + dv0 + col);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 x4 = __ldg(src + q);
                            v[4 * q] = x4.x; v[4 * q + 1] = x4.y; v[4 * q + 2] = x4.z; v[4 * q + 3] = x4.w;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) v[q] = 0.f;
                    }
                } else {
                    tc::tmem_ld32(tmem + lane_base + kTmX + col, v);
                }
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] *= scale;
                tc::tmem_st32(tmem + lane_base + kTmX + col, v);
                range_max = fmaxf(range_max, maxabs(v, 32));
                store_row32(sm + L::SC, 128, i, col, v);
            }
        }
        first = false;
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();

        // ---- I: [R; O] = [W'; Qp] S_c + [N; Aq] V^ ;  X += Kc^T V^
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id1 = tc::idesc_f16(128, DVC, false, true, false);
            for (int ks = 0; ks < kDK / 16; ++ks)
                tc::mma_f16(tmem + kTmP, tc::desc_kmajor(s_ap, 128, 0, ks), tc::desc_mnmajor(s_sc, 128, 0, ks), id1,
                            ks > 0);
            for (int ks = 0; ks < kC / 16; ++ks)
                tc::mma_f16(tmem + kTmP, tc::desc_kmajor(s_anab, 192, 0, ks), tc::desc_mnmajor(s_vh, 64, 0, ks), id1,
                            true);
            const uint32_t id2 = tc::idesc_f16(128, DVC, true, true, false);
            for (int ks = 0; ks < kC / 16; ++ks)
                tc::mma_f16(tmem + kTmX, tc::desc_mnmajor(s_bp, 128, 0, ks), tc::desc_mnmajor(s_vh, 64, 0, ks), id2,
                            true);
            tc::mma_commit(s_mbar);
        }
        if (!wait_mma()) break;

        // ---- J: R (rows 0-63) -> fp16 tile
        if (row < 64) {
            float v[2][32];
            tc::tmem_ld32x2(tmem + lane_base + kTmP + (DVC / 2) * colhalf,
                            tmem + lane_base + kTmP + (DVC / 2) * colhalf + 32, v[0], v[1]);
#pragma unroll
            for (int hf = 0; hf < DVC / 64; ++hf) {
                range_max = fmaxf(range_max, maxabs(v[hf], 32));
                store_row32(sm + L::RR, 64, row, (DVC / 2) * colhalf + 32 * hf, v[hf]);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();

        // ---- K: O -= Bq R (rows 64-127; rows 0-63 receive -Aq R, unused);  X -= K^c^T R
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id1 = tc::idesc_f16(128, DVC, false, true, true);
            for (int ks = 0; ks < kC / 16; ++ks)
                tc::mma_f16(tmem + kTmP, tc::desc_kmajor(s_anab, 192, 64, ks), tc::desc_mnmajor(s_rr, 64, 0, ks), id1,
                            true);
            const uint32_t id2 = tc::idesc_f16(128, DVC, true, true, true);
            for (int ks = 0; ks < kC / 16; ++ks)
                tc::mma_f16(tmem + kTmX, tc::desc_mnmajor(s_bp, 128, 64, ks), tc::desc_mnmajor(s_rr, 64, 0, ks), id2,
                            true);
            tc::mma_commit(s_mbar);
        }
        if (!wait_mma()) break;
        // the chunk's tiles are free: keep its decay factor, then start the
        // bulk copy of the next window's record so it overlaps the epilogue
        if (tid < kDK) fprev[tid] = fcv[tid];
        {
            const bool next_fast = t0 + n == wend && w + 1 < p.NW && p.ws != nullptr &&
                                   p.wflags[(size_t)head * p.NW + w + 1] == 0;
            __syncthreads();
            if (next_fast) {
                if (tid == 0) {
                    const uint8_t *nrec = p.ws + ((size_t)head * p.NW + w + 1) * kWinBytes;
                    tc::fence_proxy_async();
                    tc::mbar_arrive_expect_tx(s_tbar, kWinBytes - kWinPad);
                    tc::bulk_g2s(s_ap, nrec + kWinAP, 128 * 256, s_tbar);
                    tc::bulk_g2s(s_bp, nrec + kWinBP, 128 * 256, s_tbar);
                    tc::bulk_g2s(s_anab, nrec + kWinANAB, 192 * 128, s_tbar);
                    tc::bulk_g2s(s_vh, nrec + kWinVH, 64 * 2 * kDV, s_tbar);
                    tc::bulk_g2s(tc::smem_u32(ecv), nrec + kWinVEC, 2 * 128 * 4, s_tbar);
                }
                prefetched = true;
            }
        }

        // ---- L: O (rows 64-127) -> RMSNorm over the head's d_v, gate, store
        {
            const bool orow = row >= 64;
            const int t = row - 64;
            float ov[2][32];
            float ss = 0.f;
            if (orow) {
                tc::tmem_ld32x2(tmem + lane_base + kTmP + (DVC / 2) * colhalf,
                                tmem + lane_base + kTmP + (DVC / 2) * colhalf + 32, ov[0], ov[1]);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int q = 0; q < 32; ++q) ss += ov[hf][q] * ov[hf][q];
                part[t * 2 + colhalf] = ss;
            }
            __syncthreads();
            if (orow && t < n) {
                const float tot = part[t * 2] + part[t * 2 + 1];
                const float inv = rsqrtf(tot / kDV + p.eps);
                const int c0 = (DVC / 2) * colhalf;
                const size_t gi = (((size_t)bb * T + t0 + t) * H + h) * kDV + dv0 + c0;
#pragma unroll
                for (int q8 = 0; q8 < DVC / 16; ++q8) {
                    float gg[8], yy[8];
                    bf16x8_to_f(*reinterpret_cast<const uint4 *>(gsm + t * DVC + c0 + 8 * q8), gg);
                    const float *o8 = &ov[q8 >> 2][8 * (q8 & 3)];
#pragma unroll
                    for (int e = 0; e < 8; ++e) yy[e] = gg[e] * o8[e] * inv;
                    uint4 u;
                    __nv_bfloat162 *hb = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) hb[e] = __floats2bfloat162_rn(yy[2 * e], yy[2 * e + 1]);
                    *reinterpret_cast<uint4 *>(p.y + gi + 8 * q8) = u;
                    if (p.o_raw) {
                        float4 *dst = reinterpret_cast<float4 *>(p.o_raw + gi + 8 * q8);
                        dst[0] = make_float4(o8[0], o8[1], o8[2], o8[3]);
                        dst[1] = make_float4(o8[4], o8[5], o8[6], o8[7]);
                    }
                }
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        t0 += n;
    }
    }

    // a prefetch still in flight (the loop ended early) completes before exit
    if (prefetched) tc::mbar_wait(s_tbar, tphase);

    // ---- S_out = Diag(f) X
    if (flags[0] == 0 && p.S_out && T > 0) {
        const int i = row;
        for (int cblk = 0; cblk < DVC / 64; ++cblk) {
            const int col = (DVC / 2) * colhalf + 32 * cblk;
            float v[32];
            tc::tmem_ld32(tmem + lane_base + kTmX + col, v);
            float4 *dst = reinterpret_cast<float4 *>(p.S_out + sbase + (size_t)i * kDV + dv0 + col);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(v[4 * q] * fprev[i], v[4 * q + 1] * fprev[i], v[4 * q + 2] * fprev[i],
                                     v[4 * q + 3] * fprev[i]);
        }
    }
    if (range_max > 60000.f && p.status) atomicCAS(p.status, 0, (int)kDevRange);
    if (flags[0] != 0 && tid == 0 && p.status) atomicCAS(p.status, 0, (int)kDevTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Intra-chunk kernel: one CTA per 64-token window, all windows in parallel.
// It computes everything of a chunk that does not depend on the state -- the
// decay-relative products, (I + L)^-1, W' = T^-1 Kp and N = T^-1 M -- and
// writes the chunk's operand tiles to the window's workspace record in the
// byte layout the chain kernel loads with one bulk copy per tile.  A window
// whose decay span exceeds kSpanMax is flagged instead and handled by the
// chain kernel in shorter chunks.
// ---------------------------------------------------------------------------
namespace {
struct IntraSmem {
    static constexpr int AP = 0;                  // [Kp ; Qp]   128 x 128 fp16
    static constexpr int BP = AP + 128 * 256;     // [Kc ; K^c]  128 x 128; after P: fp32 L / T^-1 + merge buffer
    static constexpr int TI = BP + 128 * 256;     // T^-1         64 x 64
    static constexpr int MM = TI + 64 * 128;      // M            64 x 64
    static constexpr int WT = MM + 64 * 128;      // fp32 per-warp log-decay totals [8][128]
    static constexpr int PR = WT + 8 * 128 * 4;   // fp32 Lambda at the probe tokens [8][128]
    static constexpr int VEC = PR + 8 * 128 * 4;  // gamma_stat, exact diagonals, span maxima
    static constexpr int MISC = VEC + 512 * 4;    // mbarrier, TMEM slot, flags
    static constexpr int TOTAL = MISC + 64;
};
constexpr uint32_t kItmW = 0;      // W' (M=64) reuses the columns of P after its epilogue
constexpr uint32_t kItmN = 128;    // N  (M=64)
}  // namespace

__global__ void __launch_bounds__(kThreads, 2) gdn2_chunk_intra_tc_kernel(TcParams p, uint8_t *ws, int *wflags) {
    using L = IntraSmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wi = blockIdx.x, NW = p.NW;
    const int head = wi / NW, win = wi % NW;
    const int bb = head / p.H, h = head % p.H;
    const int T = p.T, H = p.H;
    const int t0 = kC * win, wend = min(T, t0 + kC);
    uint8_t *rec = ws + (size_t)wi * kWinBytes;

    float *lw = (float *)(sm + L::BP);
    float *yb = lw + 64 * kLW;
    float *wtot = (float *)(sm + L::WT);
    float *probe = (float *)(sm + L::PR);
    float *vec = (float *)(sm + L::VEC);
    float *gsv = vec, *diagq = vec + 128, *diagb = vec + 192, *spanred = vec + 256;
    uint64_t *mbar = (uint64_t *)(sm + L::MISC);
    uint32_t *tslot = (uint32_t *)(sm + L::MISC + 8);
    int *flags = (int *)(sm + L::MISC + 16);
    const uint32_t s_ap = tc::smem_u32(sm + L::AP), s_bp = tc::smem_u32(sm + L::BP);
    const uint32_t s_ti = tc::smem_u32(sm + L::TI), s_mm = tc::smem_u32(sm + L::MM);
    const uint32_t s_mbar = tc::smem_u32(mbar);

    if (warp == 0) {
        tc::tmem_alloc(tc::smem_u32(tslot), 256);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(s_mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
    }
    if (tid < kDK) gsv[tid] = p.gs ? p.gs[(size_t)h * kDK + tid] : 1.f;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;
    uint32_t phase = 0;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int row = 32 * (warp & 3) + lane;
    const int colhalf = warp >> 2;
    float range_max = 0.f;
    auto wait_mma = [&]() -> bool {
        const bool ok = tc::mbar_wait(s_mbar, phase);
        if (!ok) flags[0] = 1;
        phase ^= 1u;
        __syncthreads();
        tc::fence_after_sync();
        return flags[0] == 0;
    };

    do {
        // ---- loads (whole 256-byte token rows per instruction) and the log-decay
        // scan, in log2 units (Lambda * log2 e) so that every decay factor is one ex2
        const int tb = 8 * warp, c4 = 4 * lane;
        float la[8][4];
        uint2 kq[8][4];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = tb + u;
            const bool in = t0 + t < wend;
            const size_t gk = (((size_t)bb * T + t0 + t) * H + h) * kDK + c4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (in) x = __ldg(reinterpret_cast<const float4 *>(p.la + gk));
            la[u][0] = x.x * kLog2e; la[u][1] = x.y * kLog2e; la[u][2] = x.z * kLog2e; la[u][3] = x.w * kLog2e;
            kq[u][0] = in ? __ldg(reinterpret_cast<const uint2 *>(p.k + gk)) : make_uint2(0, 0);
            kq[u][1] = in ? __ldg(reinterpret_cast<const uint2 *>(p.q + gk)) : make_uint2(0, 0);
            kq[u][2] = in ? __ldg(reinterpret_cast<const uint2 *>(p.z + gk)) : make_uint2(0, 0);
            kq[u][3] = in ? __ldg(reinterpret_cast<const uint2 *>(p.b + gk)) : make_uint2(0, 0);
        }
#pragma unroll
        for (int u = 1; u < 8; ++u)
#pragma unroll
            for (int c = 0; c < 4; ++c) la[u][c] += la[u - 1][c];
        *reinterpret_cast<float4 *>(wtot + warp * kDK + c4) = make_float4(la[7][0], la[7][1], la[7][2], la[7][3]);
        __syncthreads();
        {
            float off[4] = {0.f, 0.f, 0.f, 0.f};
            for (int ww = 0; ww < warp; ++ww) {
                const float4 o4 = *reinterpret_cast<const float4 *>(wtot + ww * kDK + c4);
                off[0] += o4.x; off[1] += o4.y; off[2] += o4.z; off[3] += o4.w;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int c = 0; c < 4; ++c) la[u][c] += off[c];
        }
        // Lambda at token 0 and at the last token (zero-padded log-decay past the end)
        if (warp == 0) *reinterpret_cast<float4 *>(probe + c4) = make_float4(la[0][0], la[0][1], la[0][2], la[0][3]);
        if (warp == 7) *reinterpret_cast<float4 *>(probe + kDK + c4) = make_float4(la[7][0], la[7][1], la[7][2], la[7][3]);
        __syncthreads();
        const float4 l0 = *reinterpret_cast<const float4 *>(probe + c4);
        const float4 ln4 = *reinterpret_cast<const float4 *>(probe + kDK + c4);
        {
            float m = fmaxf(fmaxf(l0.x - ln4.x, l0.y - ln4.y), fmaxf(l0.z - ln4.z, l0.w - ln4.w));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) spanred[warp] = m;
        }
        __syncthreads();
        {
            float m = 0.f;
#pragma unroll
            for (int ww = 0; ww < 8; ++ww) m = fmaxf(m, spanred[ww]);
            if (m > kSpanMax * kLog2e) {              // the chain kernel takes this window
                if (tid == 0) wflags[wi] = 1;
                break;
            }
        }
        const int n = wend - t0;

        // ---- operand tiles: P operands to shared memory; Qp, Kc, K^c and the
        // pivot vectors straight to the window record
        {
            const float l0v[4] = {l0.x, l0.y, l0.z, l0.w};
            const float lnv[4] = {ln4.x, ln4.y, ln4.z, ln4.w};
            float cpiv[4], gq[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                cpiv[c] = 0.5f * (l0v[c] + lnv[c]);
                gq[c] = gsv[c4 + c];
            }
            if (warp == 0) {
                float4 *rv = reinterpret_cast<float4 *>(rec + kWinVEC);
                rv[lane] = make_float4(ex2(cpiv[0]), ex2(cpiv[1]), ex2(cpiv[2]), ex2(cpiv[3]));
                rv[32 + lane] = make_float4(ex2(lnv[0] - cpiv[0]), ex2(lnv[1] - cpiv[1]), ex2(lnv[2] - cpiv[2]),
                                            ex2(lnv[3] - cpiv[3]));
            }
            float dg[16];                             // [u]: q~.k, [8+u]: q~.(b*k) of token tb+u, this lane's channels
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = tb + u;
                const bool live = t < n;
                float kk[4], qq[4], zz[4], bv[4];
                {
                    const __nv_bfloat162 *hk = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][0]);
                    const __nv_bfloat162 *hq = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][1]);
                    const __nv_bfloat162 *hz = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][2]);
                    const __nv_bfloat162 *hb = reinterpret_cast<const __nv_bfloat162 *>(&kq[u][3]);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float2 f;
                        f = __bfloat1622float2(hk[e]); kk[2 * e] = f.x; kk[2 * e + 1] = f.y;
                        f = __bfloat1622float2(hq[e]); qq[2 * e] = f.x; qq[2 * e + 1] = f.y;
                        f = __bfloat1622float2(hz[e]); zz[2 * e] = f.x; zz[2 * e + 1] = f.y;
                        f = __bfloat1622float2(hb[e]); bv[2 * e] = f.x; bv[2 * e + 1] = f.y;
                    }
                }
                float kp[4], kc[4], khc[4], qp[4];
                float dq = 0.f, db = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float lam = live ? la[u][c] : lnv[c];
                    const float d = lam - cpiv[c];
                    const float ep = ex2(d), em = ex2(-d);
                    const float kv = live ? kk[c] : 0.f;
                    const float qt = live ? qq[c] * gq[c] * two_sigmoid_fast(zz[c]) : 0.f;
                    const float kh = bv[c] * kv;
                    dq += qt * kv;
                    db += qt * kh;
                    kp[c] = kv * ep;
                    kc[c] = kv * em;
                    khc[c] = kh * em;
                    qp[c] = qt * ep;
                }
                range_max = fmaxf(range_max, fmaxf(fmaxf(maxabs(kp, 4), maxabs(kc, 4)),
                                                   fmaxf(maxabs(khc, 4), maxabs(qp, 4))));
                dg[u] = dq;
                dg[8 + u] = db;
                const uint32_t off_t = tc::tile_off(128, t, c4), off_b = tc::tile_off(128, 64 + t, c4);
                const uint2 ukp = make_uint2(tc::pack_half2(kp[0], kp[1]), tc::pack_half2(kp[2], kp[3]));
                const uint2 uqp = make_uint2(tc::pack_half2(qp[0], qp[1]), tc::pack_half2(qp[2], qp[3]));
                const uint2 ukc = make_uint2(tc::pack_half2(kc[0], kc[1]), tc::pack_half2(kc[2], kc[3]));
                const uint2 ukh = make_uint2(tc::pack_half2(khc[0], khc[1]), tc::pack_half2(khc[2], khc[3]));
                *(uint2 *)(sm + L::AP + off_t) = ukp;
                *(uint2 *)(sm + L::AP + off_b) = uqp;
                *(uint2 *)(sm + L::BP + off_t) = ukc;
                *(uint2 *)(sm + L::BP + off_b) = ukh;
                *(uint2 *)(rec + kWinAP + off_b) = uqp;
                *(uint2 *)(rec + kWinBP + off_t) = ukc;
                *(uint2 *)(rec + kWinBP + off_b) = ukh;
            }
            // the exact diagonals q~_t.k_t and q~_t.(b*k)_t of Aq / Bq
            const float dsum = reduce_scatter16(dg, lane);
            if ((lane & 1) == 0) {
                const int vi = (lane >> 1) & 15;
                (vi < 8 ? diagq : diagb)[tb + (vi & 7)] = dsum;
            }
        }
        // value side: loads issued now, consumed while the P product runs
        uint2 vw[8][2];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = tb + u;
            const bool in = t0 + t < wend;
            const size_t gv = (((size_t)bb * T + t0 + t) * H + h) * kDV + c4;
            vw[u][0] = in ? __ldg(reinterpret_cast<const uint2 *>(p.v + gv)) : make_uint2(0, 0);
            vw[u][1] = in ? __ldg(reinterpret_cast<const uint2 *>(p.w + gv)) : make_uint2(0, 0);
        }
        tc::fence_proxy_async();
        __syncthreads();

        // ---- P = [Kp; Qp] [Kc; K^c]^T
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id = tc::idesc_f16(128, 128, false, false, false);
            for (int ks = 0; ks < kDK / 16; ++ks)
                tc::mma_f16(tmem, tc::desc_kmajor(s_ap, 128, 0, ks), tc::desc_kmajor(s_bp, 128, 0, ks), id, ks > 0);
            tc::mma_commit(s_mbar);
        }
        // V^ = w*v -> window record (the identity padding past n is zero)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = tb + u;
            const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&vw[u][0]);
            const __nv_bfloat162 *hw = reinterpret_cast<const __nv_bfloat162 *>(&vw[u][1]);
            float vh[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float2 fv = __bfloat1622float2(hv[e]), fw = __bfloat1622float2(hw[e]);
                vh[2 * e] = fv.x * fw.x;
                vh[2 * e + 1] = fv.y * fw.y;
            }
            *(uint2 *)(rec + kWinVH + tc::tile_off(64, t, c4)) =
                make_uint2(tc::pack_half2(vh[0], vh[1]), tc::pack_half2(vh[2], vh[3]));
        }
        if (!wait_mma()) break;

        // ---- masks; M -> MM (shared), L -> fp32 (over BP), Aq / Bq -> record.
        // This warp's rows are tokens t in [32 tb2, 32 tb2 + 32): column block hf
        // below the diagonal block is kept whole, above it zeroed, and only the
        // diagonal block is masked element by element.
        {
            const int t = row & 63;
            const bool upper = row < 64;
            const int tb2 = warp & 1;
            float v[2][32];
            tc::tmem_ld32x2(tmem + lane_base + 64 * colhalf, tmem + lane_base + 64 * colhalf + 32, v[0], v[1]);
            // all warps have read P; BP may now be overwritten with L
            tc::fence_before_sync();
            __syncthreads();
            const float dv_t = upper ? 0.f : (colhalf == 0 ? diagq[t] : diagb[t]);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                if (hf > tb2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[hf][i] = 0.f;
                } else if (hf == tb2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const bool keep = upper ? (i < lane) : (i <= lane);
                        if (!keep) v[hf][i] = 0.f;
                        if (!upper && i == lane) v[hf][i] = dv_t;
                    }
                }
                if (upper && colhalf == 1) {
                    float4 *dst = reinterpret_cast<float4 *>(lw + t * kLW + 32 * hf);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_float4(v[hf][4 * q], v[hf][4 * q + 1], v[hf][4 * q + 2], v[hf][4 * q + 3]);
                } else if (upper) {
                    store_row32(sm + L::MM, 64, t, 32 * hf, v[hf]);
                } else {
                    store_row32(rec + kWinANAB, 192, colhalf == 0 ? 64 + t : 128 + t, 32 * hf, v[hf]);
                }
            }
        }
        tc::fence_before_sync();
        __syncthreads();

        // ---- T^-1 = (I + L)^-1 (divide and conquer, fp32)
        {
            if (tid < 64) {
                const int o = 8 * (tid >> 3), j = tid & 7;
                float Lr[8][8];
#pragma unroll
                for (int i = 1; i < 8; ++i)
#pragma unroll
                    for (int s = 0; s < i; ++s) Lr[i][s] = lw[(o + i) * kLW + o + s];
                float x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
                for (int i = 1; i < 8; ++i) {
                    float acc = 0.f;
#pragma unroll
                    for (int s = 0; s < i; ++s) acc += Lr[i][s] * x[s];
                    if (i > j) x[i] = -acc;
                }
                asm volatile("bar.sync 1, 64;" ::: "memory");
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i >= j) lw[(o + i) * kLW + o + j] = x[i];
            }
            __syncthreads();
            merge_level<8>(lw, yb, tid);
            merge_level<16>(lw, yb, tid);
            merge_level<32>(lw, yb, tid);
            for (int u = tid; u < 64 * 8; u += kThreads) {
                const int t = u >> 3, g8 = u & 7;
                const float4 a = *reinterpret_cast<const float4 *>(lw + t * kLW + 8 * g8);
                const float4 b4 = *reinterpret_cast<const float4 *>(lw + t * kLW + 8 * g8 + 4);
                const float f[8] = {a.x, a.y, a.z, a.w, b4.x, b4.y, b4.z, b4.w};
                *(uint4 *)(sm + L::TI + tc::tile_chunk_off(64, t, g8)) = pack8(f);
            }
        }
        tc::fence_proxy_async();
        __syncthreads();

        // ---- W' = T^-1 Kp, N = T^-1 M
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t idw = tc::idesc_f16(64, 128, false, true, false);
            const uint32_t idn = tc::idesc_f16(64, 64, false, true, false);
            for (int ks = 0; ks < kC / 16; ++ks)
                tc::mma_f16(tmem + kItmW, tc::desc_kmajor(s_ti, 64, 0, ks), tc::desc_mnmajor(s_ap, 128, 0, ks), idw,
                            ks > 0);
            for (int ks = 0; ks < kC / 16; ++ks)
                tc::mma_f16(tmem + kItmN, tc::desc_kmajor(s_ti, 64, 0, ks), tc::desc_mnmajor(s_mm, 64, 0, ks), idn,
                            ks > 0);
            tc::mma_commit(s_mbar);
        }
        if (!wait_mma()) break;

        // ---- W' -> record rows 0-63 of [W'; Qp]; N -> record rows 0-63 of [N; Aq; Bq]
        {
            const int t = 16 * (warp & 3) + lane;
            const bool valid = lane < 16;
            float v[2][32];
            tc::tmem_ld32x2(tmem + lane_base + kItmW + 64 * colhalf, tmem + lane_base + kItmW + 64 * colhalf + 32, v[0],
                            v[1]);
            if (valid) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    range_max = fmaxf(range_max, maxabs(v[hf], 32));
                    store_row32(rec + kWinAP, 128, t, 64 * colhalf + 32 * hf, v[hf]);
                }
            }
            float nv[32];
            tc::tmem_ld32(tmem + lane_base + kItmN + 32 * colhalf, nv);
            if (valid) {
                range_max = fmaxf(range_max, maxabs(nv, 32));
                store_row32(rec + kWinANAB, 192, t, 32 * colhalf, nv);
            }
        }
        if (tid == 0) wflags[wi] = 0;
    } while (false);

    if (range_max > 60000.f && p.status) atomicCAS(p.status, 0, (int)kDevRange);
    if (flags[0] != 0 && tid == 0 && p.status) atomicCAS(p.status, 0, (int)kDevTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

size_t fwd_tc_workspace_bytes(int B, int H, int T) {
    const size_t nwin = (size_t)B * H * ((T + kC - 1) / kC);
    return nwin * kWinBytes + ((nwin * sizeof(int) + 1023) & ~(size_t)1023);
}

size_t fwd_tc_smem_bytes(int dvc) {
    return (dvc == 128 ? (size_t)Smem<128>::TOTAL : (size_t)Smem<64>::TOTAL) + 1024;
}

bool fwd_tc_supported(int dtype, int dk, int dv, int chunk) {
    return dtype == GDELTA_BF16 && dk == 128 && dv == 128 && chunk == 64;
}

cudaError_t launch_fwd_tc(const FwdParams &fp, void *workspace, cudaStream_t stream) {
    TcParams p;
    p.B = fp.B; p.T = fp.T; p.H = fp.H;
    p.q = (const __nv_bfloat16 *)fp.q; p.k = (const __nv_bfloat16 *)fp.k; p.z = (const __nv_bfloat16 *)fp.z;
    p.b = (const __nv_bfloat16 *)fp.b; p.v = (const __nv_bfloat16 *)fp.v; p.w = (const __nv_bfloat16 *)fp.w;
    p.g = (const __nv_bfloat16 *)fp.g;
    p.la = fp.la; p.gs = fp.gs; p.S_in = fp.S_in; p.S_out = fp.S_out;
    p.y = (__nv_bfloat16 *)fp.y; p.o_raw = fp.o_raw; p.eps = fp.eps; p.status = fp.status;
    p.NW = (fp.T + kC - 1) / kC;
    const size_t nwin = (size_t)fp.B * fp.H * p.NW;
    uint8_t *ws = (uint8_t *)workspace;
    int *wflags = (int *)(ws + nwin * kWinBytes);
    p.ws = ws;
    p.wflags = wflags;
    const size_t ismem = (size_t)IntraSmem::TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(gdn2_chunk_intra_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ismem);
    if (e != cudaSuccess) return e;
    gdn2_chunk_intra_tc_kernel<<<(unsigned)nwin, kThreads, ismem, stream>>>(p, ws, wflags);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = fwd_tc_smem_bytes(128);
    e = cudaFuncSetAttribute(gdn2_fwd_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gdn2_fwd_tc_kernel<128><<<fp.B * fp.H, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdelta
