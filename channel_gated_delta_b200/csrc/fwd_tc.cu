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
constexpr float kSpanMax = 12.f;
constexpr int kThreads = 256;

// shared-memory map (bytes); tiles are 1024-byte aligned
template <int DVC>
struct Smem {
    static constexpr int AP = 0;                          // [Kp | W' ; Qp]  128 x 128
    static constexpr int BP = AP + 128 * 256;             // [Kc ; K^c]      128 x 128
    static constexpr int TI = BP + 128 * 256;             // T^-1             64 x 64
    static constexpr int MM = TI + 64 * 128;              // M                64 x 64
    static constexpr int ANAB = MM + 64 * 128;            // [N ; Aq ; Bq]   192 x 64
    static constexpr int VH = ANAB + 192 * 128;           // V^               64 x DVC
    static constexpr int SC = VH + 64 * 2 * DVC;          // S_c             128 x DVC
    static constexpr int RR = SC + 128 * 2 * DVC;         // R                64 x DVC
    static constexpr int LAF = RR + 64 * 2 * DVC;         // fp32 Lambda [64][128]; later L/T^-1 [64][65] + Y
    static constexpr int VEC = LAF + 64 * 128 * 4;        // fp32 vectors
    static constexpr int nvec = 8 * 128;
    static constexpr int PART = VEC + nvec * 4;           // fp32 [64][2] RMS partial sums
    static constexpr int MISC = PART + 64 * 2 * 4;        // mbarrier, TMEM slot, flags
    static constexpr int TOTAL = MISC + 64;
};

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
};

__device__ __forceinline__ void ld_bf16x8(const __nv_bfloat16 *p, float (&f)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    return make_uint4(tc::pack_half2(f[0], f[1]), tc::pack_half2(f[2], f[3]), tc::pack_half2(f[4], f[5]),
                      tc::pack_half2(f[6], f[7]));
}

__device__ __forceinline__ float max8abs(const float *f) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
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
    constexpr int DV = 128;                       // full value width of a head
    const int dv0 = 0;                            // first value column of this CTA

    float *laf = (float *)(sm + L::LAF);
    float *vec = (float *)(sm + L::VEC);
    float *cvec = vec, *ecv = vec + 128, *fcv = vec + 256, *fprev = vec + 384, *gsv = vec + 512;
    float *spanred = vec + 640;                   // [4 warps][8]
    float *diagq = vec + 768, *diagb = vec + 896; // exact q~_t.k_t and q~_t.(b*k)_t
    float *part = (float *)(sm + L::PART);
    uint64_t *mbar = (uint64_t *)(sm + L::MISC);
    uint32_t *tslot = (uint32_t *)(sm + L::MISC + 8);
    int *flags = (int *)(sm + L::MISC + 16);      // [0] abort, [1] chosen n, [2] range
    const uint32_t s_ap = tc::smem_u32(sm + L::AP), s_bp = tc::smem_u32(sm + L::BP);
    const uint32_t s_ti = tc::smem_u32(sm + L::TI), s_mm = tc::smem_u32(sm + L::MM);
    const uint32_t s_anab = tc::smem_u32(sm + L::ANAB), s_vh = tc::smem_u32(sm + L::VH);
    const uint32_t s_sc = tc::smem_u32(sm + L::SC), s_rr = tc::smem_u32(sm + L::RR);
    const uint32_t s_mbar = tc::smem_u32(mbar);

    // ---- set-up: TMEM, mbarrier, per-head vectors
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_u32(tslot), 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(s_mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
        flags[2] = 0;
    }
    if (tid < kDK) {
        gsv[tid] = p.gs ? p.gs[(size_t)h * kDK + tid] : 1.f;
        fprev[tid] = 1.f;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tslot;
    uint32_t phase = 0;
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

    const size_t sbase = (size_t)head * kDK * DV;
    bool first = true;
    for (int t0 = 0; t0 < T;) {
        // ---- A: cumulative log-decay, span, chunk length
        for (int e = tid; e < kC * kDK / 4; e += kThreads) {
            const int t = e / (kDK / 4), c4 = e % (kDK / 4);
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t0 + t < T) x = __ldg(reinterpret_cast<const float4 *>(p.la + (((size_t)bb * T + t0 + t) * H + h) * kDK) + c4);
            reinterpret_cast<float4 *>(laf)[e] = x;
        }
        __syncthreads();
        if (tid < kDK) {
            float acc = 0.f, first_lam = 0.f;
            float sp[7];
            for (int t = 0; t < kC; ++t) {
                acc += laf[t * kDK + tid];
                laf[t * kDK + tid] = acc;
                if (t == 0) first_lam = acc;
                // span of a chunk of length 2^j ending at t = 2^j - 1
                if (t == 0) sp[0] = 0.f;
                if (t == 1) sp[1] = first_lam - acc;
                if (t == 3) sp[2] = first_lam - acc;
                if (t == 7) sp[3] = first_lam - acc;
                if (t == 15) sp[4] = first_lam - acc;
                if (t == 31) sp[5] = first_lam - acc;
                if (t == 63) sp[6] = first_lam - acc;
            }
#pragma unroll
            for (int j = 0; j < 7; ++j) {
                float m = sp[j];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) spanred[warp * 8 + j] = m;
            }
        }
        __syncthreads();
        if (tid == 0) {
            int n = 1;
            for (int j = 6; j >= 0; --j) {
                const float m = fmaxf(fmaxf(spanred[j], spanred[8 + j]), fmaxf(spanred[16 + j], spanred[24 + j]));
                if (m <= kSpanMax) { n = 1 << j; break; }
            }
            flags[1] = min(n, T - t0);
        }
        __syncthreads();
        const int n = flags[1];
        if (tid < kDK) {
            const float l0 = laf[tid], ln = laf[(n - 1) * kDK + tid];
            for (int t = n; t < kC; ++t) laf[t * kDK + tid] = ln;      // identity padding
            const float c = 0.5f * (l0 + ln);
            cvec[tid] = c;
            ecv[tid] = __expf(c);
            fcv[tid] = __expf(ln - c);
        }
        __syncthreads();

        // ---- B: operand tiles (fp16, swizzled)
        for (int u = tid; u < kC * 16; u += kThreads) {
            const int t = u >> 4, g8 = u & 15;
            float kk[8], qq[8], zz[8], bv[8];
            if (t < n) {
                const size_t gi = (((size_t)bb * T + t0 + t) * H + h) * kDK + 8 * g8;
                ld_bf16x8(p.k + gi, kk);
                ld_bf16x8(p.q + gi, qq);
                ld_bf16x8(p.z + gi, zz);
                ld_bf16x8(p.b + gi, bv);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) kk[i] = qq[i] = zz[i] = bv[i] = 0.f;
            }
            float kp[8], kc[8], khc[8], qp[8];
            float dq = 0.f, db = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int ch = 8 * g8 + i;
                const float d = laf[t * kDK + ch] - cvec[ch];
                const float ep = __expf(d), em = __expf(-d);
                const float qt = qq[i] * gsv[ch] * (2.f / (1.f + __expf(-zz[i])));
                const float kh = bv[i] * kk[i];
                dq += qt * kk[i];
                db += qt * kh;
                kp[i] = kk[i] * ep;
                kc[i] = kk[i] * em;
                khc[i] = kh * em;
                qp[i] = qt * ep;
            }
            // The diagonal of Aq / Bq carries no decay; it is taken exactly in
            // fp32 (a readout whose q~.k nearly cancels, e.g. the first token
            // of a sequence, is then free of fp16 operand rounding).
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) {
                dq += __shfl_xor_sync(0xffffffffu, dq, o);
                db += __shfl_xor_sync(0xffffffffu, db, o);
            }
            if (g8 == 0) {
                diagq[t] = dq;
                diagb[t] = db;
            }
            range_max = fmaxf(range_max, fmaxf(fmaxf(max8abs(kp), max8abs(kc)), fmaxf(max8abs(khc), max8abs(qp))));
            *(uint4 *)(sm + L::AP + tc::tile_chunk_off(128, t, g8)) = pack8(kp);
            *(uint4 *)(sm + L::AP + tc::tile_chunk_off(128, 64 + t, g8)) = pack8(qp);
            *(uint4 *)(sm + L::BP + tc::tile_chunk_off(128, t, g8)) = pack8(kc);
            *(uint4 *)(sm + L::BP + tc::tile_chunk_off(128, 64 + t, g8)) = pack8(khc);
        }
        for (int u = tid; u < kC * (DVC / 8); u += kThreads) {
            const int t = u / (DVC / 8), g8 = u % (DVC / 8);
            float vv[8], ww[8];
            if (t < n) {
                const size_t gi = (((size_t)bb * T + t0 + t) * H + h) * DV + dv0 + 8 * g8;
                ld_bf16x8(p.v + gi, vv);
                ld_bf16x8(p.w + gi, ww);
#pragma unroll
                for (int i = 0; i < 8; ++i) vv[i] *= ww[i];
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) vv[i] = 0.f;
            }
            *(uint4 *)(sm + L::VH + tc::tile_chunk_off(64, t, g8)) = pack8(vv);
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
            float *lw = laf;                       // [64][65]
            // rows 0-63: warps 0,1 (M, cols 0-63) and warps 4,5 (L, cols 64-127)
            // rows 64-127: warps 2,3 (Aq) and warps 6,7 (Bq)
            const int t = row & 63;
            const bool upper = row < 64;
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tc::tmem_ld32(tmem + lane_base + kTmP + 64 * colhalf + 32 * half, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int s = 32 * half + i;
                    const bool keep = upper ? (s < t) : (s <= t);
                    if (!keep) v[i] = 0.f;
                    if (!upper && s == t) v[i] = colhalf == 0 ? diagq[t] : diagb[t];
                }
                if (upper && colhalf == 1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) lw[t * 65 + 32 * half + i] = v[i];
                } else {
                    uint8_t *tile = upper ? sm + L::MM : sm + L::ANAB;
                    const int R = upper ? 64 : 192;
                    const int r = upper ? t : (colhalf == 0 ? 64 + t : 128 + t);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = v[8 * q4 + i];
                        *(uint4 *)(tile + tc::tile_chunk_off(R, r, 4 * half + q4)) = pack8(f);
                    }
                }
            }
        }
        tc::fence_before_sync();
        __syncthreads();

        // ---- E: T^-1 = (I + L)^-1 in place, divide and conquer (fp32)
        {
            float *lw = laf;
            float *ybuf = laf + 64 * 65;
            // leaves of 8: forward substitution per column
            float x[8];
            const int leaf = tid >> 3, j = tid & 7, o = 8 * leaf;
            if (tid < 64) {
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
                for (int i = 1; i < 8; ++i) {
                    if (i > j) {
                        float acc = 0.f;
                        for (int s = j; s < i; ++s) acc += lw[(o + i) * 65 + o + s] * x[s];
                        x[i] = -acc;
                    }
                }
            }
            __syncthreads();
            if (tid < 64) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i >= j) lw[(o + i) * 65 + o + j] = x[i];
            }
            __syncthreads();
            // merges: [[A, 0], [C, D]]^-1 = [[A^-1, 0], [-D^-1 C A^-1, D^-1]]
            for (int bs = 8; bs < 64; bs *= 2) {
                const int npairs = 64 / (2 * bs), per = bs * bs;
                for (int e = tid; e < npairs * per; e += kThreads) {
                    const int pr = e / per, i = (e % per) / bs, jj = e % bs, oo = 2 * bs * pr;
                    float acc = 0.f;
                    for (int s = jj; s < bs; ++s) acc += lw[(oo + bs + i) * 65 + oo + s] * lw[(oo + s) * 65 + oo + jj];
                    ybuf[e] = acc;
                }
                __syncthreads();
                for (int e = tid; e < npairs * per; e += kThreads) {
                    const int pr = e / per, i = (e % per) / bs, jj = e % bs, oo = 2 * bs * pr;
                    float acc = 0.f;
                    for (int s = 0; s <= i; ++s) acc += lw[(oo + bs + i) * 65 + oo + bs + s] * ybuf[pr * per + s * bs + jj];
                    lw[(oo + bs + i) * 65 + oo + jj] = -acc;
                }
                __syncthreads();
            }
            // T^-1 -> fp16 tile (row t, column s)
            for (int u = tid; u < 64 * 8; u += kThreads) {
                const int t = u >> 3, g8 = u & 7;
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int s = 8 * g8 + i;
                    f[i] = (s <= t) ? lw[t * 65 + s] : 0.f;
                }
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
            // warps 0-3: W' columns 0-63 and N; warps 4-7: W' columns 64-127
            for (int cblk = 0; cblk < 2; ++cblk) {
                float v[32];
                const int col = 64 * colhalf + 32 * cblk;
                tc::tmem_ld32(tmem + lane_base + kTmW + col, v);
                if (valid) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = v[8 * q4 + i];
                        range_max = fmaxf(range_max, max8abs(f));
                        *(uint4 *)(sm + L::AP + tc::tile_chunk_off(128, t, col / 8 + q4)) = pack8(f);
                    }
                }
            }
            if (colhalf == 0) {
                for (int cblk = 0; cblk < 2; ++cblk) {
                    float v[32];
                    tc::tmem_ld32(tmem + lane_base + kTmN + 32 * cblk, v);
                    if (valid) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) f[i] = v[8 * q4 + i];
                            range_max = fmaxf(range_max, max8abs(f));
                            *(uint4 *)(sm + L::ANAB + tc::tile_chunk_off(192, t, 4 * cblk + q4)) = pack8(f);
                        }
                    }
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
                        const float4 *src = reinterpret_cast<const float4 *>(p.S_in + sbase + (size_t)i * DV + dv0 + col);
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
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = v[8 * q4 + e];
                    range_max = fmaxf(range_max, max8abs(f));
                    *(uint4 *)(sm + L::SC + tc::tile_chunk_off(128, i, col / 8 + q4)) = pack8(f);
                }
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
            for (int cblk = 0; cblk < DVC / 64; ++cblk) {
                const int col = (DVC / 2) * colhalf + 32 * cblk;
                float v[32];
                tc::tmem_ld32(tmem + lane_base + kTmP + col, v);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = v[8 * q4 + e];
                    range_max = fmaxf(range_max, max8abs(f));
                    *(uint4 *)(sm + L::RR + tc::tile_chunk_off(64, row, col / 8 + q4)) = pack8(f);
                }
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

        // ---- L: O (rows 64-127) -> RMSNorm over the head's d_v, gate, store
        {
            const bool orow = row >= 64;
            const int t = row - 64;
            float ov[DVC / 2];
            float ss = 0.f;
            if (orow) {
                for (int cblk = 0; cblk < DVC / 64; ++cblk) {
                    float v[32];
                    tc::tmem_ld32(tmem + lane_base + kTmP + (DVC / 2) * colhalf + 32 * cblk, v);
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        ov[32 * cblk + q] = v[q];
                        ss += v[q] * v[q];
                    }
                }
                part[t * 2 + colhalf] = ss;
            }
            __syncthreads();
            if (orow && t < n) {
                const float tot = part[t * 2] + part[t * 2 + 1];
                const float inv = rsqrtf(tot / DV + p.eps);
                const size_t gi = (((size_t)bb * T + t0 + t) * H + h) * DV + dv0 + (DVC / 2) * colhalf;
                for (int q8 = 0; q8 < DVC / 16; ++q8) {
                    float gg[8], yy[8];
                    ld_bf16x8(p.g + gi + 8 * q8, gg);
#pragma unroll
                    for (int e = 0; e < 8; ++e) yy[e] = gg[e] * ov[8 * q8 + e] * inv;
                    uint4 u;
                    __nv_bfloat162 *hb = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) hb[e] = __floats2bfloat162_rn(yy[2 * e], yy[2 * e + 1]);
                    *reinterpret_cast<uint4 *>(p.y + gi + 8 * q8) = u;
                    if (p.o_raw) {
                        float4 *dst = reinterpret_cast<float4 *>(p.o_raw + gi + 8 * q8);
                        dst[0] = make_float4(ov[8 * q8], ov[8 * q8 + 1], ov[8 * q8 + 2], ov[8 * q8 + 3]);
                        dst[1] = make_float4(ov[8 * q8 + 4], ov[8 * q8 + 5], ov[8 * q8 + 6], ov[8 * q8 + 7]);
                    }
                }
            }
            if (tid < kDK) fprev[tid] = fcv[tid];
        }
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        t0 += n;
    }

    // ---- S_out = Diag(f) X
    if (flags[0] == 0 && p.S_out) {
        const int i = row;
        for (int cblk = 0; cblk < DVC / 64; ++cblk) {
            const int col = (DVC / 2) * colhalf + 32 * cblk;
            float v[32];
            if (T > 0) {
                tc::tmem_ld32(tmem + lane_base + kTmX + col, v);
            }
            float4 *dst = reinterpret_cast<float4 *>(p.S_out + sbase + (size_t)i * DV + dv0 + col);
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

size_t fwd_tc_smem_bytes(int dvc) {
    return (dvc == 128 ? (size_t)Smem<128>::TOTAL : (size_t)Smem<64>::TOTAL) + 1024;
}

bool fwd_tc_supported(int dtype, int dk, int dv, int chunk) {
    return dtype == GDELTA_BF16 && dk == 128 && dv == 128 && chunk == 64;
}

cudaError_t launch_fwd_tc(const FwdParams &fp, cudaStream_t stream) {
    TcParams p;
    p.B = fp.B; p.T = fp.T; p.H = fp.H;
    p.q = (const __nv_bfloat16 *)fp.q; p.k = (const __nv_bfloat16 *)fp.k; p.z = (const __nv_bfloat16 *)fp.z;
    p.b = (const __nv_bfloat16 *)fp.b; p.v = (const __nv_bfloat16 *)fp.v; p.w = (const __nv_bfloat16 *)fp.w;
    p.g = (const __nv_bfloat16 *)fp.g;
    p.la = fp.la; p.gs = fp.gs; p.S_in = fp.S_in; p.S_out = fp.S_out;
    p.y = (__nv_bfloat16 *)fp.y; p.o_raw = fp.o_raw; p.eps = fp.eps; p.status = fp.status;
    const size_t smem = fwd_tc_smem_bytes(128);
    cudaError_t e = cudaFuncSetAttribute(gdn2_fwd_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    gdn2_fwd_tc_kernel<128><<<fp.B * fp.H, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdelta
