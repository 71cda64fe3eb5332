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
#include <cuda.h>
#include <cstring>
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
constexpr int kChainThreads = 384;   // chain kernel: 8 state warps, 2 idle, 2 readout warps
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

// Chain-kernel shared-memory map (bytes; tiles 1024-byte aligned).  Two window
// buffers, each holding one window record in the record's own byte layout
// (V^ restricted to this CTA's 64 value columns): while window w runs from one
// buffer, the record of window w+1 is already arriving in the other.  A window
// processed in shorter chunks (decay span too large for one 64-token chunk)
// builds its tiles in its own buffer and uses the other one as scratch.
struct ChainSmem {
    static constexpr int AP = 0;                         // [W' ; Qp] (shorter chunks: [Kp ; Qp]) 128 x 128 fp16
    static constexpr int BP = AP + 128 * 256;            // [Kc ; K^c]                            128 x 128
    static constexpr int ANAB = BP + 128 * 256;          // [N ; Aq ; Bq]                         192 x 64
    static constexpr int VH = ANAB + 192 * 128;          // V^, this CTA's value columns           64 x 64
    static constexpr int EV = VH + 64 * 128;             // fp32 e^c [128], e^{Lambda_{n-1} - c} [128]
    static constexpr int BUF = EV + 1024;                // one window buffer
    // scratch of the shorter-chunk path, inside the other window buffer
    static constexpr int TI = 0;                         // T^-1  64 x 64 fp16
    static constexpr int MM = TI + 64 * 128;             // M     64 x 64 fp16
    static constexpr int LW = MM + 64 * 128;             // fp32 L, then T^-1   [64][kLW]
    static constexpr int YB = LW + 64 * kLW * 4;         // fp32 merge buffer   [32][kYS]
    static constexpr int WT = YB + 32 * kYS * 4;         // fp32 per-warp log-decay totals [8][128]
    static constexpr int PR = WT + 8 * 128 * 4;          // fp32 Lambda at the probe tokens [7][128]
    static constexpr int XV = PR + 8 * 128 * 4;          // fp32 span maxima [64], exact diagonals [2][64]
    static_assert(XV + 192 * 4 <= BUF, "shorter-chunk scratch fits in a window buffer");
    // shared by all windows
    static constexpr int SC = 2 * BUF;                   // S_c  128 x 64 fp16
    static constexpr int RR = SC + 128 * 128;            // R     64 x 64 fp16
    static constexpr int VEC = RR + 64 * 128;            // fp32 fprev [128], gamma_stat [128]
    static constexpr int PART = VEC + 256 * 4;           // fp32 peer's row sums [2][64], int peer flags [2]
    static constexpr int MISC = PART + 1536;             // 11 mbarriers, TMEM slot, flags, chunk info
    static constexpr int TOTAL = MISC + 256;
};

// Per-window record written by the intra kernel: the chunk's operand tiles in
// the exact shared-memory byte layout the chain kernel uses, then the pivot
// vectors e^c and e^{Lambda_{n-1} - c} (fp32, 128 each).
constexpr int kWinAP = 0;                     // [W' ; Qp]       128 x 128 fp16
constexpr int kWinBP = kWinAP + 128 * 256;    // [Kc ; K^c]      128 x 128
constexpr int kWinANAB = kWinBP + 128 * 256;  // [N ; Aq ; Bq]   192 x 64
constexpr int kWinVH = kWinANAB + 192 * 128;  // V^               64 x 128
constexpr int kWinVEC = kWinVH + 64 * 256;    // e^c, e^{Lambda_{n-1} - c}
constexpr int kWinBytes = kWinVEC + 1024;
static_assert(kWinVH % 32 == 0, "the shared tiles split into two 16-byte-multiple halves");
#ifndef GDN2_REC_PREFETCH
#define GDN2_REC_PREFETCH 4
#endif
// The chain kernel copies a window's record two windows ahead and prefetches
// the record this many windows ahead into L2 (0 = no prefetch).
constexpr int kRecPrefetch = GDN2_REC_PREFETCH;

// Chain-kernel TMEM columns
constexpr uint32_t kTmP = 0;       // shorter chunks: P (128 x 128)
constexpr uint32_t kTmW = 128;     // shorter chunks: W' (M=64, 128 columns)
constexpr uint32_t kTmN = 256;     // shorter chunks: N  (M=64, 64 columns)
constexpr uint32_t kTmX = 320;     // state accumulator X (128 x 64)
constexpr uint32_t kTmRO = 384;    // [R; O] (128 x 64)
constexpr int kDVC = 64;           // value columns per chain CTA; a cluster of two covers d_v = 128

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
    const __nv_bfloat16 *beta;   // one gate per token and head standing for both b and w, or null
    int decay_tok;               // 1: la holds one log-decay per token and head
    int qk_raw;                  // 1: q and k need SiLU and l2 normalisation
    int NW;                  // windows of 64 tokens per head
    uint32_t spin;           // polls before a bounded wait on another party gives up
    int stall;               // 1: wait first on a barrier nothing completes, so that the wait runs out
};

// Polls of a wait for this CTA's own asynchronous work (bulk copies, MMAs)
// before the CTA leaves or frees TMEM: independent of the configurable limit,
// so that a small limit never lets a CTA exit with a copy or MMA in flight.
constexpr uint32_t kDrainPolls = 1u << 22;

__device__ __forceinline__ void bf16x8_to_f(const uint4 &u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

// Key/query preprocessing on one token row held by a whole warp (four channels
// a lane, 128 in all): SiLU, division by the row's l2 norm (floored at 1e-12),
// and rounding to bf16 as a separate normalisation would store the result.
// Every lane of the warp must call it (full-warp shuffles).
__device__ __forceinline__ void silu_l2n_row4(float (&f)[4]) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[i] *= 0.5f * two_sigmoid_fast(f[i]);
        ss = fmaf(f[i], f[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(fmaxf(ss, 1e-24f));
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __bfloat162float(__float2bfloat16_rn(f[i] * inv));
}

// A gate given once per token and head, repeated over four channels as a bf16 quad.
__device__ __forceinline__ uint2 bf16x4_bcast(const __nv_bfloat16 *p, size_t i) {
    const uint32_t x = __ldg(reinterpret_cast<const unsigned short *>(p) + i);
    return make_uint2(x | (x << 16), x | (x << 16));
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

// Barrier of warps 0-7 (named barrier 1): the whole intra-kernel CTA, the
// state warps of the chain kernel.
__device__ __forceinline__ void main_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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
    main_sync();
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
    main_sync();
}

}  // namespace

// ---------------------------------------------------------------------------
// Chain kernel: a cluster of two CTAs per (batch, head); CTA r owns value
// columns [64 r, 64 r + 64) of the state, which stays in TMEM (fp32) for the
// whole sequence.  Value columns of the recurrence are independent, so the
// two CTAs share nothing but the RMS norm of the readout: per chunk they
// exchange per-token sums of squares through distributed shared memory.
// Windows whose tiles the intra kernel precomputed are bulk-copied one window
// ahead; a flagged window (decay span too large for one 64-token chunk) is
// processed here in shorter chunks.
//
// Warp roles: warps 0-7 run the state recurrence (operand staging, MMA issue,
// R readout); warps 10-11 (TMEM lanes 64-127, the readout rows) take each
// chunk's O out of TMEM and run the RMS exchange, gate and stores while the
// state recurrence moves on to the next chunk.  [R; O] alternates between two
// TMEM slots; warps 8-9 have no role.
// ---------------------------------------------------------------------------
// kRaw: q and k arrive before their SiLU and l2 normalisation (read only by the
// shorter-chunk path; window records hold the preprocessed operands).
template <bool kRaw>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kChainThreads, 1) gdn2_fwd_tc_kernel(TcParams p) {
    using L = ChainSmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = tc::cluster_ctarank();
    const int head = blockIdx.x >> 1;            // b * H + h
    const int bb = head / p.H, h = head % p.H;
    const int T = p.T, H = p.H;
    const int dv0 = kDVC * (int)crank;           // first value column of this CTA

    float *fprev = (float *)(sm + L::VEC), *gsv = fprev + 128;
    // mbarriers: [0] MMA, [1..2] record buffers, [3..4] exchange slots, [5..6] chunk info,
    // [7..8] O ready, [9..10] O slot free
    uint64_t *mbar = (uint64_t *)(sm + L::MISC);
    uint32_t *tslot = (uint32_t *)(sm + L::MISC + 88);
    float *peer = (float *)(sm + L::PART);        // [2][64] the peer's per-row sums
    int *pflag = (int *)(sm + L::PART + 512);     // [2] the peer's abort flags
    volatile int *flags = (volatile int *)(sm + L::MISC + 96);  // [0] local abort, [1] chosen n, [2] log2 of the chunk, [3] agreed abort
    int *info = (int *)(sm + L::MISC + 112);      // per O slot: t0, n, done
    volatile int *req = (volatile int *)(sm + L::MISC + 176);  // record requests: [2] x (window, buffer)
    const uint32_t s_mbar = tc::smem_u32(mbar), s_rbar = s_mbar + 8, s_xbar = s_mbar + 24;
    const uint32_t s_ibar = s_mbar + 40, s_obar = s_mbar + 56, s_fbar = s_mbar + 72;
    const uint32_t s_lq = s_mbar + 144, s_lfree = s_mbar + 160;  // record request posted / slot read
    const uint32_t s_stall = s_mbar + 192;                         // never completed (failure-path tests)
    const uint32_t peer_rank = crank ^ 1u;
    const uint32_t r_peer = tc::mapa(tc::smem_u32(peer), peer_rank);
    const uint32_t r_pflag = tc::mapa(tc::smem_u32(pflag), peer_rank);
    const uint32_t r_xbar = tc::mapa(s_xbar, peer_rank);
    const uint32_t s_sc = tc::smem_u32(sm + L::SC), s_rr = tc::smem_u32(sm + L::RR);

    // ---- set-up: TMEM, mbarriers, per-head vectors; the peer's barriers exist before first use
    if (warp == 0) {
        tc::tmem_alloc(tc::smem_u32(tslot), 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 11; ++i) tc::mbar_init(s_mbar + 8 * i, 1);
        for (int i = 0; i < 4; ++i) tc::mbar_init(s_lq + 8 * i, 1);
        tc::mbar_init(s_stall, 1);
        tc::mbar_arrive_expect_tx(s_xbar, 65 * 4);   // the peer's sums of chunk 0 (64 rows and a flag)
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
        flags[3] = 0;
        pflag[0] = pflag[1] = 0;
    }
    if (tid < kDK) {
        gsv[tid] = p.gs ? p.gs[(size_t)h * kDK + tid] : 1.f;
        fprev[tid] = 1.f;
    }
    tc::fence_before_sync();
    tc::cluster_sync();
    tc::fence_after_sync();
    // launched as a programmatic dependent of the intra kernel: the set-up above
    // may overlap that kernel's last CTAs; its records and flags are read only
    // after this wait (a hardware wait for the whole prerequisite grid)
    tc::grid_dependency_wait();
    const uint32_t tmem = *tslot;
    uint32_t phase = 0;
    uint32_t rph = 0u;                           // bit b: parity of record buffer b's next copy
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's TMEM lanes
    const int row = 32 * (warp & 3) + lane;                         // accumulator row (M = 128)
    const int colhalf = warp >> 2;                                  // 32-column half of this CTA's 64
    float range_max = 0.f;

    const int NW = p.NW;
    const size_t wbase = (size_t)head * NW;
    // Record copies are issued by one lane of warp 8, which executes no proxy
    // fence: a thread that has bulk copies in flight and then fences the async
    // proxy (as the state warps do after staging operand tiles) waits for those
    // copies, which would tie every window to the record two windows ahead.
    // Window wp's record into L2; the two CTAs of the cluster split the shared
    // tiles between them and each fetches its own half of V^.
    auto prefetch_rec = [&](int wp) {
        const uint8_t *pf = p.ws + (wbase + wp) * kWinBytes;
        const uint32_t half = (uint32_t)kWinVH / 2;
        tc::bulk_prefetch_l2(pf + crank * half, half);
        tc::bulk_prefetch_l2(pf + kWinVH + crank * (64 * 128), 64 * 128);
        if (crank == 0) tc::bulk_prefetch_l2(pf + kWinVEC, 2 * 128 * 4);
    };
    auto issue_rec = [&](int w, int b) {         // window w's record -> buffer b
        const uint8_t *rec = p.ws + (wbase + w) * kWinBytes;
        uint8_t *dst = sm + b * L::BUF;
        const uint32_t bar = s_rbar + 8u * b;
        tc::mbar_arrive_expect_tx(bar, L::BUF);
        tc::bulk_g2s(tc::smem_u32(dst + L::AP), rec + kWinAP, 128 * 256, bar);
        tc::bulk_g2s(tc::smem_u32(dst + L::BP), rec + kWinBP, 128 * 256, bar);
        tc::bulk_g2s(tc::smem_u32(dst + L::ANAB), rec + kWinANAB, 192 * 128, bar);
        tc::bulk_g2s(tc::smem_u32(dst + L::VH), rec + kWinVH + crank * (64 * 128), 64 * 128, bar);
        tc::bulk_g2s(tc::smem_u32(dst + L::EV), rec + kWinVEC, 2 * 128 * 4, bar);
        // the record kRecPrefetch windows further on is brought into L2 now, so that
        // its copy into shared memory is served from L2 instead of DRAM (the first
        // two copies also cover the windows before that distance)
        if (kRecPrefetch > 2) {
            for (int wp = (w < 2 ? w + 2 : w + kRecPrefetch); wp <= w + kRecPrefetch; wp += 2)
                if (wp < NW) prefetch_rec(wp);
        }
    };
    static_assert(L::BUF == 2 * 128 * 256 + 192 * 128 + 64 * 128 + 1024, "record buffer = bytes of one record copy");

    int mma_pending = -1;                         // parity of an MMA commit whose wait ran out
    if (warp < 8) {
        // Wait for the MMAs committed so far; a timeout marks a local abort (the
        // commit is drained before TMEM is freed).
        auto wait_mma = [&]() -> bool {
            if (!tc::mbar_wait(s_mbar, phase, p.spin)) {
                flags[0] = 1;
                mma_pending = (int)phase;
            }
            phase ^= 1u;
            main_sync();
            tc::fence_after_sync();
            return flags[0] == 0;
        };

        auto win_fast = [&](int w) -> bool { return p.ws != nullptr && w < NW && p.wflags[wbase + w] == 0; };
        // Thread kAux (warp 2, lane 0; its warp holds no R rows) keeps thread 0, the
        // MMA issuer, free of everything else: it posts every record request
        // (window w into buffer b; w < 0 stops the loader) and checks each chunk's
        // O slot.
        constexpr int kAux = 64;
        uint32_t nreq = 0;
        auto enqueue = [&](int w, int b) {
            const uint32_t k = nreq++, sl = k & 1u;
            if (k >= 2 && !tc::mbar_wait(s_lfree + 8u * sl, ((k >> 1) - 1) & 1u, p.spin)) flags[0] = 1;
            req[2 * sl] = w;
            req[2 * sl + 1] = b;
            tc::mbar_arrive_local(s_lq + 8u * sl);
        };

        // failure-path test: a wait that nothing completes runs out before any work is issued
        if (p.stall) {
            if (tid == 0 && !tc::mbar_wait(s_stall, 0, p.spin)) flags[0] = 1;
            main_sync();
        }
        // Per record buffer b (0 or 1; selected by value, not by index, so that
        // nothing lives in local memory): the window it holds or receives, and
        // whether a copy into it has not been waited for (bit b of infl).
        int loaded0 = -1, loaded1 = -1;
        uint32_t infl = 0u;
        auto loaded_of = [&](int b) -> int { return b ? loaded1 : loaded0; };
        auto set_loaded = [&](int b, int v) {
            if (b) loaded1 = v;
            else loaded0 = v;
        };
        for (int b = 0; b < 2 && flags[0] == 0; ++b)
            if (win_fast(b)) {
                if (tid == kAux) enqueue(b, b);
                set_loaded(b, b);
                infl |= 1u << b;
            }

        const size_t sbase = (size_t)head * kDK * kDV;
        bool first = true;
        int chunk = 0;
        uint32_t uses0 = 0u, uses1 = 0u;                // chunks that used [R; O] slot 0 / 1
        // thread kAux: a record request held back until the next chunk's first MMA
        // group has completed, so that the copy's shared-memory writes do not land
        // during the state rescale
        int pend_w = -1, pend_b = 0;
        for (int w = 0; w < NW && flags[0] == 0; ++w) {
            const int B = w & 1;
            uint8_t *buf = sm + B * L::BUF, *xbuf = sm + (B ^ 1) * L::BUF;
            const uint32_t s_ap = tc::smem_u32(buf + L::AP), s_bp = tc::smem_u32(buf + L::BP);
            const uint32_t s_anab = tc::smem_u32(buf + L::ANAB), s_vh = tc::smem_u32(buf + L::VH);
            float *ecv = (float *)(buf + L::EV), *fcv = ecv + 128;
            const int wend = min(T, kC * (w + 1));
            const bool fast = loaded_of(B) == w;
            // an abort agreed by the readout warps becomes this group's abort at the barrier below
            if (tid == 0 && flags[3] != 0) flags[0] = 1;
            if (fast) {
                if (!tc::mbar_wait(s_rbar + 8u * B, (rph >> B) & 1u, p.spin)) flags[0] = 1;
                rph ^= 1u << B;
                infl &= ~(1u << B);
            } else if ((infl >> (B ^ 1)) & 1u) {
                // the other buffer is this window's scratch: a record arriving there
                // lands first (a request still held back is issued now), and is
                // copied again after the window
                if (tid == kAux && pend_w >= 0) {
                    enqueue(pend_w, pend_b);
                    pend_w = -1;
                }
                if (!tc::mbar_wait(s_rbar + 8u * (B ^ 1), (rph >> (B ^ 1)) & 1u, p.spin)) flags[0] = 1;
                rph ^= 1u << (B ^ 1);
                infl &= ~(1u << (B ^ 1));
            }
            main_sync();
            // The products of one chunk (H to K) on the tiles in `buf`.  Called from two
            // places: a precomputed window is one chunk and takes the first call alone,
            // so its code stays compact; windows processed in shorter chunks build the
            // tiles first (a large block that, placed in line before the products,
            // measured 3 % slower on windows that never use it).
            auto chunk_products = [&](const int t0, const int n) {
                const uint32_t slot = (uint32_t)(chunk & 1);      // TMEM slot of this chunk's [R; O]
                const uint32_t ro = kTmRO + (uint32_t)kDVC * slot;
                ++chunk;
                if (flags[0] == 0) {
                    // ---- H: state operand S_c = Diag(e^c) S, X <- S_c (fp32, TMEM)
                    {
                        const int i = row;                                   // key channel
                        const float scale = ecv[i] * fprev[i];
                        const int col = 32 * colhalf;
                        float v[32];
                        if (first) {
                            if (p.S_in) {
                                const float4 *src =
                                    reinterpret_cast<const float4 *>(p.S_in + sbase + (size_t)i * kDV + dv0 + col);
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
                    if (tid == kAux) {
                        // the slot's previous O has been read out of TMEM (and its chunk
                        // info); the readout warps learn this chunk's tokens now (to fetch
                        // the gate early)
                        const uint32_t us = slot ? uses1 : uses0;
                        if (us > 0 && !tc::mbar_wait(s_fbar + 8u * slot, (us - 1) & 1u, p.spin))
                            flags[0] = 1;
                        info[4 * slot] = t0;
                        info[4 * slot + 1] = n;
                        info[4 * slot + 2] = 0;
                        tc::mbar_arrive_local(s_ibar + 8u * slot);
                    }
                    first = false;
                    tc::fence_proxy_async();
                    tc::fence_before_sync();
                    main_sync();

                    // ---- I: [R; O] = [W'; Qp] S_c + [N; Aq] V^ ;  X += Kc^T V^
                    if (tid == 0) {
                        tc::fence_after_sync();
                        const uint32_t id1 = tc::idesc_f16(128, kDVC, false, true, false);
                        if (flags[0] == 0) {
#pragma unroll
                            for (int ks = 0; ks < kDK / 16; ++ks)
                                tc::mma_f16(tmem + ro, tc::desc_kmajor_step(tc::desc_kmajor(s_ap, 128, 0, 0), 128, ks), tc::desc_mnmajor_step(tc::desc_mnmajor(s_sc, 128, 0, 0), ks),
                                            id1, ks > 0);
#pragma unroll
                            for (int ks = 0; ks < kC / 16; ++ks)
                                tc::mma_f16(tmem + ro, tc::desc_kmajor_step(tc::desc_kmajor(s_anab, 192, 0, 0), 192, ks), tc::desc_mnmajor_step(tc::desc_mnmajor(s_vh, 64, 0, 0), ks),
                                            id1, true);
                        }
                        tc::mma_commit(s_mbar);                   // [R; O]: R is read out next
                        // the state's V^ term runs on the tensor core while R is read out
                        // (the next commit covers it)
                        const uint32_t id2 = tc::idesc_f16(128, kDVC, true, true, false);
                        if (flags[0] == 0)
#pragma unroll
                            for (int ks = 0; ks < kC / 16; ++ks)
                                tc::mma_f16(tmem + kTmX, tc::desc_mnmajor_step(tc::desc_mnmajor(s_bp, 128, 0, 0), ks), tc::desc_mnmajor_step(tc::desc_mnmajor(s_vh, 64, 0, 0), ks),
                                            id2, true);
                    }
                }
                if (flags[0] == 0 && wait_mma()) {
                    // a held-back record request (kAux's warp has no R rows below)
                    if (tid == kAux && pend_w >= 0) {
                        enqueue(pend_w, pend_b);
                        pend_w = -1;
                    }
                    // ---- J: R (rows 0-63) -> fp16 tile
                    if (row < 64) {
                        float v[32];
                        tc::tmem_ld32(tmem + lane_base + ro + 32 * colhalf, v);
                        range_max = fmaxf(range_max, maxabs(v, 32));
                        store_row32(sm + L::RR, 64, row, 32 * colhalf, v);
                    }
                    tc::fence_proxy_async();
                    tc::fence_before_sync();
                    main_sync();

                    // ---- K: O -= Bq R (rows 64-127; rows 0-63 receive -Aq R, unused);  X -= K^c^T R
                    if (tid == 0) {
                        tc::fence_after_sync();
                        const uint32_t id1 = tc::idesc_f16(128, kDVC, false, true, true);
#pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            tc::mma_f16(tmem + ro, tc::desc_kmajor_step(tc::desc_kmajor(s_anab, 192, 64, 0), 192, ks), tc::desc_mnmajor_step(tc::desc_mnmajor(s_rr, 64, 0, 0), ks),
                                        id1, true);
                        const uint32_t id2 = tc::idesc_f16(128, kDVC, true, true, true);
#pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            tc::mma_f16(tmem + kTmX, tc::desc_mnmajor_step(tc::desc_mnmajor(s_bp, 128, 64, 0), ks), tc::desc_mnmajor_step(tc::desc_mnmajor(s_rr, 64, 0, 0), ks),
                                        id2, true);
                        tc::mma_commit(s_mbar);
                        tc::mma_commit(s_obar + 8u * slot);      // O of this chunk is final
                    }
                    // tile flag of window w + 2, loaded while every thread waits for the
                    // MMAs (loaded at the top of the window, its first use stalled there)
                    const int wflag2 = (p.ws != nullptr && w + 2 < NW) ? __ldg(p.wflags + wbase + w + 2) : 1;
                    if (wait_mma()) {
                        // the chunk's tiles are free: keep its decay factor; once the window's
                        // last chunk is done, its buffer takes the record of window w + 2
                        if (tid < kDK) fprev[tid] = fcv[tid];
                        main_sync();
                        if (t0 + n == wend) {
                            if (wflag2 == 0) {
                                if (tid == kAux) {
                                    pend_w = w + 2;
                                    pend_b = B;
                                }
                                set_loaded(B, w + 2);
                                infl |= 1u << B;
                            } else {
                                set_loaded(B, -1);
                            }
                        }
                    }
                }

                tc::fence_before_sync();
                main_sync();
                tc::fence_after_sync();
                if (slot) ++uses1;
                else ++uses0;
            };
            if (fast) {
                if (flags[0] == 0) chunk_products(kC * w, wend - kC * w);
            } else {
                for (int t0 = kC * w; t0 < wend && flags[0] == 0;) {
                    int n = wend - t0;
                    if (flags[0] == 0) do {
                        // ---- A: loads, cumulative log-decay, span, chunk length.
                        // Warp w owns tokens [8w, 8w+8); lane l owns key channels [4l, 4l+4)
                        // and, for l < 16, value channels dv0 + [4l, 4l+4).
                        float *wtot = (float *)(xbuf + L::WT), *probe = (float *)(xbuf + L::PR);
                        float *spanred = (float *)(xbuf + L::XV), *diagq = spanred + 64, *diagb = spanred + 128;
                        float *lw = (float *)(xbuf + L::LW), *yb = (float *)(xbuf + L::YB);
                        const uint32_t s_ti = tc::smem_u32(xbuf + L::TI), s_mm = tc::smem_u32(xbuf + L::MM);
                        const int tb = 8 * warp, c4 = 4 * lane;
                        // token u's inputs, loaded one token ahead of their use below so that a
                        // thread never holds more than two tokens' worth (a register peak here
                        // would make the whole chain kernel spill)
                        auto gt_of = [&](int u) -> size_t { return ((size_t)bb * T + t0 + tb + u) * H + h; };
                        auto load_la = [&](int u) -> float4 {
                            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (t0 + tb + u < wend) {
                                if (p.decay_tok) {
                                    const float sc = __ldg(p.la + gt_of(u));
                                    x = make_float4(sc, sc, sc, sc);
                                } else {
                                    x = __ldg(reinterpret_cast<const float4 *>(p.la + gt_of(u) * kDK + c4));
                                }
                            }
                            return x;
                        };
                        auto load_kq = [&](int u, uint2 (&o)[4]) {        // k, q, z, b: 4 bf16 each
                            const bool in = t0 + tb + u < wend;
                            const size_t gt = gt_of(u), gk = gt * kDK + c4;
                            o[0] = in ? __ldg(reinterpret_cast<const uint2 *>(p.k + gk)) : make_uint2(0, 0);
                            o[1] = in ? __ldg(reinterpret_cast<const uint2 *>(p.q + gk)) : make_uint2(0, 0);
                            o[2] = in && p.z ? __ldg(reinterpret_cast<const uint2 *>(p.z + gk)) : make_uint2(0, 0);
                            o[3] = !in ? make_uint2(0, 0)
                                  : p.beta ? bf16x4_bcast(p.beta, gt) : __ldg(reinterpret_cast<const uint2 *>(p.b + gk));
                        };
                        auto load_vw = [&](int u, uint2 (&o)[2]) {        // v, w of this CTA's value columns
                            const bool in = t0 + tb + u < wend && c4 < kDVC;
                            const size_t gt = gt_of(u), gv = gt * kDV + dv0 + c4;
                            o[0] = in ? __ldg(reinterpret_cast<const uint2 *>(p.v + gv)) : make_uint2(0, 0);
                            o[1] = !in ? make_uint2(0, 0)
                                  : p.beta ? bf16x4_bcast(p.beta, gt) : __ldg(reinterpret_cast<const uint2 *>(p.w + gv));
                        };
                        // inclusive scan over tokens: this warp's sum (and its prefix at tokens
                        // 0, 1, 3 and 7 of the warp, the probe tokens it may own), then across warps
                        float off[4] = {0.f, 0.f, 0.f, 0.f};
                        {
                            float run[4] = {0.f, 0.f, 0.f, 0.f}, pre[4][4];
    #pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const float4 x = load_la(u);
                                run[0] += x.x; run[1] += x.y; run[2] += x.z; run[3] += x.w;
                                const int j = u == 0 ? 0 : u == 1 ? 1 : u == 3 ? 2 : u == 7 ? 3 : -1;
                                if (j >= 0)
    #pragma unroll
                                    for (int c = 0; c < 4; ++c) pre[j][c] = run[c];
                            }
                            *reinterpret_cast<float4 *>(wtot + warp * kDK + c4) = make_float4(run[0], run[1], run[2], run[3]);
                            main_sync();
                            for (int ww = 0; ww < warp; ++ww) {
                                const float4 o4 = *reinterpret_cast<const float4 *>(wtot + ww * kDK + c4);
                                off[0] += o4.x; off[1] += o4.y; off[2] += o4.z; off[3] += o4.w;
                            }
                            // Lambda at tokens 0, 1, 3, 7, 15, 31, 63 (the last token of a chunk of 2^j):
                            // tokens 0-7 are warp 0's, 15 warp 1's, 31 warp 3's, 63 warp 7's last
                            auto put = [&](int j, int k) {
                                *reinterpret_cast<float4 *>(probe + j * kDK + c4) =
                                    make_float4(off[0] + pre[k][0], off[1] + pre[k][1], off[2] + pre[k][2], off[3] + pre[k][3]);
                            };
                            if (warp == 0) {
                                put(0, 0);
                                put(1, 1);
                                put(2, 2);
                                put(3, 3);
                            } else if (warp == 1) {
                                put(4, 3);
                            } else if (warp == 3) {
                                put(5, 3);
                            } else if (warp == 7) {
                                put(6, 3);
                            }
                        }
                        main_sync();
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
                        main_sync();
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
                        const bool vlane = c4 < kDVC;
                        main_sync();
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
                            float lam_run[4] = {off[0], off[1], off[2], off[3]};     // Lambda before token u
                            float4 la_nx = load_la(0);
                            uint2 kq_nx[4];
                            load_kq(0, kq_nx);
    #pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const int t = tb + u;
                                const bool live = t < n;
                                const float4 la_c = la_nx;
                                const uint2 kq_c[4] = {kq_nx[0], kq_nx[1], kq_nx[2], kq_nx[3]};
                                if (u + 1 < 8) {
                                    la_nx = load_la(u + 1);
                                    load_kq(u + 1, kq_nx);
                                }
                                lam_run[0] += la_c.x; lam_run[1] += la_c.y; lam_run[2] += la_c.z; lam_run[3] += la_c.w;
                                float kk[4], qq[4], zz[4], bv[4];
                                {
                                    const __nv_bfloat162 *hk = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[0]);
                                    const __nv_bfloat162 *hq = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[1]);
                                    const __nv_bfloat162 *hz = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[2]);
                                    const __nv_bfloat162 *hb = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[3]);
    #pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        float2 f;
                                        f = __bfloat1622float2(hk[e]); kk[2 * e] = f.x; kk[2 * e + 1] = f.y;
                                        f = __bfloat1622float2(hq[e]); qq[2 * e] = f.x; qq[2 * e + 1] = f.y;
                                        f = __bfloat1622float2(hz[e]); zz[2 * e] = f.x; zz[2 * e + 1] = f.y;
                                        f = __bfloat1622float2(hb[e]); bv[2 * e] = f.x; bv[2 * e + 1] = f.y;
                                    }
                                    if (kRaw) {                 // the q/k preprocessing, one token a call
                                        silu_l2n_row4(kk);
                                        silu_l2n_row4(qq);
                                    }
                                }
                                float kp[4], kc[4], khc[4], qp[4];
                                float dq = 0.f, db = 0.f;
    #pragma unroll
                                for (int c = 0; c < 4; ++c) {
                                    const float lam = live ? lam_run[c] : lnv[c];   // identity padding past n
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
                                *(uint2 *)(buf + L::AP + off_t) = make_uint2(tc::pack_half2(kp[0], kp[1]), tc::pack_half2(kp[2], kp[3]));
                                *(uint2 *)(buf + L::AP + off_b) = make_uint2(tc::pack_half2(qp[0], qp[1]), tc::pack_half2(qp[2], qp[3]));
                                *(uint2 *)(buf + L::BP + off_t) = make_uint2(tc::pack_half2(kc[0], kc[1]), tc::pack_half2(kc[2], kc[3]));
                                *(uint2 *)(buf + L::BP + off_b) =
                                    make_uint2(tc::pack_half2(khc[0], khc[1]), tc::pack_half2(khc[2], khc[3]));
                            }
                            if (vlane) {
                                uint2 vw_nx[2];
                                load_vw(0, vw_nx);
    #pragma unroll
                                for (int u = 0; u < 8; ++u) {
                                    const int t = tb + u;
                                    const bool live = t < n;
                                    const uint2 vw_c[2] = {vw_nx[0], vw_nx[1]};
                                    if (u + 1 < 8) load_vw(u + 1, vw_nx);
                                    const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&vw_c[0]);
                                    const __nv_bfloat162 *hw = reinterpret_cast<const __nv_bfloat162 *>(&vw_c[1]);
                                    float vh[4];
    #pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        const float2 fv = __bfloat1622float2(hv[e]), fw = __bfloat1622float2(hw[e]);
                                        vh[2 * e] = live ? fv.x * fw.x : 0.f;
                                        vh[2 * e + 1] = live ? fv.y * fw.y : 0.f;
                                    }
                                    *(uint2 *)(buf + L::VH + tc::tile_off(64, t, c4)) =
                                        make_uint2(tc::pack_half2(vh[0], vh[1]), tc::pack_half2(vh[2], vh[3]));
                                }
                            }
                        }
                        tc::fence_proxy_async();
                        main_sync();

                        // ---- C: decay-relative products P = [Kp; Qp] [Kc; K^c]^T
                        if (tid == 0) {
                            tc::fence_after_sync();
                            const uint32_t id = tc::idesc_f16(128, 128, false, false, false);
#pragma unroll
                            for (int ks = 0; ks < kDK / 16; ++ks)
                                tc::mma_f16(tmem + kTmP, tc::desc_kmajor_step(tc::desc_kmajor(s_ap, 128, 0, 0), 128, ks), tc::desc_kmajor_step(tc::desc_kmajor(s_bp, 128, 0, 0), 128, ks), id,
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
                                    uint8_t *tile = upper ? xbuf + L::MM : buf + L::ANAB;
                                    const int R = upper ? 64 : 192;
                                    const int r = upper ? t : (colhalf == 0 ? 64 + t : 128 + t);
                                    store_row32(tile, R, r, 32 * hf, v[hf]);
                                }
                            }
                        }
                        tc::fence_before_sync();
                        main_sync();

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
                                asm volatile("bar.sync 2, 64;" ::: "memory");     // the 64 leaf threads only
    #pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    if (i >= j) lw[(o + i) * kLW + o + j] = x[i];
                            }
                            main_sync();
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
                                *(uint4 *)(xbuf + L::TI + tc::tile_chunk_off(64, t, g8)) = pack8(f);
                            }
                        }
                        tc::fence_proxy_async();
                        main_sync();

                        // ---- F: W' = T^-1 Kp, N = T^-1 M
                        if (tid == 0) {
                            tc::fence_after_sync();
                            const uint32_t idw = tc::idesc_f16(64, 128, false, true, false);
                            const uint32_t idn = tc::idesc_f16(64, 64, false, true, false);
#pragma unroll
                            for (int ks = 0; ks < kC / 16; ++ks)
                                tc::mma_f16(tmem + kTmW, tc::desc_kmajor_step(tc::desc_kmajor(s_ti, 64, 0, 0), 64, ks), tc::desc_mnmajor_step(tc::desc_mnmajor(s_ap, 128, 0, 0), ks), idw,
                                            ks > 0);
#pragma unroll
                            for (int ks = 0; ks < kC / 16; ++ks)
                                tc::mma_f16(tmem + kTmN, tc::desc_kmajor_step(tc::desc_kmajor(s_ti, 64, 0, 0), 64, ks), tc::desc_mnmajor_step(tc::desc_mnmajor(s_mm, 64, 0, 0), ks), idn,
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
                            tc::tmem_ld32x2(tmem + lane_base + kTmW + 64 * colhalf, tmem + lane_base + kTmW + 64 * colhalf + 32,
                                            v[0], v[1]);
                            if (valid) {
    #pragma unroll
                                for (int hf = 0; hf < 2; ++hf) {
                                    range_max = fmaxf(range_max, maxabs(v[hf], 32));
                                    store_row32(buf + L::AP, 128, t, 64 * colhalf + 32 * hf, v[hf]);
                                }
                            }
                            // warps 0-3: N columns 0-31; warps 4-7: N columns 32-63
                            float nv[32];
                            tc::tmem_ld32(tmem + lane_base + kTmN + 32 * colhalf, nv);
                            if (valid) {
                                range_max = fmaxf(range_max, maxabs(nv, 32));
                                store_row32(buf + L::ANAB, 192, t, 32 * colhalf, nv);
                            }
                        }
                    } while (false);
                    chunk_products(t0, n);
                    t0 += n;
                }
            }
            // after a window processed in shorter chunks: the record of window w + 1
            // (its scratch buffer) is copied again, and this buffer takes window w + 2
            if (!fast && flags[0] == 0) {
                if (loaded_of(B ^ 1) == w + 1) {
                    if (tid == kAux) enqueue(w + 1, B ^ 1);
                    infl |= 1u << (B ^ 1);
                }
            }
        }

        // no more chunks: tell the readout warps
        if (tid == 0) {
            const uint32_t slot = (uint32_t)(chunk & 1);
            const uint32_t us = slot ? uses1 : uses0;
            if (us > 0) tc::mbar_wait(s_fbar + 8u * slot, (us - 1) & 1u, p.spin);
            info[4 * slot + 2] = 1;
            tc::mbar_arrive_local(s_ibar + 8u * slot);
        }
        if (tid == kAux) {
            if (pend_w >= 0) enqueue(pend_w, pend_b);   // its buffer is marked in flight: the copy is drained below
            enqueue(-1, 0);
        }
        // copies still in flight (the loop ended early) complete before exit
        for (int b = 0; b < 2; ++b)
            if ((infl >> b) & 1u) tc::mbar_wait(s_rbar + 8u * b, (rph >> b) & 1u, kDrainPolls);

        // ---- S_out = Diag(fprev) X
        if (flags[0] == 0 && p.S_out && T > 0) {
            const int i = row;
            const int col = 32 * colhalf;
            float v[32];
            tc::tmem_ld32(tmem + lane_base + kTmX + col, v);
            float4 *dst = reinterpret_cast<float4 *>(p.S_out + sbase + (size_t)i * kDV + dv0 + col);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(v[4 * q] * fprev[i], v[4 * q + 1] * fprev[i], v[4 * q + 2] * fprev[i],
                                     v[4 * q + 3] * fprev[i]);
        }
    } else if (warp == 8) {
        // ---- record loader: one lane serves the state warps' requests in order
        if (lane == 0) {
            for (uint32_t k = 0;; ++k) {
                const uint32_t sl = k & 1u;
                bool got = false;
                for (int tries = 0; tries < 64 && !got; ++tries) {
                    got = tc::mbar_wait(s_lq + 8u * sl, (k >> 1) & 1u, p.spin);
                    if (!got && (flags[0] != 0 || flags[3] != 0)) break;
                }
                if (!got) break;
                const int w = req[2 * sl], b = req[2 * sl + 1];
                tc::mbar_arrive_local(s_lfree + 8u * sl);
                if (w < 0) break;
                issue_rec(w, b);
            }
        }
    } else if (warp >= 10) {
        // ---- readout warps: O (TMEM lanes 64-127) -> RMS norm over d_v (both
        // CTAs' columns, exchanged through distributed shared memory), gate, store
        const int et = tid - 320;                    // token row of the chunk
        for (int c = 0;; ++c) {
            const uint32_t slot = (uint32_t)(c & 1), ph = (uint32_t)(c >> 1) & 1u;
            // one thread waits, the barrier hands its view (and the chunk info) to the rest
            if (et == 0 && !tc::mbar_wait(s_ibar + 8u * slot, ph, p.spin)) flags[3] = 1;
            asm volatile("bar.sync 3, 64;" ::: "memory");
            if (flags[3] != 0) break;
            // every row is done with the previous chunk's exchange slot: it now
            // expects the peer's sums of chunk c + 1
            if (et == 0) tc::mbar_arrive_expect_tx(s_xbar + 8u * (slot ^ 1u), 65 * 4);
            const int t0 = info[4 * slot], n = info[4 * slot + 1];
            if (info[4 * slot + 2] != 0) break;      // no more chunks
            // the gate of this row, fetched while the chunk's products run
            const bool live = et < n;
            const size_t gi = (((size_t)bb * T + t0 + et) * H + h) * kDV + dv0;
            // 32-byte accesses when the tensors allow them: the row pieces of a chunk
            // are 4 KB apart, and full-sector accesses keep the SM's memory queue
            // short for the record copies that share it
            const bool a32 = ((reinterpret_cast<uintptr_t>(p.g) | reinterpret_cast<uintptr_t>(p.y) |
                               reinterpret_cast<uintptr_t>(p.o_raw)) & 31u) == 0;
            uint4 gq[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) gq[q] = make_uint4(0, 0, 0, 0);
            if (live) {
                if (a32) {
#pragma unroll
                    for (int q = 0; q < 8; q += 2) tc::ld_global_nc_v8(p.g + gi + 8 * q, gq[q], gq[q + 1]);
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) gq[q] = __ldg(reinterpret_cast<const uint4 *>(p.g + gi) + q);
                }
            }
            bool ok = true;
            if (et == 0) ok = tc::mbar_wait(s_obar + 8u * slot, ph, p.spin);
            asm volatile("bar.sync 3, 64;" ::: "memory");
            tc::fence_after_sync();
            float ov[2][32];
            const uint32_t ro = kTmRO + (uint32_t)kDVC * slot;
            tc::tmem_ld32x2(tmem + lane_base + ro, tmem + lane_base + ro + 32, ov[0], ov[1]);
            tc::fence_before_sync();
            asm volatile("bar.sync 3, 64;" ::: "memory");
            // the slot may take a new chunk; a releasing arrival would first wait for
            // this thread's y stores of the previous chunk to reach L2
            if (et == 0) tc::mbar_arrive_local_relaxed(s_fbar + 8u * slot);
            float ss = 0.f;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int q = 0; q < 32; ++q) ss += ov[hf][q] * ov[hf][q];
            // exchange: this row's sum (and the abort flag) into the peer's slot as
            // asynchronous stores counted on the peer's barrier
            tc::st_async_f32(r_peer + slot * 256u + 4u * et, ss, r_xbar + 8u * slot);
            if (et == 0) tc::st_async_s32(r_pflag + 4u * slot, (ok && flags[0] == 0) ? 0 : 1, r_xbar + 8u * slot);
            if (et == 0) {
                const bool got = tc::mbar_wait_cluster(s_xbar + 8u * slot, ph, p.spin);
                if (!got || pflag[slot] != 0 || !ok) flags[3] = 1;
            }
            asm volatile("bar.sync 3, 64;" ::: "memory");
            if (flags[3] != 0) break;
            if (live) {
                const float inv = rsqrtf((ss + peer[slot * 64 + et]) / kDV + p.eps);
                uint4 yq[8];
#pragma unroll
                for (int q8 = 0; q8 < 8; ++q8) {
                    float gg[8];
                    bf16x8_to_f(gq[q8], gg);
                    const float *o8 = &ov[q8 >> 2][8 * (q8 & 3)];
                    __nv_bfloat162 *hb = reinterpret_cast<__nv_bfloat162 *>(&yq[q8]);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hb[e] = __floats2bfloat162_rn(gg[2 * e] * o8[2 * e] * inv, gg[2 * e + 1] * o8[2 * e + 1] * inv);
                }
                if (a32) {
#pragma unroll
                    for (int q8 = 0; q8 < 8; q8 += 2) tc::st_global_v8(p.y + gi + 8 * q8, yq[q8], yq[q8 + 1]);
                } else {
#pragma unroll
                    for (int q8 = 0; q8 < 8; ++q8) *reinterpret_cast<uint4 *>(p.y + gi + 8 * q8) = yq[q8];
                }
                if (p.o_raw) {
#pragma unroll
                    for (int q8 = 0; q8 < 8; ++q8) {
                        const float *o8 = &ov[q8 >> 2][8 * (q8 & 3)];
                        const uint4 lo = make_uint4(__float_as_uint(o8[0]), __float_as_uint(o8[1]), __float_as_uint(o8[2]),
                                                    __float_as_uint(o8[3]));
                        const uint4 hi = make_uint4(__float_as_uint(o8[4]), __float_as_uint(o8[5]), __float_as_uint(o8[6]),
                                                    __float_as_uint(o8[7]));
                        if (a32) {
                            tc::st_global_v8(p.o_raw + gi + 8 * q8, lo, hi);
                        } else {
                            reinterpret_cast<uint4 *>(p.o_raw + gi + 8 * q8)[0] = lo;
                            reinterpret_cast<uint4 *>(p.o_raw + gi + 8 * q8)[1] = hi;
                        }
                    }
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (range_max > 60000.f && p.status) atomicCAS(p.status, 0, (int)kDevRange);
    if ((flags[0] != 0 || flags[3] != 0) && tid == 0 && p.status) atomicCAS(p.status, 0, (int)kDevTimeout);
    // an MMA whose completion wait ran out finishes before its TMEM is freed
    if (tid == 0 && mma_pending >= 0) tc::mbar_wait(s_mbar, (uint32_t)mma_pending, kDrainPolls);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
    // no CTA leaves while its peer may still write into its shared memory
    tc::cluster_sync();
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
// 74.8 KB, so that three CTAs share an SM.  Regions are reused as the window
// proceeds: after P, the [Kc; K^c] tile (bulk-copied to the record) holds the
// fp32 L / T^-1, the merge buffer and the fp16 T^-1 tile; after the operand
// build, the scan scratch holds the fp16 M tile.
struct IntraSmem {
    static constexpr int AP = 0;                  // [Kp ; Qp]   128 x 128 fp16 (then W' over Kp, Aq/Bq over Qp)
    static constexpr int BP = AP + 128 * 256;     // [Kc ; K^c]  128 x 128
    static constexpr int LW = BP;                 //   after P: fp32 L, then T^-1   [64][kLW]
    static constexpr int YB = LW + 64 * kLW * 4;  //   merge buffer                 [32][kYS]
    static constexpr int TI = BP + 23 * 1024;     //   T^-1, 64 x 64 fp16 (1024-byte aligned)
    static constexpr int SCR = BP + 128 * 256;    // scan scratch, then M (64 x 64 fp16)
    static constexpr int WT = SCR;                //   fp32 per-warp log-decay totals [8][128]
    static constexpr int PR = WT + 8 * 128 * 4;   //   fp32 Lambda of tokens 0 and 63 [2][128]
    static constexpr int MM = SCR;
    static constexpr int VEC = SCR + 64 * 128;    // gamma_stat [128], exact diagonals [2][64], span maxima [8]
    static constexpr int MISC = VEC + (128 + 128 + 8) * 4;   // mbarriers, TMEM slot, flags
    static constexpr int TOTAL = MISC + 64;
};
static_assert(IntraSmem::YB + 32 * kYS * 4 <= IntraSmem::TI, "merge buffer before the T^-1 tile");
static_assert(IntraSmem::TI + 64 * 128 <= IntraSmem::SCR, "T^-1 tile inside the [Kc; K^c] region");
static_assert(IntraSmem::PR + 2 * 128 * 4 <= IntraSmem::VEC, "scan scratch inside the M region");
static_assert(3 * (IntraSmem::TOTAL + 1024 + 1024) <= 228 * 1024, "three CTAs per SM");
// TMEM (128 columns): P (M = 128) at column 0; after its epilogue W' (M = 64)
// in lanes 0-15 of each 32-lane quadrant and N (M = 64) in lanes 16-31, both
// from column 0.
constexpr uint32_t kItmW = 0;
constexpr uint32_t kItmN = 16u << 16;
}  // namespace

// The intra kernel's raw inputs k, q, z, b as 4-D TMA maps over [B, T, H, 128]
// bf16 (innermost first: channel, head, token, batch; tokens past T read as
// zeros), boxes of 64 channels x 1 head x 64 tokens x 1 with the 128-byte
// swizzle: one box is one 64-column block of 64 rows of a row tile.
struct IntraMaps {
    CUtensorMap k, q, z, b;
};

// Input forms, fixed at compile time: kNoZ reads no z (2 sigmoid(z) = 1), kBeta
// reads one beta per token and head for both b and w, kTok one log-decay per
// token and head, kRaw applies SiLU and l2 normalisation to q and k.  All false
// is the per-channel GDN-2 form on preprocessed q and k.
template <bool kNoZ, bool kBeta, bool kTok, bool kRaw>
__global__ void __launch_bounds__(kThreads, 3)
    gdn2_chunk_intra_tc_kernel(TcParams p, uint8_t *ws, int *wflags, const __grid_constant__ IntraMaps im) {
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
    tc::grid_launch_dependents();                 // the chain kernel may launch once every CTA has started

    float *lw = (float *)(sm + L::LW);
    float *yb = (float *)(sm + L::YB);
    float *wtot = (float *)(sm + L::WT);
    float *probe = (float *)(sm + L::PR);
    float *vec = (float *)(sm + L::VEC);
    float *gsv = vec, *diagq = vec + 128, *diagb = vec + 192, *spanred = vec + 256;
    uint64_t *mbar = (uint64_t *)(sm + L::MISC);
    uint32_t *tslot = (uint32_t *)(sm + L::MISC + 8);
    int *flags = (int *)(sm + L::MISC + 16);
    const uint32_t s_stall = tc::smem_u32(sm + L::MISC + 32);    // never completed (failure-path tests)
    const uint32_t s_tbar = tc::smem_u32(sm + L::MISC + 40);     // the raw input tiles
    const uint32_t s_ap = tc::smem_u32(sm + L::AP), s_bp = tc::smem_u32(sm + L::BP);
    const uint32_t s_ti = tc::smem_u32(sm + L::TI), s_mm = tc::smem_u32(sm + L::MM);
    const uint32_t s_mbar = tc::smem_u32(mbar);

    if (warp == 0) {
        tc::tmem_alloc(tc::smem_u32(tslot), 128);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(s_mbar, 1);
        tc::mbar_init(s_stall, 1);
        tc::mbar_init(s_tbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        flags[0] = 0;
        // until its record is complete the window is marked for the chain kernel to
        // process itself, so an abandoned record is never read
        wflags[wi] = 1;
        // The window's raw k, q, z and b, by TMA, straight into the places of the
        // operand tiles they become (k -> Kp rows, q -> Qp rows of [Kp; Qp]; z -> Kc
        // rows, b -> K^c rows of [Kc; K^c]): the build turns them over in place, each
        // thread reading and writing the same elements.  They arrive during the scan.
        constexpr uint32_t kBox = 64 * 128;                      // one box: 64 rows x 128 bytes
        tc::mbar_arrive_expect_tx(s_tbar, (uint32_t)((4 - (kNoZ ? 1 : 0) - (kBeta ? 1 : 0)) * 2) * kBox);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t blk = (uint32_t)c * 128 * 128;       // column block c of a 128-row tile
            tc::tma_load_4d(s_ap + blk, &im.k, 64 * c, h, t0, bb, s_tbar);
            tc::tma_load_4d(s_ap + blk + kBox, &im.q, 64 * c, h, t0, bb, s_tbar);
            if (!kNoZ) tc::tma_load_4d(s_bp + blk, &im.z, 64 * c, h, t0, bb, s_tbar);
            if (!kBeta) tc::tma_load_4d(s_bp + blk + kBox, &im.b, 64 * c, h, t0, bb, s_tbar);
        }
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
    int mma_pending = -1;                         // parity of an MMA commit whose wait ran out
    auto wait_mma = [&]() -> bool {
        const bool ok = tc::mbar_wait(s_mbar, phase, p.spin);
        if (!ok) {
            flags[0] = 1;
            mma_pending = (int)phase;
        }
        phase ^= 1u;
        __syncthreads();
        tc::fence_after_sync();
        return flags[0] == 0;
    };

    do {
        // failure-path test: a wait that nothing completes runs out before any work is issued
        if (p.stall) {
            if (tid == 0 && !tc::mbar_wait(s_stall, 0, p.spin)) flags[0] = 1;
            __syncthreads();
            if (flags[0] != 0) break;
        }
        // ---- the log-decay scan, in log2 units (Lambda * log2 e) so that every decay
        // factor is one ex2.  Warp w owns tokens [8w, 8w+8), lane l channels [4l, 4l+4)
        // (whole 256-byte token rows per load instruction).  Pass 1 sums the warp's
        // log-decays for the cross-warp prefix; the build below reads them again token
        // by token (from L2, one token ahead) and keeps only a running sum.
        const int tb = 8 * warp, c4 = 4 * lane;
        // Look-ahead loads are unconditional, from the token index clamped into the
        // window, and keep their raw bits; the zeros past the end of the sequence
        // and any broadcast are applied where the value is used.  (A load whose
        // result is selected against a zero, or shifted, right away makes the warp
        // wait for it there, which defeats loading it ahead.)
        auto live = [&](int u) { return t0 + tb + u < wend; };
        auto gtc_of = [&](int u) -> size_t { return ((size_t)bb * T + min(t0 + tb + u, wend - 1)) * H + h; };
        auto load_la = [&](int u) -> float4 {       // kTok: the token's scalar in .x
            float4 x;
            if (kTok) x.x = __ldg(p.la + gtc_of(u));
            else x = __ldg(reinterpret_cast<const float4 *>(p.la + gtc_of(u) * kDK + c4));
            return x;
        };
        auto la_val = [&](float4 x, int u) -> float4 {
            if (kTok) x = make_float4(x.x, x.x, x.x, x.x);
            return live(u) ? x : make_float4(0.f, 0.f, 0.f, 0.f);
        };
        // token u's beta, when b comes per token: the raw bf16, then as a quad
        auto load_beta = [&](int u) -> uint32_t {
            return kBeta ? (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.beta) + gtc_of(u)) : 0u;
        };
        auto beta_val = [&](uint32_t x, int u) -> uint2 {
            const uint32_t q2 = live(u) ? (x | (x << 16)) : 0u;
            return make_uint2(q2, q2);
        };
        float off[4] = {0.f, 0.f, 0.f, 0.f};
        {
            float tot[4] = {0.f, 0.f, 0.f, 0.f}, first[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 x = la_val(load_la(u), u);
                if (u == 0) {
                    first[0] = x.x * kLog2e; first[1] = x.y * kLog2e; first[2] = x.z * kLog2e; first[3] = x.w * kLog2e;
                }
                tot[0] += x.x * kLog2e; tot[1] += x.y * kLog2e; tot[2] += x.z * kLog2e; tot[3] += x.w * kLog2e;
            }
            *reinterpret_cast<float4 *>(wtot + warp * kDK + c4) = make_float4(tot[0], tot[1], tot[2], tot[3]);
            __syncthreads();
            for (int ww = 0; ww < warp; ++ww) {
                const float4 o4 = *reinterpret_cast<const float4 *>(wtot + ww * kDK + c4);
                off[0] += o4.x; off[1] += o4.y; off[2] += o4.z; off[3] += o4.w;
            }
            // Lambda at token 0 and at the last token (zero-padded log-decay past the end)
            if (warp == 0) *reinterpret_cast<float4 *>(probe + c4) = make_float4(first[0], first[1], first[2], first[3]);
            if (warp == 7)
                *reinterpret_cast<float4 *>(probe + kDK + c4) =
                    make_float4(off[0] + tot[0], off[1] + tot[1], off[2] + tot[2], off[3] + tot[3]);
        }
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
        // the raw input tiles, issued at the start
        if (tid == 0 && !tc::mbar_wait(s_tbar, 0, p.spin)) flags[0] = 1;
        __syncthreads();
        if (flags[0] != 0) break;

        // ---- operand tiles: P operands to shared memory (Qp, Kc and K^c reach the
        // record from there by bulk copy); the pivot vectors straight to the record
        uint2 vw_nx[2];                               // token 0's v and w, loaded during the build
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
            float lam_run[4] = {off[0], off[1], off[2], off[3]};     // Lambda before token u
            float4 la_nx = load_la(0);
            uint32_t beta_nx = load_beta(0);
            float dg[16];                             // [u]: q~.k, [8+u]: q~.(b*k) of token tb+u, this lane's channels
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int t = tb + u;
                const bool live_t = t < n;
                const float4 la_c = la_val(la_nx, u);
                const uint2 beta_c = beta_val(beta_nx, u);
                const uint32_t off_t = tc::tile_off(128, t, c4), off_b = tc::tile_off(128, 64 + t, c4);
                // this thread's four channels of the raw k, q, z, b (their tile places)
                const uint2 kq_c[4] = {*(const uint2 *)(sm + L::AP + off_t), *(const uint2 *)(sm + L::AP + off_b),
                                       kNoZ ? make_uint2(0, 0) : *(const uint2 *)(sm + L::BP + off_t),
                                       kBeta ? beta_c : *(const uint2 *)(sm + L::BP + off_b)};
                if (u + 1 < 8) {                      // the next token's log-decay is in flight meanwhile
                    la_nx = load_la(u + 1);
                    beta_nx = load_beta(u + 1);
                } else {                              // the value side of token 0, for after the build
                    const size_t gt = gtc_of(0), gv = gt * kDV + c4;
                    vw_nx[0] = __ldg(reinterpret_cast<const uint2 *>(p.v + gv));
                    vw_nx[1] = kBeta ? make_uint2(load_beta(0), 0u) : __ldg(reinterpret_cast<const uint2 *>(p.w + gv));
                }
                lam_run[0] += la_c.x * kLog2e; lam_run[1] += la_c.y * kLog2e;
                lam_run[2] += la_c.z * kLog2e; lam_run[3] += la_c.w * kLog2e;
                float kk[4], qq[4], zz[4], bv[4];
                {
                    const __nv_bfloat162 *hk = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[0]);
                    const __nv_bfloat162 *hq = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[1]);
                    const __nv_bfloat162 *hz = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[2]);
                    const __nv_bfloat162 *hb = reinterpret_cast<const __nv_bfloat162 *>(&kq_c[3]);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float2 f;
                        f = __bfloat1622float2(hk[e]); kk[2 * e] = f.x; kk[2 * e + 1] = f.y;
                        f = __bfloat1622float2(hq[e]); qq[2 * e] = f.x; qq[2 * e + 1] = f.y;
                        f = __bfloat1622float2(hz[e]); zz[2 * e] = f.x; zz[2 * e + 1] = f.y;
                        f = __bfloat1622float2(hb[e]); bv[2 * e] = f.x; bv[2 * e + 1] = f.y;
                    }
                    if (kRaw) {                         // the q/k preprocessing, one token a call
                        silu_l2n_row4(kk);
                        silu_l2n_row4(qq);
                    }
                }
                float kp[4], kc[4], khc[4], qp[4];
                float dq = 0.f, db = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float lam = live_t ? lam_run[c] : lnv[c];
                    const float d = lam - cpiv[c];
                    const float ep = ex2(d), em = ex2(-d);
                    const float kv = live_t ? kk[c] : 0.f;
                    const float qt = live_t ? qq[c] * gq[c] * two_sigmoid_fast(zz[c]) : 0.f;
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
                const uint2 ukp = make_uint2(tc::pack_half2(kp[0], kp[1]), tc::pack_half2(kp[2], kp[3]));
                const uint2 uqp = make_uint2(tc::pack_half2(qp[0], qp[1]), tc::pack_half2(qp[2], qp[3]));
                const uint2 ukc = make_uint2(tc::pack_half2(kc[0], kc[1]), tc::pack_half2(kc[2], kc[3]));
                const uint2 ukh = make_uint2(tc::pack_half2(khc[0], khc[1]), tc::pack_half2(khc[2], khc[3]));
                *(uint2 *)(sm + L::AP + off_t) = ukp;
                *(uint2 *)(sm + L::AP + off_b) = uqp;
                *(uint2 *)(sm + L::BP + off_t) = ukc;
                *(uint2 *)(sm + L::BP + off_b) = ukh;
            }
        // the exact diagonals q~_t.k_t and q~_t.(b*k)_t of Aq / Bq
            const float dsum = reduce_scatter16(dg, lane);
            if ((lane & 1) == 0) {
                const int vi = (lane >> 1) & 15;
                (vi < 8 ? diagq : diagb)[tb + (vi & 7)] = dsum;
            }
        }
        tc::fence_proxy_async();
        __syncthreads();

        // ---- P = [Kp; Qp] [Kc; K^c]^T; the record's [Kc; K^c] tile and the Qp rows
        // of [W'; Qp] are copied out of the same shared-memory tiles meanwhile
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t id = tc::idesc_f16(128, 128, false, false, false);
            for (int ks = 0; ks < kDK / 16; ++ks)
                tc::mma_f16(tmem, tc::desc_kmajor(s_ap, 128, 0, ks), tc::desc_kmajor(s_bp, 128, 0, ks), id, ks > 0);
            tc::mma_commit(s_mbar);
            tc::bulk_s2g(rec + kWinBP, s_bp, 128 * 256);
            tc::bulk_s2g(rec + kWinAP + 64 * 128, s_ap + 64 * 128, 64 * 128);                 // Qp, columns 0-63
            tc::bulk_s2g(rec + kWinAP + 128 * 128 + 64 * 128, s_ap + 128 * 128 + 64 * 128, 64 * 128);  // columns 64-127
            tc::bulk_commit();
        }
        // V^ = w*v -> window record (the identity padding past n is zero), while the P
        // product runs: token 0's v and w were loaded during the build, the other
        // seven tokens' are all issued here before the first is used
        uint2 vr[8][2];
        vr[0][0] = vw_nx[0];
        vr[0][1] = vw_nx[1];
#pragma unroll
        for (int u = 1; u < 8; ++u) {
            const size_t gv = gtc_of(u) * kDV + c4;
            vr[u][0] = __ldg(reinterpret_cast<const uint2 *>(p.v + gv));
            vr[u][1] = kBeta ? make_uint2(load_beta(u), 0u) : __ldg(reinterpret_cast<const uint2 *>(p.w + gv));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = tb + u;
            const bool in = live(u);
            const uint2 vw_c[2] = {in ? vr[u][0] : make_uint2(0, 0),
                                   !in ? make_uint2(0, 0) : kBeta ? beta_val(vr[u][1].x, u) : vr[u][1]};
            const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&vw_c[0]);
            const __nv_bfloat162 *hw = reinterpret_cast<const __nv_bfloat162 *>(&vw_c[1]);
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

        // ---- masks; M -> MM (shared), L -> fp32 (over BP), Aq / Bq -> staged over
        // the Qp rows of AP (in the record's byte layout) and copied to the record.
        // This warp's rows are tokens t in [32 tb2, 32 tb2 + 32): column block hf
        // below the diagonal block is kept whole, above it zeroed, and only the
        // diagonal block is masked element by element.
        {
            const int t = row & 63;
            const bool upper = row < 64;
            const int tb2 = warp & 1;
            // the bulk copies have read BP and the Qp rows: both may now be overwritten
            // (P stays in TMEM until the W' / N products, issued after a later barrier)
            if (tid == 0) tc::bulk_wait_read();
            __syncthreads();
            const float dv_t = upper ? 0.f : (colhalf == 0 ? diagq[t] : diagb[t]);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float v[32];
                tc::tmem_ld32(tmem + lane_base + 64 * colhalf + 32 * hf, v);
                if (hf > tb2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.f;
                } else if (hf == tb2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const bool keep = upper ? (i < lane) : (i <= lane);
                        if (!keep) v[i] = 0.f;
                        if (!upper && i == lane) v[i] = dv_t;
                    }
                }
                if (upper && colhalf == 1) {
                    float4 *dst = reinterpret_cast<float4 *>(lw + t * kLW + 32 * hf);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                } else if (upper) {
                    store_row32(sm + L::MM, 64, t, 32 * hf, v);
                } else {
                    store_row32(sm + L::AP + (colhalf == 0 ? 64 * 128 : 128 * 128 + 64 * 128), 64, t, 32 * hf, v);
                }
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::bulk_s2g(rec + kWinANAB + 64 * 128, s_ap + 64 * 128, 64 * 128);                 // Aq
            tc::bulk_s2g(rec + kWinANAB + 128 * 128, s_ap + 128 * 128 + 64 * 128, 64 * 128);    // Bq
            tc::bulk_commit();
        }

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
                asm volatile("bar.sync 2, 64;" ::: "memory");
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

        // ---- W' -> staged over Kp (rows 0-63 of AP), N -> over M; both copied to
        // rows 0-63 of the record's [W'; Qp] and [N; Aq; Bq].  One load gives a warp
        // W' rows in its lanes 0-15 and N rows in lanes 16-31 (N has 64 columns, so
        // only the warps of the first column half keep those).
        {
            const int t = 16 * (warp & 3) + (lane & 15);
            const bool nrow = lane >= 16;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int col = 64 * colhalf + 32 * hf;
                float v[32];
                tc::tmem_ld32(tmem + lane_base + col, v);
                if (!nrow) {
                    range_max = fmaxf(range_max, maxabs(v, 32));
                    store_row32(sm + L::AP, 128, t, col, v);
                } else if (colhalf == 0) {
                    range_max = fmaxf(range_max, maxabs(v, 32));
                    store_row32(sm + L::MM, 64, t, 32 * hf, v);
                }
            }
        }
        tc::fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            tc::bulk_s2g(rec + kWinAP, s_ap, 64 * 128);                              // W', columns 0-63
            tc::bulk_s2g(rec + kWinAP + 128 * 128, s_ap + 128 * 128, 64 * 128);      // columns 64-127
            tc::bulk_s2g(rec + kWinANAB, s_mm, 64 * 128);                            // N
            tc::bulk_commit();
            wflags[wi] = 0;
        }
    } while (false);
    // the record's bulk copies complete before the CTA's shared memory goes away,
    // and so do the input loads (a window handed to the chain kernel, or an abort,
    // leaves before waiting for them)
    if (tid == 0) {
        tc::bulk_wait_all();
        tc::mbar_wait(s_tbar, 0, kDrainPolls);
    }

    if (range_max > 60000.f && p.status) atomicCAS(p.status, 0, (int)kDevRange);
    if (flags[0] != 0 && tid == 0 && p.status) atomicCAS(p.status, 0, (int)kDevTimeout);
    // an MMA whose completion wait ran out finishes before its TMEM is freed
    if (tid == 0 && mma_pending >= 0) tc::mbar_wait(s_mbar, (uint32_t)mma_pending, kDrainPolls);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

size_t fwd_tc_workspace_bytes(int B, int H, int T) {
    const size_t nwin = (size_t)B * H * ((T + kC - 1) / kC);
    return nwin * kWinBytes + ((nwin * sizeof(int) + 1023) & ~(size_t)1023);
}

bool fwd_tc_supported(int dtype, int dk, int dv, int chunk) {
    return dtype == GDELTA_BF16 && dk == 128 && dv == 128 && chunk == 64;
}

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

// A [B, T, H, 128] bf16 token tensor as the 4-D map the intra kernel loads from.
bool input_map(CUtensorMap *m, const void *base, int B, int T, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kDK, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t row = (cuuint64_t)kDK * 2;                  // bytes of one token row of one head
    const cuuint64_t strides[3] = {row, row * (cuuint64_t)H, row * (cuuint64_t)H * (cuuint64_t)T};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdParams &fp, void *workspace, cudaStream_t stream) {
    TcParams p;
    p.B = fp.B; p.T = fp.T; p.H = fp.H;
    p.q = (const __nv_bfloat16 *)fp.q; p.k = (const __nv_bfloat16 *)fp.k; p.z = (const __nv_bfloat16 *)fp.z;
    p.b = (const __nv_bfloat16 *)fp.b; p.v = (const __nv_bfloat16 *)fp.v; p.w = (const __nv_bfloat16 *)fp.w;
    p.g = (const __nv_bfloat16 *)fp.g;
    p.la = fp.la; p.gs = fp.gs; p.S_in = fp.S_in; p.S_out = fp.S_out;
    p.beta = (const __nv_bfloat16 *)fp.beta; p.decay_tok = fp.decay_tok; p.qk_raw = fp.qk_raw;
    p.y = (__nv_bfloat16 *)fp.y; p.o_raw = fp.o_raw; p.eps = fp.eps; p.status = fp.status;
    p.NW = (fp.T + kC - 1) / kC;
    p.spin = fp.wait_limit;
    p.stall = fp.stall;
    const size_t nwin = (size_t)fp.B * fp.H * p.NW;
    uint8_t *ws = (uint8_t *)workspace;
    int *wflags = (int *)(ws + nwin * kWinBytes);
    p.ws = ws;
    p.wflags = wflags;

    const size_t ismem = (size_t)IntraSmem::TOTAL + 1024;
    // the raw inputs the intra kernel loads by TMA (z and b only in the forms that read them)
    IntraMaps im;
    memset(&im, 0, sizeof(im));
    if (fp.T > 0) {
        if (!input_map(&im.k, p.k, fp.B, fp.T, fp.H) || !input_map(&im.q, p.q, fp.B, fp.T, fp.H) ||
            (p.z && !input_map(&im.z, p.z, fp.B, fp.T, fp.H)) || (p.b && !input_map(&im.b, p.b, fp.B, fp.T, fp.H)))
            return cudaErrorInvalidValue;
    }
    using IntraFn = void (*)(TcParams, uint8_t *, int *, IntraMaps);
#define GDN2_INTRA_FORMS(R)                                                                                    \
    gdn2_chunk_intra_tc_kernel<false, false, false, R>, gdn2_chunk_intra_tc_kernel<false, false, true, R>,    \
        gdn2_chunk_intra_tc_kernel<false, true, false, R>, gdn2_chunk_intra_tc_kernel<false, true, true, R>,  \
        gdn2_chunk_intra_tc_kernel<true, false, false, R>, gdn2_chunk_intra_tc_kernel<true, false, true, R>,  \
        gdn2_chunk_intra_tc_kernel<true, true, false, R>, gdn2_chunk_intra_tc_kernel<true, true, true, R>
    static constexpr IntraFn kIntra[16] = {GDN2_INTRA_FORMS(false), GDN2_INTRA_FORMS(true)};
#undef GDN2_INTRA_FORMS
    const IntraFn intra = kIntra[(p.qk_raw != 0) * 8 + (p.z == nullptr) * 4 + (p.beta != nullptr) * 2 +
                                 (p.decay_tok != 0)];
    cudaError_t e = cudaFuncSetAttribute(intra, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ismem);
    if (e != cudaSuccess) return e;
    intra<<<(unsigned)nwin, kThreads, ismem, stream>>>(p, ws, wflags, im);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)ChainSmem::TOTAL + 1024;
    auto chain = fp.qk_raw ? gdn2_fwd_tc_kernel<true> : gdn2_fwd_tc_kernel<false>;
    e = cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // clusters of two CTAs (value-column halves of one head), set by the kernel's
    // attribute; a programmatic dependent of the intra kernel
    return tc::launch_dependent(chain, dim3(2 * fp.B * fp.H), dim3(kChainThreads), smem, stream, p);
}

}  // namespace gdelta
