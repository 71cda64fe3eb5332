// Backward pass of the token mixer (fp32 CUDA cores, d_k = d_v = 128): the
// gradient of a loss with respect to every input, the static readout profile
// and the initial state, given its gradient with respect to y (and optionally
// the final state).
//
// A cluster of two CTAs per (batch, head); CTA c owns value columns
// [64 c, 64 c + 64) of every d_k x d_v matrix.  The columns of the recurrence
// are independent, so each CTA runs it on its half alone; what couples the
// halves is (a) the RMS norm of o over all d_v columns and (b) the key-side
// gradients, which are sums over the columns:
//  (a) phase F computes, per token, this CTA's partial sums of o^2 and of
//      g * dy * o (one pair per warp that reduces them) into the workspace;
//      one cluster barrier after phase F, and every later read sums the four
//      pairs in the same order, so both CTAs use the same rho;
//  (b) each CTA adds its share of dk, db, d log alpha, dq, dz to the outputs
//      (zeroed by the launcher) with atomic reductions: two addends to a zero,
//      so the result does not depend on their order.
//
// Phase F runs the recurrence forward and keeps the state every kBC tokens
// (checkpoints), and each token's o and r on this CTA's columns.  Phase B walks
// the chunks from the last: it recomputes the chunk's kBC + 1 states from its
// checkpoint (with the stored r, a state step needs no column sum and one
// barrier a token), passing them through two shared-memory tiles to a per-CTA
// chunk buffer by bulk copies, then takes the tokens in reverse with the exact
// per-token gradient recurrence below (o and r again from phase F), loading
// each state back by bulk copy one token ahead.  Per-token inputs are fetched
// into registers a few tokens ahead (phase F and the recompute: four, the
// walk: two), the token loops unrolled so that the register sets rotate
// without moves.
// Per token, with S_hat = Diag(alpha) S_{t-1}, r = k S_hat,
// S_t = S_hat - (b*k)^T r + k^T (w*v), o = q~ S_t and y = g * o * rho,
// rho = 1 / sqrt(mean(o^2) + eps) (Muir review §2.1):
//
//   do      = rho (g*dy) - rho^3 / d_v * o * sum(g*dy*o)        dg = dy * o * rho
//   dS     += q~^T do                                          dq~ = S_t do^T
//   dv^     = k dS            dr = -(b*k) dS                   d(b*k) = -dS r^T
//   dk      = dS v^T + Diag(alpha) S_{t-1} dr^T + b * d(b*k)   db = k * d(b*k)
//   dS_hat  = dS + k^T dr     dalpha = rowsum(dS_hat * S_{t-1}) dS_{t-1} = Diag(alpha) dS_hat
//
// and the chain rule through q~ = q * gamma * 2 sigmoid(z), v^ = w * v,
// alpha = exp(log_alpha).  The checkpoints, chunk states, per-token o and r and
// RMS partials live in the caller's workspace; the running dS (this CTA's half)
// lives in registers, each thread holding its own elements.
//
// Thread layout (256 threads): warp w, lane l = 16 h + c holds rows
// w + 8 h + 16 m (m = 0..7) and the CTA's columns 4c..4c+3, so a row's sum over
// the CTA's columns is a reduction over a half-warp and a column's sum one over
// the 16 (warp, half) groups.
#include "common.cuh"
#include "tc_common.cuh"

namespace gdelta {

namespace {

constexpr int kBD = 128;             // d_k = d_v
constexpr int kBH = 64;              // value columns per CTA
constexpr int kBT = 256;             // threads
constexpr int kBRows = 8;            // rows per thread
constexpr int kBC = 32;              // tokens per checkpoint
constexpr uint32_t kSlotBytes = kBD * kBH * 4;   // one [128][64] fp32 state half-matrix
constexpr uint32_t kBwdDrainPolls = 1u << 22;    // polls of the wait that drains a copy after a timeout
// The thread that issues the walk's state loads: in warp 6, which has no key or
// value role, so that its proxy fence never waits on gradient atomics.
constexpr int kLoader = 192;
static_assert(kLoader >= kBD + kBH && kLoader < kBT, "the loader thread has no key or value role");

// Reduce-scatter of 8 per-lane values over a half-warp: afterwards lane l
// holds the sum over its 16 lanes of value (l >> 1) & 7.
__device__ __forceinline__ float rows_reduce_scatter8(const float (&v)[8], int lane) {
    float w4[4], w2[2];
    const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float keep = b3 ? v[4 + j] : v[j], send = b3 ? v[j] : v[4 + j];
        w4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float keep = b2 ? w4[2 + j] : w4[j], send = b2 ? w4[j] : w4[2 + j];
        w2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    const float keep = b1 ? w2[1] : w2[0], send = b1 ? w2[0] : w2[1];
    const float w1 = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    return w1 + __shfl_xor_sync(0xffffffffu, w1, 1);
}

// An input element's raw bits, converted to fp32 only where it is used: a value
// fetched tokens ahead of its use then keeps its load in flight instead of
// stalling the warp at the conversion right after the load.
__device__ __forceinline__ uint32_t ldraw(const float *p, size_t i) { return __float_as_uint(p[i]); }
__device__ __forceinline__ uint32_t ldraw(const __nv_bfloat16 *p, size_t i) {
    return (uint32_t)reinterpret_cast<const unsigned short *>(p)[i];
}
__device__ __forceinline__ float cvraw(uint32_t x, const float *) { return __uint_as_float(x); }
__device__ __forceinline__ float cvraw(uint32_t x, const __nv_bfloat16 *) { return __uint_as_float(x << 16); }

// Atomic add with no return value (a reduction): the issuing thread never waits
// for the old value to come back from L2.
__device__ __forceinline__ void red_add(float *p, float x) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(x) : "memory");
}

// alpha = e^{log alpha} and 2 sigmoid(z) with the special-function unit's
// exponential (relative error about 1e-6, far inside what the fp32 recurrence
// needs); the exponent of the sigmoid is clamped so that its sum stays finite.
__device__ __forceinline__ float alpha_of(float la) { return __expf(la); }
__device__ __forceinline__ float two_sigmoid_bwd(float z) { return __fdividef(2.f, 1.f + __expf(fminf(-z, 80.f))); }

__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

// One token's vectors in shared memory.  Two of these alternate by token
// parity, so that staging a token never overwrites what the previous one is
// still being read from; the barriers each phase needs for its own data order
// the rest.
struct __align__(16) TokBuf {
    float k[kBD], kh[kBD], ka[kBD], al[kBD], qt[kBD];        // key side: k, b*k, k*alpha, alpha, q~
    float vh[kBH], r[kBH], dO[kBH];                           // value side, this CTA's columns: w*v, r, do
};

struct BwdSmem {
    TokBuf tb[2];
    float dr[kBH];                                            // dr of the token being walked
    float redA[16][kBH], redB[16][kBH];                       // column partials per (warp, half)
    float rows[5][kBD];                                       // row sums over this CTA's columns
};

// fmaf form of S_t = alpha S_{t-1} - (b*k) r + k (w*v) for one element, shared by
// phase F and the recompute so that the recomputed states equal the checkpointed
// trajectory bit for bit
__device__ __forceinline__ float state_step(float s, float al, float kh, float rj, float kk, float vj) {
    return fmaf(kk, vj, fmaf(-kh, rj, al * s));
}

template <typename T>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kBT, 1) gdn2_bwd_kernel(BwdParams p) {
    __shared__ BwdSmem sm;
    extern __shared__ float4 dsm_base[];                     // two state tiles, then their mbarriers
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hl = lane >> 4, lc = lane & 15, col4 = 4 * lc;
    const int c = (int)tc::cluster_ctarank(), gc0 = kBH * c;  // this CTA's first value column
    const int head = blockIdx.x >> 1, h = head % p.H, bb = head / p.H;
    const int T_ = p.T, H = p.H;
    const int NC = (T_ + kBC - 1) / kBC;
    const size_t mat = (size_t)kBD * kBH;                    // one half-matrix buffer: [128][64]
    const size_t hc = (size_t)head * 2 + c;
    float *ckpt = p.ws_ckpt + hc * (NC + 1) * mat;
    float *chunk = p.ws_chunk + hc * (kBC + 1) * mat;
    float *part = p.ws_part + (size_t)head * T_ * 8;         // per token: (sum o^2, sum g dy o) x 4 warps-of-a-CTA
    float *orw = p.ws_or + hc * (size_t)T_ * 2 * kBH;        // per token: o, then r, of this CTA's columns
    const T *q = (const T *)p.q, *k = (const T *)p.k, *z = (const T *)p.z, *b = (const T *)p.b;
    const T *v = (const T *)p.v, *w = (const T *)p.w, *g = (const T *)p.g;
    const bool keyt = tid < kBD, valt = tid >= kBD && tid < kBD + kBH;
    const int j = tid - kBD;                                  // a value thread's column in this CTA
    auto row_of = [&](int m) { return warp + 8 * hl + 16 * m; };
    auto own = [&](int m) { return (size_t)row_of(m) * kBH + col4; };           // in a half-matrix buffer
    auto own_full = [&](int m) { return (size_t)row_of(m) * kBD + gc0 + col4; };  // in a [128][128] matrix
    // Two state tiles in shared memory (each a [128][64] half-matrix, the chunk
    // buffer's layout) and their mbarriers (a third one is never completed: the
    // failure-path test waits on it).  The chunk's states move between them and
    // the chunk buffer by bulk copies (one thread, 32 KiB each), which keeps that
    // traffic off the threads' load/store path.
    float *const slot0 = reinterpret_cast<float *>(dsm_base);
    auto slot = [&](int x) { return slot0 + (size_t)x * mat; };
    const uint32_t s_slot0 = tc::smem_u32(slot0), s_mb = s_slot0 + 2 * kSlotBytes;
    uint32_t ph = 0;                                          // bit x: parity of the next wait on slot x
    if (tid == 0) {
        tc::mbar_init(s_mb, 1);
        tc::mbar_init(s_mb + 8, 1);
        tc::mbar_init(s_mb + 16, 1);                          // never completed (failure-path tests)
    }
    __syncthreads();
    // failure-path test: a wait that nothing completes runs out and is reported;
    // both CTAs of the cluster leave here, before any cluster barrier
    if (p.stall) {
        if (tid == 0 && !tc::mbar_wait(s_mb + 16, 0, p.wait_limit) && p.status) atomicCAS(p.status, 0, (int)kDevTimeout);
        return;
    }
    // bounded wait for slot x's bulk load; a wait that runs out is reported and then
    // drained, so that no copy is still landing when the slot is used again
    auto wait_slot = [&](int x) {
        const uint32_t mb = s_mb + 8 * x, par = (ph >> x) & 1u;
        if (!tc::mbar_wait(mb, par, p.wait_limit)) {
            if (p.status) atomicCAS(p.status, 0, (int)kDevTimeout);
            tc::mbar_wait(mb, par, kBwdDrainPolls);
        }
        ph ^= 1u << x;
    };

    // Token t's inputs, fetched into registers tokens ahead of use (raw bits; cv
    // and fl convert them): the key side of channel tid & 127 (k0-k4: k, log
    // alpha, b, q, z), used by threads 0-127, and the value side of this CTA's
    // column tid & 63 (v0-v5: w, v, dy, g, and in phase B r and o; in the walk
    // also the token's eight RMS partials), used by threads 128-191.  Every thread
    // loads every field, from an index that is valid for any thread: a field that
    // one role loads and another leaves alone would make the compiler merge the
    // two at the end of the branch, and that merge waits for the load.  The
    // gradient step reads the same registers again.  Phases: kF (forward,
    // checkpoints), kRe (recompute a chunk), kWalk.
    enum { kF = 0, kRe = 1, kWalk = 2 };
    struct Tok {
        uint32_t k0, k1, k2, k3, k4;
        uint32_t v0, v1, v2, v3, v4, v5;
        float4 pa, pb;
    };
    auto cv = [&](uint32_t x) { return cvraw(x, q); };       // a token-dtype input
    auto fl = [](uint32_t x) { return __uint_as_float(x); };  // an fp32 input
    const float gs_own = (keyt && p.gs) ? p.gs[(size_t)h * kBD + tid] : 1.f;
    const float *dy_src = p.dy ? p.dy : p.la;                  // (read but unused when dy is absent)
    auto fetch = [&](int t, int ph) -> Tok {
        Tok r;
        const size_t gt = ((size_t)bb * T_ + t) * H + h;
        const size_t gi = gt * kBD + (tid & (kBD - 1)), gj = gt * kBD + gc0 + (tid & (kBH - 1));
        const size_t oj = (size_t)t * 2 * kBH + (tid & (kBH - 1));
        r.k0 = ldraw(k, gi);
        r.k1 = ldraw(p.la, gi);
        r.k2 = ldraw(b, gi);
        r.v0 = ldraw(w, gj);
        r.v1 = ldraw(v, gj);
        if (ph != kRe) {
            r.k3 = ldraw(q, gi);
            r.k4 = ldraw(z, gi);
            r.v2 = ldraw(dy_src, gj);
            r.v3 = ldraw(g, gj);
        }
        if (ph != kF) r.v4 = ldraw(orw, oj + kBH);
        if (ph == kWalk) {
            r.v5 = ldraw(orw, oj);
            r.pa = ld4(part + (size_t)t * 8);
            r.pb = ld4(part + (size_t)t * 8 + 4);
        }
        return r;
    };
    auto dy_of = [&](const Tok &r) { return p.dy ? fl(r.v2) : 0.f; };
    // the token's vectors into buffer bf (no barrier here: see TokBuf)
    auto stage = [&](const Tok &r, int ph, TokBuf &bf) {
        if (keyt) {
            const float kk = cv(r.k0), al = alpha_of(fl(r.k1));
            bf.k[tid] = kk;
            bf.kh[tid] = cv(r.k2) * kk;
            bf.al[tid] = al;
            if (ph == kF) bf.ka[tid] = kk * al;
            if (ph != kRe) bf.qt[tid] = cv(r.k3) * gs_own * two_sigmoid_bwd(cv(r.k4));
        } else if (valt) {
            bf.vh[j] = cv(r.v0) * cv(r.v1);
            if (ph != kF) bf.r[j] = fl(r.v4);
        }
    };
    auto store_rows = [&](float *dst, const float4 (&S)[kBRows]) {
#pragma unroll
        for (int m = 0; m < kBRows; ++m) *reinterpret_cast<float4 *>(dst + own(m)) = S[m];
    };
    auto load_rows = [&](const float *src, float4 (&S)[kBRows]) {
#pragma unroll
        for (int m = 0; m < kBRows; ++m) S[m] = ld4(src + own(m));
    };
    // S <- S_t of the staged token, given its r on this thread's columns
    auto update = [&](float4 (&S)[kBRows], const TokBuf &bf, float4 rr) {
        const float4 vv = ld4(&bf.vh[col4]);
#pragma unroll
        for (int m = 0; m < kBRows; ++m) {
            const int i = row_of(m);
            const float al = bf.al[i], kh = bf.kh[i], kk = bf.k[i];
            S[m].x = state_step(S[m].x, al, kh, rr.x, kk, vv.x);
            S[m].y = state_step(S[m].y, al, kh, rr.y, kk, vv.y);
            S[m].z = state_step(S[m].z, al, kh, rr.z, kk, vv.z);
            S[m].w = state_step(S[m].w, al, kh, rr.w, kk, vv.w);
        }
    };
    // warps 4-5: o of token to (column j) from the 16 partials in redB, written to
    // the workspace with this warp's RMS partials (g*dy of that token: gdy)
    auto finish_o = [&](int to, float gdy) {
        float oo = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) oo += sm.redB[u][j];
        orw[(size_t)to * 2 * kBH + j] = oo;
        const float ss = warp_sum(oo * oo), cs = warp_sum(gdy * oo);
        if (lane == 0) *reinterpret_cast<float2 *>(part + (size_t)to * 8 + 2 * (2 * c + warp - 4)) = make_float2(ss, cs);
    };

    // ---- phase F: checkpoints S_0, S_kBC, S_2kBC, ..., and per token o, r and
    // the RMS partials.  Two barriers a token: after the staging, and after the
    // column partials of r_t = (k alpha) S_{t-1} and o_{t-1} = q~_{t-1} S_{t-1}.
    // Every thread then sums the partials of its own four columns of r itself.
    {
        float4 S[kBRows];
        const float *s_in = p.S_in ? p.S_in + (size_t)head * kBD * kBD : nullptr;
#pragma unroll
        for (int m = 0; m < kBRows; ++m) S[m] = s_in ? ld4(s_in + own_full(m)) : make_float4(0.f, 0.f, 0.f, 0.f);
        store_rows(ckpt, S);
        Tok c0 = T_ > 0 ? fetch(0, kF) : Tok{}, c1 = T_ > 1 ? fetch(1, kF) : Tok{};
        Tok c2 = T_ > 2 ? fetch(2, kF) : Tok{}, c3 = T_ > 3 ? fetch(3, kF) : Tok{};
        float gdy_prev = 0.f;                                 // value threads: g*dy of the previous token
        // token t from cx, which then takes token t + 4's inputs (four register
        // sets, used in turn, so that no move waits for a load in flight)
        auto f_token = [&](int t, Tok &cx) {
            TokBuf &cb = sm.tb[t & 1];
            const TokBuf &pb = sm.tb[(t & 1) ^ 1];
            stage(cx, kF, cb);
            const float gdy_cur = cv(cx.v3) * dy_of(cx);
            if (t + 4 < T_) cx = fetch(t + 4, kF);
            __syncthreads();
            {
                float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), o4 = r4;
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = row_of(m);
                    const float a = cb.ka[i];
                    r4.x = fmaf(a, S[m].x, r4.x); r4.y = fmaf(a, S[m].y, r4.y);
                    r4.z = fmaf(a, S[m].z, r4.z); r4.w = fmaf(a, S[m].w, r4.w);
                }
                *reinterpret_cast<float4 *>(&sm.redA[2 * warp + hl][col4]) = r4;
                if (t > 0) {
#pragma unroll
                    for (int m = 0; m < kBRows; ++m) {
                        const float qp = pb.qt[row_of(m)];
                        o4.x = fmaf(qp, S[m].x, o4.x); o4.y = fmaf(qp, S[m].y, o4.y);
                        o4.z = fmaf(qp, S[m].z, o4.z); o4.w = fmaf(qp, S[m].w, o4.w);
                    }
                    *reinterpret_cast<float4 *>(&sm.redB[2 * warp + hl][col4]) = o4;
                }
            }
            __syncthreads();
            float4 rr = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float4 a = ld4(&sm.redA[u][col4]);
                rr.x += a.x; rr.y += a.y; rr.z += a.z; rr.w += a.w;
            }
            if (valt) {
                float rj = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) rj += sm.redA[u][j];
                orw[(size_t)t * 2 * kBH + kBH + j] = rj;
                if (t > 0) finish_o(t - 1, gdy_prev);
                gdy_prev = gdy_cur;
            }
            update(S, cb, rr);
            if ((t + 1) % kBC == 0 && (t + 1) / kBC < NC) store_rows(ckpt + (size_t)((t + 1) / kBC) * mat, S);
        };
        for (int t = 0; t < T_; t += 4) {
            f_token(t, c0);
            if (t + 1 < T_) f_token(t + 1, c1);
            if (t + 2 < T_) f_token(t + 2, c2);
            if (t + 3 < T_) f_token(t + 3, c3);
        }
        if (T_ > 0) {                                          // o of the last token
            const TokBuf &lb = sm.tb[(T_ - 1) & 1];
            float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int m = 0; m < kBRows; ++m) {
                const float qp = lb.qt[row_of(m)];
                o4.x = fmaf(qp, S[m].x, o4.x); o4.y = fmaf(qp, S[m].y, o4.y);
                o4.z = fmaf(qp, S[m].z, o4.z); o4.w = fmaf(qp, S[m].w, o4.w);
            }
            __syncthreads();                                   // warps 4-5 are done with redB
            *reinterpret_cast<float4 *>(&sm.redB[2 * warp + hl][col4]) = o4;
            __syncthreads();
            if (valt) finish_o(T_ - 1, gdy_prev);
        }
    }
    // both CTAs' RMS partials are in the workspace before either reads them; the
    // checkpoints are visible to the bulk copies that read state 0 of each chunk
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    tc::cluster_sync();

    // ---- phase B.  The running dS of this thread's elements (its rows, its four
    // columns) stays in registers: no other thread reads them.
    float4 dS[kBRows];
    {
        const float *ds_out = p.dS_out ? p.dS_out + (size_t)head * kBD * kBD : nullptr;
#pragma unroll
        for (int m = 0; m < kBRows; ++m) dS[m] = ds_out ? ld4(ds_out + own_full(m)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float dgam = 0.f;                                          // this CTA's share of d gamma_stat, channel tid (tid < 128)
    for (int ch = NC - 1; ch >= 0; --ch) {
        const int t0 = ch * kBC, t1 = min(T_, t0 + kBC);
        // The chunk's states: state s is S before token t0 + s (state 0 is the
        // checkpoint), s = 0 .. n.  The recompute (one barrier a token, with each
        // token's r from phase F) writes each state to slot s & 1; states 1 .. n-2
        // go on to the chunk buffer.  The walk keeps state n in registers, finds
        // state n-1 still in its slot and loads states n-2 .. 0 back one token
        // ahead (state 0 from the checkpoint).
        const int n = t1 - t0;
        float4 S[kBRows];
        {
            load_rows(ckpt + (size_t)ch * mat, S);
            store_rows(slot(0), S);
            Tok c0 = fetch(t0, kRe), c1 = t0 + 1 < t1 ? fetch(t0 + 1, kRe) : Tok{};
            Tok c2 = t0 + 2 < t1 ? fetch(t0 + 2, kRe) : Tok{}, c3 = t0 + 3 < t1 ? fetch(t0 + 3, kRe) : Tok{};
            auto r_token = [&](int t, Tok &cx) {
                const int st = t - t0 + 1;                     // the state this token makes
                TokBuf &cb = sm.tb[t & 1];
                stage(cx, kRe, cb);
                if (t + 4 < t1) cx = fetch(t + 4, kRe);
                if (tid == 0) tc::bulk_wait_read();            // slot st & 1 has been read out
                __syncthreads();
                if (tid == 0 && st - 1 >= 1 && st - 1 <= n - 2) {
                    tc::bulk_s2g(chunk + (size_t)(st - 1) * mat, s_slot0 + ((st - 1) & 1) * kSlotBytes, kSlotBytes);
                    tc::bulk_commit();
                }
                update(S, cb, ld4(&cb.r[col4]));
                store_rows(slot(st & 1), S);
                tc::fence_proxy_async();
            };
            for (int t = t0; t < t1; t += 4) {
                r_token(t, c0);
                if (t + 1 < t1) r_token(t + 1, c1);
                if (t + 2 < t1) r_token(t + 2, c2);
                if (t + 3 < t1) r_token(t + 3, c3);
            }
        }
        Tok n0 = fetch(t1 - 1, kWalk), n1 = t1 - 2 >= t0 ? fetch(t1 - 2, kWalk) : Tok{};
        // this thread's rows of S_t and S_{t-1}, held in registers for the whole
        // token; walking backward, S_{t-1} of one token is S_t of the next
        float4 stv[kBRows], spv[kBRows];
#pragma unroll
        for (int m = 0; m < kBRows; ++m) stv[m] = S[m];
        if (tid == 0) tc::bulk_wait_all();                     // the chunk buffer holds states 1 .. n-2
        __syncthreads();                                       // the recompute's last token is read before it is staged again
        auto w_token = [&](int t, Tok &cx) {
            const int st = t - t0;                             // S_{t-1} is state st
            if (tid == kLoader && st >= 1) {                   // state st - 1, for the next token
                const int x = (st - 1) & 1;
                const float *src = st - 1 == 0 ? ckpt + (size_t)ch * mat : chunk + (size_t)(st - 1) * mat;
                tc::fence_proxy_async();
                tc::mbar_arrive_expect_tx(s_mb + 8 * x, kSlotBytes);
                tc::bulk_g2s(s_slot0 + x * kSlotBytes, src, kSlotBytes, s_mb + 8 * x);
            }
            TokBuf &cb = sm.tb[t & 1];
            const Tok cur = cx;                                // token t (also read by steps 4 and 6)
            const size_t gt = ((size_t)bb * T_ + t) * H + h;
            stage(cur, kWalk, cb);
            // (2) the value side of column j: the RMS norm over both CTAs' columns
            // (the four partial pairs, summed in a fixed order), do and dg
            if (valt) {
                const float ss = ((cur.pa.x + cur.pa.z) + cur.pb.x) + cur.pb.z;
                const float cs = ((cur.pa.y + cur.pa.w) + cur.pb.y) + cur.pb.w;
                const float rho = rsqrtf(ss / kBD + p.eps), oo = fl(cur.v5), dyv = dy_of(cur);
                cb.dO[j] = rho * (cv(cur.v3) * dyv) - rho * rho * rho / kBD * oo * cs;
                p.grad_g[gt * kBD + gc0 + j] = dyv * oo * rho;
            }
            if (t - 2 >= t0) cx = fetch(t - 2, kWalk);
            __syncthreads();
            // (3) dS += q~^T do; dq~ = S_t do^T (rows); k dS and (b*k) dS (columns)
            {
                const float4 d4 = ld4(&cb.dO[col4]);
                float rowv[kBRows];
                float4 cA = make_float4(0.f, 0.f, 0.f, 0.f), cB = cA;
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = row_of(m);
                    const float4 st = stv[m];
                    rowv[m] = dot4(st, d4);
                    float4 ds = dS[m];
                    const float a = cb.qt[i];
                    ds.x = fmaf(a, d4.x, ds.x); ds.y = fmaf(a, d4.y, ds.y);
                    ds.z = fmaf(a, d4.z, ds.z); ds.w = fmaf(a, d4.w, ds.w);
                    dS[m] = ds;
                    const float kk = cb.k[i], kh = cb.kh[i];
                    cA.x = fmaf(kk, ds.x, cA.x); cA.y = fmaf(kk, ds.y, cA.y);
                    cA.z = fmaf(kk, ds.z, cA.z); cA.w = fmaf(kk, ds.w, cA.w);
                    cB.x = fmaf(kh, ds.x, cB.x); cB.y = fmaf(kh, ds.y, cB.y);
                    cB.z = fmaf(kh, ds.z, cB.z); cB.w = fmaf(kh, ds.w, cB.w);
                }
                const float rs = rows_reduce_scatter8(rowv, lane);
                if ((lane & 1) == 0) sm.rows[0][row_of((lane >> 1) & 7)] = rs;
                *reinterpret_cast<float4 *>(&sm.redA[2 * warp + hl][col4]) = cA;
                *reinterpret_cast<float4 *>(&sm.redB[2 * warp + hl][col4]) = cB;
            }
            __syncthreads();
            // (4) dv^ and dr on this CTA's columns; dv, dw
            if (valt) {
                float sa = 0.f, sb = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    sa += sm.redA[u][j];
                    sb += sm.redB[u][j];
                }
                sm.dr[j] = -sb;
                const size_t gj = gt * kBD + gc0 + j;
                p.grad_v[gj] = cv(cur.v0) * sa;
                p.grad_w[gj] = cv(cur.v1) * sa;
            }
            __syncthreads();
            // (5) row sums dS v^T, -dS r^T, S_{t-1} dr^T, (dS + k^T dr) * S_{t-1}; dS <- Diag(alpha) dS_hat
            if (st <= n - 2) wait_slot(st & 1);
            load_rows(slot(st & 1), spv);
            {
                const float4 vv = ld4(&cb.vh[col4]), rr = ld4(&cb.r[col4]), dd = ld4(&sm.dr[col4]);
                float ra[kBRows], rb[kBRows], rc[kBRows], rd[kBRows];
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = row_of(m);
                    const float4 sp = spv[m];
                    float4 ds = dS[m];
                    ra[m] = dot4(ds, vv);
                    rb[m] = -dot4(ds, rr);
                    rc[m] = dot4(sp, dd);
                    const float kk = cb.k[i], al = cb.al[i];
                    ds.x = fmaf(kk, dd.x, ds.x); ds.y = fmaf(kk, dd.y, ds.y);
                    ds.z = fmaf(kk, dd.z, ds.z); ds.w = fmaf(kk, dd.w, ds.w);
                    rd[m] = dot4(ds, sp);
                    ds.x *= al; ds.y *= al; ds.z *= al; ds.w *= al;
                    dS[m] = ds;
                }
                const int ri = row_of((lane >> 1) & 7);
                const float sa = rows_reduce_scatter8(ra, lane), sb = rows_reduce_scatter8(rb, lane);
                const float sc = rows_reduce_scatter8(rc, lane), sd = rows_reduce_scatter8(rd, lane);
                if ((lane & 1) == 0) {
                    sm.rows[1][ri] = sa;
                    sm.rows[2][ri] = sb;
                    sm.rows[3][ri] = sc;
                    sm.rows[4][ri] = sd;
                }
            }
            __syncthreads();
            // (6) this CTA's share of token t's key-side gradients (the other CTA adds its share)
            if (keyt) {
                const size_t gi = gt * kBD + tid;
                const float kk = cb.k[tid], al = cb.al[tid];
                const float bv = cv(cur.k2), qv = cv(cur.k3), zv = cv(cur.k4);
                const float ts = two_sigmoid_bwd(zv);
                const float dqt = sm.rows[0][tid], dkh = sm.rows[2][tid];
                red_add(p.grad_k + gi, sm.rows[1][tid] + al * sm.rows[3][tid] + bv * dkh);
                red_add(p.grad_b + gi, kk * dkh);
                red_add(p.grad_la + gi, al * sm.rows[4][tid]);
                red_add(p.grad_q + gi, dqt * gs_own * ts);
                red_add(p.grad_z + gi, dqt * qv * gs_own * ts * (1.f - 0.5f * ts));
                dgam = fmaf(dqt * qv, ts, dgam);
            }
#pragma unroll
            for (int m = 0; m < kBRows; ++m) stv[m] = spv[m];
        };
        for (int t = t1 - 1; t >= t0; t -= 2) {
            w_token(t, n0);
            if (t - 1 >= t0) w_token(t - 1, n1);
        }
    }
    __syncthreads();
    if (p.grad_S_in) {
#pragma unroll
        for (int m = 0; m < kBRows; ++m)
            *reinterpret_cast<float4 *>(p.grad_S_in + (size_t)head * kBD * kBD + own_full(m)) = dS[m];
    }
    if (keyt) p.ws_dgam[hc * kBD + tid] = dgam;
}

// d gamma_stat[h] = sum over the batch rows and both value halves of the per-CTA partials
__global__ void __launch_bounds__(kBD) gdn2_bwd_dgamma_kernel(const float *part, float *out, int B, int H) {
    const int h = blockIdx.x, i = threadIdx.x;
    float s = 0.f;
    for (int bb = 0; bb < B; ++bb)
        for (int c = 0; c < 2; ++c) s += part[(((size_t)bb * H + h) * 2 + c) * kBD + i];
    out[(size_t)h * kBD + i] = s;
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int T) {
    const size_t mat = (size_t)kBD * kBH * sizeof(float);          // one half-matrix
    const size_t NC = (size_t)(T + kBC - 1) / kBC;
    const size_t BH = (size_t)B * H;
    return BH * 2 * ((NC + 1) * mat + (kBC + 1) * mat + kBD * sizeof(float)) + BH * (size_t)T * 8 * sizeof(float) +
           BH * 2 * (size_t)T * 2 * kBH * sizeof(float);
}

cudaError_t launch_bwd(BwdParams p, void *workspace, int dtype, cudaStream_t stream) {
    const size_t mat = (size_t)kBD * kBH;
    const size_t BH = (size_t)p.B * p.H;
    const size_t NC = (size_t)(p.T + kBC - 1) / kBC;
    float *ws = (float *)workspace;
    p.ws_ckpt = ws;
    p.ws_chunk = p.ws_ckpt + BH * 2 * (NC + 1) * mat;
    p.ws_dgam = p.ws_chunk + BH * 2 * (kBC + 1) * mat;
    p.ws_part = p.ws_dgam + BH * 2 * kBD;
    p.ws_or = p.ws_part + BH * (size_t)p.T * 8;
    // the key-side gradients are accumulated by the two CTAs of each head
    const size_t ntok = BH * (size_t)p.T * kBD * sizeof(float);
    cudaError_t e = cudaSuccess;
    if (ntok) {
        float *const acc[] = {p.grad_k, p.grad_b, p.grad_la, p.grad_q, p.grad_z};
        for (float *a : acc) {
            e = cudaMemsetAsync(a, 0, ntok, stream);
            if (e != cudaSuccess) return e;
        }
    }
    // two state tiles and three mbarriers (the slots' and the failure-test one)
    const size_t dsm = 2 * (size_t)kSlotBytes + 24;
    if (dtype == GDELTA_BF16) {
        e = cudaFuncSetAttribute(gdn2_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm);
        if (e != cudaSuccess) return e;
        gdn2_bwd_kernel<__nv_bfloat16><<<(unsigned)(2 * BH), kBT, dsm, stream>>>(p);
    } else {
        e = cudaFuncSetAttribute(gdn2_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm);
        if (e != cudaSuccess) return e;
        gdn2_bwd_kernel<float><<<(unsigned)(2 * BH), kBT, dsm, stream>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess || !p.grad_gs) return e;
    gdn2_bwd_dgamma_kernel<<<(unsigned)p.H, kBD, 0, stream>>>(p.ws_dgam, p.grad_gs, p.B, p.H);
    return cudaGetLastError();
}

}  // namespace gdelta
