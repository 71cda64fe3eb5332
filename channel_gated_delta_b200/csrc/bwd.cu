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
//      (zeroed by the launcher) with atomics: two addends to a zero, so the
//      result does not depend on their order.
//
// Phase F runs the recurrence forward and keeps the state every kBC tokens
// (checkpoints).  Phase B walks the chunks from the last: it recomputes the
// chunk's kBC + 1 states from its checkpoint into a per-CTA buffer, then takes
// the tokens in reverse with the exact per-token gradient recurrence below.
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
// alpha = exp(log_alpha).  The checkpoints, chunk states and RMS partials live
// in the caller's workspace; the running dS (this CTA's half) lives in shared
// memory.
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

__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

struct BwdSmem {
    float k[kBD], kh[kBD], ka[kBD], al[kBD], qt[kBD], qtp[kBD];   // token vectors, key side (qtp: previous token's q~)
    float vh[kBH], gdy[kBH], gdyp[kBH], r[kBH], dO[kBH], dr[kBH];   // value side, this CTA's columns
    float redA[16][kBH], redB[16][kBH];                      // column partials per (warp, half)
    float rows[5][kBD];                                      // row sums over this CTA's columns
    float2 part[4];                                          // this token's RMS partials (both CTAs)
};

template <typename T>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kBT, 1) gdn2_bwd_kernel(BwdParams p) {
    __shared__ BwdSmem sm;
    extern __shared__ float4 sdS[];                          // running dS of this CTA's columns, [row][16]
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
    const T *q = (const T *)p.q, *k = (const T *)p.k, *z = (const T *)p.z, *b = (const T *)p.b;
    const T *v = (const T *)p.v, *w = (const T *)p.w, *g = (const T *)p.g;
    auto row_of = [&](int m) { return warp + 8 * hl + 16 * m; };
    auto own = [&](int m) { return (size_t)row_of(m) * kBH + col4; };           // in a half-matrix buffer
    auto own_full = [&](int m) { return (size_t)row_of(m) * kBD + gc0 + col4; };  // in a [128][128] matrix

    // Token t's inputs for this thread, fetched into registers two tokens ahead
    // of use: threads 0-127 the key side of channel tid (k, log alpha, b, q, z),
    // threads 128-191 the value side of this CTA's column tid - 128 (w, v, dy,
    // g), and in phase B threads 0-7 the token's eight RMS partials.  The
    // gradient step reads the same registers again instead of reloading.
    struct Tok {
        float x0, x1, x2, x3, x4, x5;
    };
    const float gs_own = (tid < kBD && p.gs) ? p.gs[(size_t)h * kBD + tid] : 1.f;
    auto fetch = [&](int t, bool with_part) -> Tok {
        Tok r{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const size_t gt = ((size_t)bb * T_ + t) * H + h;
        if (tid < kBD) {
            const size_t gi = gt * kBD + tid;
            r.x0 = ldf(k, gi);
            r.x1 = p.la[gi];
            r.x2 = ldf(b, gi);
            r.x3 = ldf(q, gi);
            r.x4 = ldf(z, gi);
            if (with_part && tid < 8) r.x5 = part[(size_t)t * 8 + tid];
        } else if (tid < kBD + kBH) {
            const size_t gj = gt * kBD + gc0 + (tid - kBD);
            r.x0 = ldf(w, gj);
            r.x1 = ldf(v, gj);
            r.x2 = p.dy ? p.dy[gj] : 0.f;
            r.x3 = ldf(g, gj);
        }
        return r;
    };
    // the token's vectors into shared memory (the caller syncs before and after);
    // keep_prev: first move this token's predecessor's q~ and g*dy aside (phase F
    // reduces o of the previous token with the next token's r)
    auto stage = [&](const Tok &r, bool keep_prev, bool with_part) {
        if (tid < kBD) {
            if (keep_prev) sm.qtp[tid] = sm.qt[tid];
            const float kk = r.x0, al = expf(r.x1);
            sm.k[tid] = kk;
            sm.kh[tid] = r.x2 * kk;
            sm.ka[tid] = kk * al;
            sm.al[tid] = al;
            sm.qt[tid] = r.x3 * gs_own * two_sigmoid(r.x4);
            if (with_part && tid < 8) reinterpret_cast<float *>(sm.part)[tid] = r.x5;
        } else if (tid < kBD + kBH) {
            const int j = tid - kBD;
            if (keep_prev) sm.gdyp[j] = sm.gdy[j];
            sm.vh[j] = r.x0 * r.x1;
            sm.gdy[j] = r.x3 * r.x2;
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
    // r = (k alpha) S (column sums over the rows) and, when o_tok >= 0, o of the
    // previous token, q~_prev S, whose RMS partials go to the workspace; then,
    // when update, the state step of the staged token
    auto fwd_step = [&](float4 (&S)[kBRows], int o_tok, bool update) {
        float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), o4 = r4;
#pragma unroll
        for (int m = 0; m < kBRows; ++m) {
            const int i = row_of(m);
            const float a = sm.ka[i], qp = sm.qtp[i];
            r4.x = fmaf(a, S[m].x, r4.x); r4.y = fmaf(a, S[m].y, r4.y);
            r4.z = fmaf(a, S[m].z, r4.z); r4.w = fmaf(a, S[m].w, r4.w);
            o4.x = fmaf(qp, S[m].x, o4.x); o4.y = fmaf(qp, S[m].y, o4.y);
            o4.z = fmaf(qp, S[m].z, o4.z); o4.w = fmaf(qp, S[m].w, o4.w);
        }
        *reinterpret_cast<float4 *>(&sm.redA[2 * warp + hl][col4]) = r4;
        if (o_tok >= 0) *reinterpret_cast<float4 *>(&sm.redB[2 * warp + hl][col4]) = o4;
        __syncthreads();
        if (tid < kBH) {
            float s = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) s += sm.redA[u][tid];
            sm.r[tid] = s;
            if (o_tok >= 0) {                                  // warps 0 and 1: this CTA's 64 columns of o
                float oo = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) oo += sm.redB[u][tid];
                const float ss = warp_sum(oo * oo), cs = warp_sum(sm.gdyp[tid] * oo);
                if (lane == 0)
                    *reinterpret_cast<float2 *>(part + (size_t)o_tok * 8 + 2 * (2 * c + warp)) = make_float2(ss, cs);
            }
        }
        __syncthreads();
        if (!update) return;
        const float4 rr = ld4(&sm.r[col4]), vv = ld4(&sm.vh[col4]);
#pragma unroll
        for (int m = 0; m < kBRows; ++m) {
            const int i = row_of(m);
            const float al = sm.al[i], kh = sm.kh[i], kk = sm.k[i];
            S[m].x = al * S[m].x - kh * rr.x + kk * vv.x;
            S[m].y = al * S[m].y - kh * rr.y + kk * vv.y;
            S[m].z = al * S[m].z - kh * rr.z + kk * vv.z;
            S[m].w = al * S[m].w - kh * rr.w + kk * vv.w;
        }
    };

    // ---- phase F: checkpoints S_0, S_kBC, S_2kBC, ... and the RMS partials of every token
    {
        float4 S[kBRows];
        const float *s_in = p.S_in ? p.S_in + (size_t)head * kBD * kBD : nullptr;
#pragma unroll
        for (int m = 0; m < kBRows; ++m) S[m] = s_in ? ld4(s_in + own_full(m)) : make_float4(0.f, 0.f, 0.f, 0.f);
        store_rows(ckpt, S);
        Tok c0 = T_ > 0 ? fetch(0, false) : Tok{}, c1 = T_ > 1 ? fetch(1, false) : Tok{};
        for (int t = 0; t < T_; ++t) {
            __syncthreads();
            stage(c0, true, false);
            c0 = c1;
            if (t + 2 < T_) c1 = fetch(t + 2, false);
            __syncthreads();
            fwd_step(S, t - 1, true);                          // r of token t, o of token t - 1
            if ((t + 1) % kBC == 0 && (t + 1) / kBC < NC) store_rows(ckpt + (size_t)((t + 1) / kBC) * mat, S);
        }
        if (T_ > 0) {                                          // o of the last token
            __syncthreads();
            if (tid < kBD) sm.qtp[tid] = sm.qt[tid];
            else if (tid < kBD + kBH) sm.gdyp[tid - kBD] = sm.gdy[tid - kBD];
            __syncthreads();
            fwd_step(S, T_ - 1, false);
        }
    }
    // both CTAs' RMS partials are in the workspace before either reads them
    __threadfence();
    tc::cluster_sync();

    // ---- phase B
    {
        const float *ds_out = p.dS_out ? p.dS_out + (size_t)head * kBD * kBD : nullptr;
#pragma unroll
        for (int m = 0; m < kBRows; ++m)
            sdS[row_of(m) * 16 + lc] = ds_out ? ld4(ds_out + own_full(m)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float dgam = 0.f;                                          // this CTA's share of d gamma_stat, channel tid (tid < 128)
    for (int ch = NC - 1; ch >= 0; --ch) {
        const int t0 = ch * kBC, t1 = min(T_, t0 + kBC);
        {   // the chunk's states S_{t0} .. S_{t1}
            float4 S[kBRows];
            load_rows(ckpt + (size_t)ch * mat, S);
            store_rows(chunk, S);
            Tok c0 = fetch(t0, false), c1 = t0 + 1 < t1 ? fetch(t0 + 1, false) : Tok{};
            for (int t = t0; t < t1; ++t) {
                __syncthreads();
                stage(c0, false, false);
                c0 = c1;
                if (t + 2 < t1) c1 = fetch(t + 2, false);
                __syncthreads();
                fwd_step(S, -1, true);
                store_rows(chunk + (size_t)(t - t0 + 1) * mat, S);
            }
        }
        Tok n0 = fetch(t1 - 1, true), n1 = t1 - 2 >= t0 ? fetch(t1 - 2, true) : Tok{};
        // this thread's rows of S_t and S_{t-1}, held in registers for the whole
        // token; walking backward, S_{t-1} of one token is S_t of the next, so each
        // token loads one state (issued before its barriers)
        float4 stv[kBRows], spv[kBRows];
        load_rows(chunk + (size_t)(t1 - t0) * mat, stv);
        for (int t = t1 - 1; t >= t0; --t) {
            load_rows(chunk + (size_t)(t - t0) * mat, spv);
            __syncthreads();
            const Tok cur = n0;                                // token t (also read by steps 2, 4 and 6)
            stage(cur, false, true);
            n0 = n1;
            if (t - 2 >= t0) n1 = fetch(t - 2, true);
            __syncthreads();
            const size_t gt = ((size_t)bb * T_ + t) * H + h;
            // (1) o = q~ S_t and r = (k alpha) S_{t-1}: column partials
            {
                float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f), r4 = o4;
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = row_of(m);
                    const float4 st = stv[m], sp = spv[m];
                    const float a = sm.qt[i], c2 = sm.ka[i];
                    o4.x = fmaf(a, st.x, o4.x); o4.y = fmaf(a, st.y, o4.y);
                    o4.z = fmaf(a, st.z, o4.z); o4.w = fmaf(a, st.w, o4.w);
                    r4.x = fmaf(c2, sp.x, r4.x); r4.y = fmaf(c2, sp.y, r4.y);
                    r4.z = fmaf(c2, sp.z, r4.z); r4.w = fmaf(c2, sp.w, r4.w);
                }
                *reinterpret_cast<float4 *>(&sm.redA[2 * warp + hl][col4]) = o4;
                *reinterpret_cast<float4 *>(&sm.redB[2 * warp + hl][col4]) = r4;
            }
            __syncthreads();
            // (2) the value side of column j: o and r, the RMS norm over both CTAs'
            // columns (the four partial pairs, summed in a fixed order), do and dg
            if (tid >= kBD && tid < kBD + kBH) {
                const int j = tid - kBD;
                float oo = 0.f, sr = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    oo += sm.redA[u][j];
                    sr += sm.redB[u][j];
                }
                sm.r[j] = sr;
                const float *pp = reinterpret_cast<const float *>(sm.part);
                const float ss = ((pp[0] + pp[2]) + pp[4]) + pp[6], cs = ((pp[1] + pp[3]) + pp[5]) + pp[7];
                const float rho = rsqrtf(ss / kBD + p.eps);
                sm.dO[j] = rho * sm.gdy[j] - rho * rho * rho / kBD * oo * cs;
                p.grad_g[gt * kBD + gc0 + j] = cur.x2 * oo * rho;
            }
            __syncthreads();
            // (3) dS += q~^T do; dq~ = S_t do^T (rows); k dS and (b*k) dS (columns)
            {
                const float4 d4 = ld4(&sm.dO[col4]);
                float rowv[kBRows];
                float4 cA = make_float4(0.f, 0.f, 0.f, 0.f), cB = cA;
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = row_of(m);
                    const float4 st = stv[m];
                    rowv[m] = dot4(st, d4);
                    float4 ds = sdS[i * 16 + lc];
                    const float a = sm.qt[i];
                    ds.x = fmaf(a, d4.x, ds.x); ds.y = fmaf(a, d4.y, ds.y);
                    ds.z = fmaf(a, d4.z, ds.z); ds.w = fmaf(a, d4.w, ds.w);
                    sdS[i * 16 + lc] = ds;
                    const float kk = sm.k[i], kh = sm.kh[i];
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
            if (tid >= kBD && tid < kBD + kBH) {
                const int j = tid - kBD;
                float sa = 0.f, sb = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    sa += sm.redA[u][j];
                    sb += sm.redB[u][j];
                }
                sm.dr[j] = -sb;
                const size_t gj = gt * kBD + gc0 + j;
                p.grad_v[gj] = cur.x0 * sa;
                p.grad_w[gj] = cur.x1 * sa;
            }
            __syncthreads();
            // (5) row sums dS v^T, -dS r^T, S_{t-1} dr^T, (dS + k^T dr) * S_{t-1}; dS <- Diag(alpha) dS_hat
            {
                const float4 vv = ld4(&sm.vh[col4]), rr = ld4(&sm.r[col4]), dd = ld4(&sm.dr[col4]);
                float ra[kBRows], rb[kBRows], rc[kBRows], rd[kBRows];
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = row_of(m);
                    const float4 sp = spv[m];
                    float4 ds = sdS[i * 16 + lc];
                    ra[m] = dot4(ds, vv);
                    rb[m] = -dot4(ds, rr);
                    rc[m] = dot4(sp, dd);
                    const float kk = sm.k[i], al = sm.al[i];
                    ds.x = fmaf(kk, dd.x, ds.x); ds.y = fmaf(kk, dd.y, ds.y);
                    ds.z = fmaf(kk, dd.z, ds.z); ds.w = fmaf(kk, dd.w, ds.w);
                    rd[m] = dot4(ds, sp);
                    ds.x *= al; ds.y *= al; ds.z *= al; ds.w *= al;
                    sdS[i * 16 + lc] = ds;
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
            if (tid < kBD) {
                const size_t gi = gt * kBD + tid;
                const float kk = sm.k[tid], al = sm.al[tid];
                const float bv = cur.x2, qv = cur.x3, zv = cur.x4;
                const float ts = two_sigmoid(zv);
                const float dqt = sm.rows[0][tid], dkh = sm.rows[2][tid];
                atomicAdd(p.grad_k + gi, sm.rows[1][tid] + al * sm.rows[3][tid] + bv * dkh);
                atomicAdd(p.grad_b + gi, kk * dkh);
                atomicAdd(p.grad_la + gi, al * sm.rows[4][tid]);
                atomicAdd(p.grad_q + gi, dqt * gs_own * ts);
                atomicAdd(p.grad_z + gi, dqt * qv * gs_own * ts * (1.f - 0.5f * ts));
                dgam = fmaf(dqt * qv, ts, dgam);
            }
#pragma unroll
            for (int m = 0; m < kBRows; ++m) stv[m] = spv[m];
        }
    }
    __syncthreads();
    if (p.grad_S_in) {
#pragma unroll
        for (int m = 0; m < kBRows; ++m)
            *reinterpret_cast<float4 *>(p.grad_S_in + (size_t)head * kBD * kBD + own_full(m)) = sdS[row_of(m) * 16 + lc];
    }
    if (tid < kBD) p.ws_dgam[hc * kBD + tid] = dgam;
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
    return BH * 2 * ((NC + 1) * mat + (kBC + 1) * mat + kBD * sizeof(float)) + BH * (size_t)T * 8 * sizeof(float);
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
    const size_t dsm = (size_t)kBD * kBH * sizeof(float);           // running dS of one CTA's columns
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
