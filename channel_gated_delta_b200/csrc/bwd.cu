// Backward pass of the token mixer (fp32 CUDA cores, d_k = d_v = 128): the
// gradient of a loss with respect to every input, the static readout profile
// and the initial state, given its gradient with respect to y (and optionally
// the final state).
//
// One CTA per (batch, head).  Phase F runs the recurrence forward and keeps
// the state every kBC tokens (checkpoints).  Phase B walks the chunks from the
// last: it recomputes the chunk's kBC + 1 states from its checkpoint into a
// per-head buffer, then takes the tokens in reverse with the exact per-token
// gradient recurrence below.  Per token, with S_hat = Diag(alpha) S_{t-1},
// r = k S_hat, S_t = S_hat - (b*k)^T r + k^T (w*v), o = q~ S_t and
// y = g * o * rho, rho = 1 / sqrt(mean(o^2) + eps) (Muir review §2.1):
//
//   do      = rho (g*dy) - rho^3 / d_v * o * sum(g*dy*o)        dg = dy * o * rho
//   dS     += q~^T do                                          dq~ = S_t do^T
//   dv^     = k dS            dr = -(b*k) dS                   d(b*k) = -dS r^T
//   dk      = dS v^T + Diag(alpha) S_{t-1} dr^T + b * d(b*k)   db = k * d(b*k)
//   dS_hat  = dS + k^T dr     dalpha = rowsum(dS_hat * S_{t-1}) dS_{t-1} = Diag(alpha) dS_hat
//
// and the chain rule through q~ = q * gamma * 2 sigmoid(z), v^ = w * v,
// alpha = exp(log_alpha).  The checkpoints and chunk states live in the
// caller's workspace; the running dS lives in shared memory.
//
// Thread layout (256 threads): warp w holds rows w + 8 m (m = 0..15) of every
// d_k x d_v matrix, lane l columns 4l..4l+3, so a row's sum is a warp
// reduction and a column's sum a reduction over the 8 warps.
#include "common.cuh"

namespace gdelta {

namespace {

constexpr int kBD = 128;             // d_k = d_v
constexpr int kBT = 256;             // threads
constexpr int kBRows = 16;           // rows per thread
constexpr int kBC = 32;              // tokens per checkpoint

// Warp reduce-scatter of 16 per-lane values: afterwards lane l holds the sum
// over the warp's 32 lanes of value (l >> 1) & 15.
__device__ __forceinline__ float rows_reduce_scatter(const float (&v)[16], int lane) {
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
    const float keep = b1 ? w2[1] : w2[0], send = b1 ? w2[0] : w2[1];
    const float w1 = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    return w1 + __shfl_xor_sync(0xffffffffu, w1, 1);
}

__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

struct BwdSmem {
    float k[kBD], kh[kBD], ka[kBD], al[kBD], qt[kBD];      // token vectors, key side
    float vh[kBD], gdy[kBD], o[kBD], r[kBD], dO[kBD], dr[kBD];
    float redA[8][kBD], redB[8][kBD];                       // column partials per warp
    float rows[5][kBD];                                      // row sums
    float scal[2];
};

template <typename T>
__global__ void __launch_bounds__(kBT, 1) gdn2_bwd_kernel(BwdParams p) {
    __shared__ BwdSmem sm;
    extern __shared__ float4 sdS[];                          // running dS, [row][lane]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int head = blockIdx.x, h = head % p.H, bb = head / p.H;
    const int T_ = p.T, H = p.H;
    const int NC = (T_ + kBC - 1) / kBC;
    const size_t mat = (size_t)kBD * kBD;
    float *ckpt = p.ws_ckpt + (size_t)head * (NC + 1) * mat;
    float *chunk = p.ws_chunk + (size_t)head * (kBC + 1) * mat;
    const T *q = (const T *)p.q, *k = (const T *)p.k, *z = (const T *)p.z, *b = (const T *)p.b;
    const T *v = (const T *)p.v, *w = (const T *)p.w, *g = (const T *)p.g;
    const size_t own = (size_t)warp * kBD + 4 * lane;       // this thread's row warp, columns 4 lane..

    // forward step of the recurrence on this thread's state rows (key-side
    // vectors k, kh = b*k, ka = k*alpha, al = alpha and v^ already in shared memory)
    auto fwd_step = [&](float4 (&S)[kBRows]) {
        float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < kBRows; ++m) {
            const float a = sm.ka[warp + 8 * m];
            r4.x = fmaf(a, S[m].x, r4.x); r4.y = fmaf(a, S[m].y, r4.y);
            r4.z = fmaf(a, S[m].z, r4.z); r4.w = fmaf(a, S[m].w, r4.w);
        }
        *reinterpret_cast<float4 *>(&sm.redA[warp][4 * lane]) = r4;
        __syncthreads();
        if (tid < kBD) {
            float s = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) s += sm.redA[u][tid];
            sm.r[tid] = s;
        }
        __syncthreads();
        const float4 rr = ld4(&sm.r[4 * lane]), vv = ld4(&sm.vh[4 * lane]);
#pragma unroll
        for (int m = 0; m < kBRows; ++m) {
            const int i = warp + 8 * m;
            const float al = sm.al[i], kh = sm.kh[i], kk = sm.k[i];
            S[m].x = al * S[m].x - kh * rr.x + kk * vv.x;
            S[m].y = al * S[m].y - kh * rr.y + kk * vv.y;
            S[m].z = al * S[m].z - kh * rr.z + kk * vv.z;
            S[m].w = al * S[m].w - kh * rr.w + kk * vv.w;
        }
    };
    // Token t's inputs for this thread's channel, fetched into registers ahead of
    // use (two tokens ahead in every pass, so a token's loads are in flight while
    // the two before it are processed): threads 0-127 the key side of channel
    // tid (k, log alpha, b, q, z), threads 128-255 the value side of channel
    // tid - 128 (w, v, dy, g).  The backward step reads the same registers again
    // instead of reloading.
    struct Tok {
        float x0, x1, x2, x3, x4;
    };
    const float gs_own = (tid < kBD && p.gs) ? p.gs[(size_t)h * kBD + tid] : 1.f;
    auto fetch = [&](int t) -> Tok {
        Tok r{0.f, 0.f, 0.f, 0.f, 0.f};
        const size_t gt = ((size_t)bb * T_ + t) * H + h;
        if (tid < kBD) {
            const size_t gi = gt * kBD + tid;
            r.x0 = ldf(k, gi);
            r.x1 = p.la[gi];
            r.x2 = ldf(b, gi);
            r.x3 = ldf(q, gi);
            r.x4 = ldf(z, gi);
        } else {
            const size_t gj = gt * kBD + (tid - kBD);
            r.x0 = ldf(w, gj);
            r.x1 = ldf(v, gj);
            r.x2 = p.dy ? p.dy[gj] : 0.f;
            r.x3 = ldf(g, gj);
        }
        return r;
    };
    // the token's key-side and value-side vectors into shared memory (the caller
    // syncs before, so that the previous token's are no longer read, and after)
    auto stage = [&](const Tok &r) {
        if (tid < kBD) {
            const float kk = r.x0, al = expf(r.x1);
            sm.k[tid] = kk;
            sm.kh[tid] = r.x2 * kk;
            sm.ka[tid] = kk * al;
            sm.al[tid] = al;
            sm.qt[tid] = r.x3 * gs_own * two_sigmoid(r.x4);
        } else {
            const int j = tid - kBD;
            sm.vh[j] = r.x0 * r.x1;
            sm.gdy[j] = r.x3 * r.x2;
        }
    };
    auto store_rows = [&](float *dst, const float4 (&S)[kBRows]) {
#pragma unroll
        for (int m = 0; m < kBRows; ++m) *reinterpret_cast<float4 *>(dst + own + (size_t)8 * m * kBD) = S[m];
    };
    auto load_rows = [&](const float *src, float4 (&S)[kBRows]) {
#pragma unroll
        for (int m = 0; m < kBRows; ++m) S[m] = ld4(src + own + (size_t)8 * m * kBD);
    };

    // ---- phase F: checkpoints S_0, S_kBC, S_2kBC, ...
    {
        float4 S[kBRows];
        const float *s_in = p.S_in ? p.S_in + (size_t)head * mat : nullptr;
#pragma unroll
        for (int m = 0; m < kBRows; ++m)
            S[m] = s_in ? ld4(s_in + own + (size_t)8 * m * kBD) : make_float4(0.f, 0.f, 0.f, 0.f);
        store_rows(ckpt, S);
        Tok c0 = T_ > 0 ? fetch(0) : Tok{}, c1 = T_ > 1 ? fetch(1) : Tok{};
        for (int t = 0; t < T_; ++t) {
            __syncthreads();
            stage(c0);
            c0 = c1;
            if (t + 2 < T_) c1 = fetch(t + 2);
            __syncthreads();
            fwd_step(S);
            if ((t + 1) % kBC == 0 && (t + 1) / kBC < NC) store_rows(ckpt + (size_t)((t + 1) / kBC) * mat, S);
        }
    }

    // ---- phase B
    {
        const float *ds_out = p.dS_out ? p.dS_out + (size_t)head * mat : nullptr;
#pragma unroll
        for (int m = 0; m < kBRows; ++m)
            sdS[(warp + 8 * m) * 32 + lane] = ds_out ? ld4(ds_out + own + (size_t)8 * m * kBD)
                                                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float dgam = 0.f;                                          // d gamma_stat, channel tid (tid < 128)
    for (int c = NC - 1; c >= 0; --c) {
        const int t0 = c * kBC, t1 = min(T_, t0 + kBC);
        {   // the chunk's states S_{t0} .. S_{t1}
            float4 S[kBRows];
            load_rows(ckpt + (size_t)c * mat, S);
            store_rows(chunk, S);
            Tok c0 = fetch(t0), c1 = t0 + 1 < t1 ? fetch(t0 + 1) : Tok{};
            for (int t = t0; t < t1; ++t) {
                __syncthreads();
                stage(c0);
                c0 = c1;
                if (t + 2 < t1) c1 = fetch(t + 2);
                __syncthreads();
                fwd_step(S);
                store_rows(chunk + (size_t)(t - t0 + 1) * mat, S);
            }
        }
        Tok n0 = fetch(t1 - 1), n1 = t1 - 2 >= t0 ? fetch(t1 - 2) : Tok{};
        for (int t = t1 - 1; t >= t0; --t) {
            __syncthreads();
            const Tok cur = n0;                      // token t (also read by steps 2, 4 and 6)
            stage(cur);
            n0 = n1;
            if (t - 2 >= t0) n1 = fetch(t - 2);
            __syncthreads();
            const float *St = chunk + (size_t)(t - t0 + 1) * mat, *Sp = chunk + (size_t)(t - t0) * mat;
            // (1) o = q~ S_t and r = (k alpha) S_{t-1}: column partials
            {
                float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f), r4 = o4;
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = warp + 8 * m;
                    const float4 st = ld4(St + own + (size_t)8 * m * kBD), sp = ld4(Sp + own + (size_t)8 * m * kBD);
                    const float a = sm.qt[i], c2 = sm.ka[i];
                    o4.x = fmaf(a, st.x, o4.x); o4.y = fmaf(a, st.y, o4.y);
                    o4.z = fmaf(a, st.z, o4.z); o4.w = fmaf(a, st.w, o4.w);
                    r4.x = fmaf(c2, sp.x, r4.x); r4.y = fmaf(c2, sp.y, r4.y);
                    r4.z = fmaf(c2, sp.z, r4.z); r4.w = fmaf(c2, sp.w, r4.w);
                }
                *reinterpret_cast<float4 *>(&sm.redA[warp][4 * lane]) = o4;
                *reinterpret_cast<float4 *>(&sm.redB[warp][4 * lane]) = r4;
            }
            __syncthreads();
            if (tid < kBD) {
                float so = 0.f, sr = 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    so += sm.redA[u][tid];
                    sr += sm.redB[u][tid];
                }
                sm.o[tid] = so;
                sm.r[tid] = sr;
            }
            __syncthreads();
            // (2) the RMS norm and output gate: rho and sum(g dy o), then do and dg
            if (warp == 0) {
                float ss = 0.f, cs = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float oo = sm.o[lane + 32 * u];
                    ss = fmaf(oo, oo, ss);
                    cs = fmaf(sm.gdy[lane + 32 * u], oo, cs);
                }
                ss = warp_sum(ss);
                cs = warp_sum(cs);
                if (lane == 0) {
                    sm.scal[0] = rsqrtf(ss / kBD + p.eps);
                    sm.scal[1] = cs;
                }
            }
            __syncthreads();
            if (tid >= kBD) {
                const int j = tid - kBD;
                const float rho = sm.scal[0], oo = sm.o[j];
                sm.dO[j] = rho * sm.gdy[j] - rho * rho * rho / kBD * oo * sm.scal[1];
                const size_t gj = (((size_t)bb * T_ + t) * H + h) * kBD + j;
                p.grad_g[gj] = cur.x2 * oo * rho;
            }
            __syncthreads();
            // (3) dS += q~^T do; dq~ = S_t do^T (rows); k dS and (b*k) dS (columns)
            {
                const float4 d4 = ld4(&sm.dO[4 * lane]);
                float rowv[kBRows];
                float4 cA = make_float4(0.f, 0.f, 0.f, 0.f), cB = cA;
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = warp + 8 * m;
                    const float4 st = ld4(St + own + (size_t)8 * m * kBD);
                    rowv[m] = dot4(st, d4);
                    float4 ds = sdS[i * 32 + lane];
                    const float a = sm.qt[i];
                    ds.x = fmaf(a, d4.x, ds.x); ds.y = fmaf(a, d4.y, ds.y);
                    ds.z = fmaf(a, d4.z, ds.z); ds.w = fmaf(a, d4.w, ds.w);
                    sdS[i * 32 + lane] = ds;
                    const float kk = sm.k[i], kh = sm.kh[i];
                    cA.x = fmaf(kk, ds.x, cA.x); cA.y = fmaf(kk, ds.y, cA.y);
                    cA.z = fmaf(kk, ds.z, cA.z); cA.w = fmaf(kk, ds.w, cA.w);
                    cB.x = fmaf(kh, ds.x, cB.x); cB.y = fmaf(kh, ds.y, cB.y);
                    cB.z = fmaf(kh, ds.z, cB.z); cB.w = fmaf(kh, ds.w, cB.w);
                }
                const float rs = rows_reduce_scatter(rowv, lane);
                if ((lane & 1) == 0) sm.rows[0][warp + 8 * ((lane >> 1) & 15)] = rs;
                *reinterpret_cast<float4 *>(&sm.redA[warp][4 * lane]) = cA;
                *reinterpret_cast<float4 *>(&sm.redB[warp][4 * lane]) = cB;
            }
            __syncthreads();
            // (4) dv^ and dr; dv, dw
            if (tid >= kBD) {
                const int j = tid - kBD;
                float sa = 0.f, sb = 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    sa += sm.redA[u][j];
                    sb += sm.redB[u][j];
                }
                sm.dr[j] = -sb;
                const size_t gj = (((size_t)bb * T_ + t) * H + h) * kBD + j;
                p.grad_v[gj] = cur.x0 * sa;
                p.grad_w[gj] = cur.x1 * sa;
            }
            __syncthreads();
            // (5) row sums dS v^T, -dS r^T, S_{t-1} dr^T, (dS + k^T dr) * S_{t-1}; dS <- Diag(alpha) dS_hat
            {
                const float4 vv = ld4(&sm.vh[4 * lane]), rr = ld4(&sm.r[4 * lane]), dd = ld4(&sm.dr[4 * lane]);
                float ra[kBRows], rb[kBRows], rc[kBRows], rd[kBRows];
#pragma unroll
                for (int m = 0; m < kBRows; ++m) {
                    const int i = warp + 8 * m;
                    const float4 sp = ld4(Sp + own + (size_t)8 * m * kBD);
                    float4 ds = sdS[i * 32 + lane];
                    ra[m] = dot4(ds, vv);
                    rb[m] = -dot4(ds, rr);
                    rc[m] = dot4(sp, dd);
                    const float kk = sm.k[i], al = sm.al[i];
                    ds.x = fmaf(kk, dd.x, ds.x); ds.y = fmaf(kk, dd.y, ds.y);
                    ds.z = fmaf(kk, dd.z, ds.z); ds.w = fmaf(kk, dd.w, ds.w);
                    rd[m] = dot4(ds, sp);
                    ds.x *= al; ds.y *= al; ds.z *= al; ds.w *= al;
                    sdS[i * 32 + lane] = ds;
                }
                const int ri = warp + 8 * ((lane >> 1) & 15);
                const float sa = rows_reduce_scatter(ra, lane), sb = rows_reduce_scatter(rb, lane);
                const float sc = rows_reduce_scatter(rc, lane), sd = rows_reduce_scatter(rd, lane);
                if ((lane & 1) == 0) {
                    sm.rows[1][ri] = sa;
                    sm.rows[2][ri] = sb;
                    sm.rows[3][ri] = sc;
                    sm.rows[4][ri] = sd;
                }
            }
            __syncthreads();
            // (6) key-side gradients of token t
            if (tid < kBD) {
                const size_t gi = (((size_t)bb * T_ + t) * H + h) * kBD + tid;
                const float kk = sm.k[tid], al = sm.al[tid];
                const float bv = cur.x2, qv = cur.x3, zv = cur.x4;
                const float gs = gs_own;
                const float ts = two_sigmoid(zv);
                const float dqt = sm.rows[0][tid], dkh = sm.rows[2][tid];
                p.grad_k[gi] = sm.rows[1][tid] + al * sm.rows[3][tid] + bv * dkh;
                p.grad_b[gi] = kk * dkh;
                p.grad_la[gi] = al * sm.rows[4][tid];
                p.grad_q[gi] = dqt * gs * ts;
                p.grad_z[gi] = dqt * qv * gs * ts * (1.f - 0.5f * ts);
                dgam = fmaf(dqt * qv, ts, dgam);
            }
        }
    }
    __syncthreads();
    if (p.grad_S_in) {
#pragma unroll
        for (int m = 0; m < kBRows; ++m)
            *reinterpret_cast<float4 *>(p.grad_S_in + (size_t)head * mat + own + (size_t)8 * m * kBD) =
                sdS[(warp + 8 * m) * 32 + lane];
    }
    if (tid < kBD) p.ws_dgam[(size_t)head * kBD + tid] = dgam;
}

// d gamma_stat[h] = sum over the batch rows of the per-head partials
__global__ void __launch_bounds__(kBD) gdn2_bwd_dgamma_kernel(const float *part, float *out, int B, int H) {
    const int h = blockIdx.x, i = threadIdx.x;
    float s = 0.f;
    for (int bb = 0; bb < B; ++bb) s += part[((size_t)bb * H + h) * kBD + i];
    out[(size_t)h * kBD + i] = s;
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int T) {
    const size_t mat = (size_t)kBD * kBD * sizeof(float);
    const size_t NC = (size_t)(T + kBC - 1) / kBC;
    return (size_t)B * H * ((NC + 1) * mat + (kBC + 1) * mat + kBD * sizeof(float));
}

cudaError_t launch_bwd(BwdParams p, void *workspace, int dtype, cudaStream_t stream) {
    const size_t mat = (size_t)kBD * kBD;
    const size_t BH = (size_t)p.B * p.H;
    const size_t NC = (size_t)(p.T + kBC - 1) / kBC;
    float *ws = (float *)workspace;
    p.ws_ckpt = ws;
    p.ws_chunk = ws + BH * (NC + 1) * mat;
    p.ws_dgam = p.ws_chunk + BH * (kBC + 1) * mat;
    const size_t dsm = (size_t)kBD * kBD * sizeof(float);      // running dS
    cudaError_t e;
    if (dtype == GDELTA_BF16) {
        e = cudaFuncSetAttribute(gdn2_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm);
        if (e != cudaSuccess) return e;
        gdn2_bwd_kernel<__nv_bfloat16><<<(unsigned)BH, kBT, dsm, stream>>>(p);
    } else {
        e = cudaFuncSetAttribute(gdn2_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm);
        if (e != cudaSuccess) return e;
        gdn2_bwd_kernel<float><<<(unsigned)BH, kBT, dsm, stream>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess || !p.grad_gs) return e;
    gdn2_bwd_dgamma_kernel<<<(unsigned)p.H, kBD, 0, stream>>>(p.ws_dgam, p.grad_gs, p.B, p.H);
    return cudaGetLastError();
}

}  // namespace gdelta
