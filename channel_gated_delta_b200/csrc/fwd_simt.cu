// fp32 CUDA-core chunked forward: one CTA per (batch, head), chunks in order,
// the state S held in shared memory across chunks.
//
// This is the exact-fp32 path (all arithmetic in fp32, decays taken pairwise
// from non-positive log-decay differences, so nothing is divided by a
// cumulative decay).  Within a chunk of C tokens starting from state S
// (row-vector convention; Lambda_t = cumulative log-decay inside the chunk):
//
//   M_ts  = sum_i k_ti e^{Lambda_ti - Lambda_si} k_si        t > s
//   L_ts  = sum_i k_ti e^{Lambda_ti - Lambda_si} (b*k)_si    t > s
//   Aq_ts = sum_i q~_ti e^{Lambda_ti - Lambda_si} k_si       t >= s
//   Bq_ts = sum_i q~_ti e^{Lambda_ti - Lambda_si} (b*k)_si   t >= s
//   (I + L) R = (K * e^Lambda) S + M V^        (forward substitution)
//   O   = (Q~ * e^Lambda) S + Aq V^ - Bq R
//   S  <- e^{Lambda_C} * S + (K * pi)^T V^ - ((b*k) * pi)^T R,  pi_t = e^{Lambda_C - Lambda_t}
//
// with V^ = w*v and q~ = q * gamma_stat * 2 sigmoid(z).  R holds the erase
// projections r_t = k_t Diag(alpha_t) S_{t-1} of the token recurrence (Muir
// review §2.1 update; the chunked structure follows §2.4 and the chunked
// DeltaNet of "Kimi3 = GPT2 x 22580" §4).  A ragged last chunk is padded with
// identity tokens (k = 0, log_alpha = 0, v^ = 0), which leave S unchanged.
#include "common.cuh"

namespace gdelta {

namespace {

struct SimtLayout {
    int dkp, cp;   // padded strides
    size_t k, kh, qt, lam, tmp, vh, x, o, M, L, Aq, Bq, S, total;  // float offsets
};

__host__ __device__ inline SimtLayout simt_layout(int dk, int dv, int C) {
    SimtLayout l;
    l.dkp = dk + 1;
    l.cp = C + 1;
    size_t off = 0;
    const size_t ck = (size_t)C * l.dkp, cv = (size_t)C * dv, cc = (size_t)C * l.cp;
    l.k = off; off += ck;
    l.kh = off; off += ck;
    l.qt = off; off += ck;
    l.lam = off; off += ck;
    l.tmp = off; off += ck;
    l.vh = off; off += cv;
    l.x = off; off += cv;
    l.o = off; off += cv;
    l.M = off; off += cc;
    l.L = off; off += cc;
    l.Aq = off; off += cc;
    l.Bq = off; off += cc;
    off = (off + 3) & ~(size_t)3;          // 16-byte align the state
    l.S = off; off += (size_t)dk * dv;
    l.total = off;
    return l;
}

}  // namespace

size_t fwd_simt_smem_bytes(int dk, int dv, int C) { return simt_layout(dk, dv, C).total * sizeof(float); }

int fwd_simt_chunk(int dk, int dv, int requested) {
    int C = requested;
    while (C > 16 && fwd_simt_smem_bytes(dk, dv, C) > 227 * 1024) C /= 2;
    return fwd_simt_smem_bytes(dk, dv, C) <= 227 * 1024 ? C : 0;
}

template <typename T>
__global__ void __launch_bounds__(256) gdn2_fwd_simt_kernel(FwdParams p) {
    extern __shared__ __align__(16) float sm[];
    const int NT = blockDim.x;
    const int tid = threadIdx.x;
    const int dk = p.dk, dv = p.dv, C = p.C, H = p.H, T_ = p.T;
    const SimtLayout l = simt_layout(dk, dv, C);
    const int dkp = l.dkp, cp = l.cp;
    float *sk = sm + l.k, *skh = sm + l.kh, *sqt = sm + l.qt, *slam = sm + l.lam, *stmp = sm + l.tmp;
    float *svh = sm + l.vh, *sx = sm + l.x, *so = sm + l.o;
    float *sM = sm + l.M, *sL = sm + l.L, *sAq = sm + l.Aq, *sBq = sm + l.Bq, *sS = sm + l.S;

    const int head = blockIdx.x;
    const int bb = head / H, h = head % H;
    const T *q = (const T *)p.q, *k = (const T *)p.k, *z = (const T *)p.z, *b = (const T *)p.b;
    const T *v = (const T *)p.v, *w = (const T *)p.w, *g = (const T *)p.g, *beta = (const T *)p.beta;

    // S_0
    const size_t sbase = (size_t)head * dk * dv;
    for (int e = tid; e < dk * dv; e += NT) sS[e] = p.S_in ? p.S_in[sbase + e] : 0.f;

    for (int t0 = 0; t0 < T_; t0 += C) {
        const int n = min(C, T_ - t0);
        __syncthreads();
        // (a) load the chunk; identity padding past the end of the sequence
        for (int e = tid; e < C * dk; e += NT) {
            const int t = e / dk, i = e % dk;
            float kv = 0.f, bv = 0.f, qv = 0.f, lv = 0.f, gate = 0.f;
            if (t < n) {
                const size_t gt = ((size_t)bb * T_ + t0 + t) * H + h;   // token and head
                const size_t gi = gt * dk + i;
                kv = ldf(k, gi);
                bv = beta ? ldf(beta, gt) : ldf(b, gi);
                const float gs = p.gs ? p.gs[(size_t)h * dk + i] : 1.f;
                gate = gs * two_sigmoid(z ? ldf(z, gi) : 0.f);
                qv = ldf(q, gi);
                if (p.qk_raw) {
                    kv = silu(kv);
                    qv = silu(qv);
                } else {
                    qv *= gate;
                }
                lv = p.decay_tok ? p.la[gt] : p.la[gi];
            }
            sk[t * dkp + i] = kv;
            skh[t * dkp + i] = p.qk_raw ? bv : bv * kv;   // raw: finished after the norms below
            sqt[t * dkp + i] = qv;
            slam[t * dkp + i] = lv;
            if (p.qk_raw) stmp[t * dkp + i] = gate;        // stmp is free until (b)
        }
        for (int e = tid; e < C * dv; e += NT) {
            const int t = e / dv, j = e % dv;
            float x = 0.f;
            if (t < n) {
                const size_t gt = ((size_t)bb * T_ + t0 + t) * H + h;
                const size_t gi = gt * dv + j;
                x = (beta ? ldf(beta, gt) : ldf(w, gi)) * ldf(v, gi);
            }
            svh[t * dv + j] = x;
        }
        if (p.qk_raw) {
            // per-token l2 norms of SiLU(k) and SiLU(q) over the head's d_k channels;
            // the normalised values are held in the token dtype, then gated
            __syncthreads();
            float *sinv = sM;                                 // [2][C]; sM is written only in (c)
            for (int r = tid; r < 2 * C; r += NT) {
                const float *row = r < C ? sk + r * dkp : sqt + (r - C) * dkp;
                float ss = 0.f;
                for (int i = 0; i < dk; ++i) ss = fmaf(row[i], row[i], ss);
                sinv[r] = rsqrtf(fmaxf(ss, 1e-24f));
            }
            __syncthreads();
            for (int e = tid; e < C * dk; e += NT) {
                const int t = e / dk, i = e % dk;
                const float kn = as_dtype(sk[t * dkp + i] * sinv[t], k);
                sk[t * dkp + i] = kn;
                skh[t * dkp + i] *= kn;
                sqt[t * dkp + i] = as_dtype(sqt[t * dkp + i] * sinv[C + t], q) * stmp[t * dkp + i];
            }
        }
        __syncthreads();
        // (b) cumulative log-decay and gamma_t = e^{Lambda_t} (<= 1)
        for (int i = tid; i < dk; i += NT) {
            float acc = 0.f;
            for (int t = 0; t < C; ++t) {
                acc += slam[t * dkp + i];
                slam[t * dkp + i] = acc;
                stmp[t * dkp + i] = expf(acc);
            }
        }
        __syncthreads();
        // (c) decay-relative products, pairwise non-positive exponents
        for (int e = tid; e < C * C; e += NT) {
            const int t = e / C, s = e % C;
            float m = 0.f, lm = 0.f, aq = 0.f, bq = 0.f;
            if (s <= t) {
                const float *kt = sk + t * dkp, *qt = sqt + t * dkp, *lt = slam + t * dkp;
                const float *ks = sk + s * dkp, *khs = skh + s * dkp, *ls = slam + s * dkp;
                for (int i = 0; i < dk; ++i) {
                    const float d = expf(lt[i] - ls[i]);
                    const float kd = kt[i] * d, qd = qt[i] * d;
                    m += kd * ks[i];
                    lm += kd * khs[i];
                    aq += qd * ks[i];
                    bq += qd * khs[i];
                }
                if (s == t) { m = 0.f; lm = 0.f; }
            }
            sM[t * cp + s] = m;
            sL[t * cp + s] = lm;
            sAq[t * cp + s] = aq;
            sBq[t * cp + s] = bq;
        }
        __syncthreads();
        // (d) right-hand side X = (K * gamma) S + M V^
        for (int e = tid; e < C * dv; e += NT) {
            const int t = e / dv, j = e % dv;
            float x = 0.f;
            const float *kt = sk + t * dkp, *gt = stmp + t * dkp;
            for (int i = 0; i < dk; ++i) x += kt[i] * gt[i] * sS[i * dv + j];
            for (int s = 0; s < t; ++s) x += sM[t * cp + s] * svh[s * dv + j];
            sx[t * dv + j] = x;
        }
        // (e) forward substitution (I + L) R = X, row by row
        for (int t = 1; t < C; ++t) {
            __syncthreads();
            for (int j = tid; j < dv; j += NT) {
                float x = sx[t * dv + j];
                for (int s = 0; s < t; ++s) x -= sL[t * cp + s] * sx[s * dv + j];
                sx[t * dv + j] = x;
            }
        }
        __syncthreads();
        // (f) O = (Q~ * gamma) S + Aq V^ - Bq R
        for (int e = tid; e < C * dv; e += NT) {
            const int t = e / dv, j = e % dv;
            float o = 0.f;
            const float *qt = sqt + t * dkp, *gt = stmp + t * dkp;
            for (int i = 0; i < dk; ++i) o += qt[i] * gt[i] * sS[i * dv + j];
            for (int s = 0; s <= t; ++s) o += sAq[t * cp + s] * svh[s * dv + j] - sBq[t * cp + s] * sx[s * dv + j];
            so[t * dv + j] = o;
        }
        __syncthreads();
        // (g) per-head RMSNorm over d_v and the output gate; one warp per token
        {
            const int warp = tid >> 5, lane = tid & 31, nw = NT >> 5;
            for (int t = warp; t < n; t += nw) {
                float ss = 0.f;
                for (int j = lane; j < dv; j += 32) ss += so[t * dv + j] * so[t * dv + j];
                ss = warp_sum(ss);
                const float inv = rsqrtf(ss / dv + p.eps);
                const size_t gi = (((size_t)bb * T_ + t0 + t) * H + h) * dv;
                for (int j = lane; j < dv; j += 32) {
                    const float o = so[t * dv + j];
                    stf((T *)p.y, gi + j, ldf(g, gi + j) * o * inv);
                    if (p.o_raw) p.o_raw[gi + j] = o;
                }
            }
        }
        // (h) pi_t = e^{Lambda_C - Lambda_t} (<= 1) replaces gamma in stmp
        for (int e = tid; e < C * dk; e += NT) {
            const int t = e / dk, i = e % dk;
            stmp[t * dkp + i] = expf(slam[(C - 1) * dkp + i] - slam[t * dkp + i]);
        }
        __syncthreads();
        // (i) S <- e^{Lambda_C} S + (K * pi)^T V^ - ((b*k) * pi)^T R
        for (int e = tid; e < dk * dv; e += NT) {
            const int i = e / dv, j = e % dv;
            float s = expf(slam[(C - 1) * dkp + i]) * sS[e];
            for (int t = 0; t < C; ++t) {
                const float pt = stmp[t * dkp + i];
                s += pt * (sk[t * dkp + i] * svh[t * dv + j] - skh[t * dkp + i] * sx[t * dv + j]);
            }
            sS[e] = s;
        }
    }
    __syncthreads();
    if (p.S_out)
        for (int e = tid; e < dk * dv; e += NT) p.S_out[sbase + e] = sS[e];
}

template <typename T>
static cudaError_t launch_t(const FwdParams &p, cudaStream_t s) {
    const size_t smem = fwd_simt_smem_bytes(p.dk, p.dv, p.C);
    cudaError_t e = cudaFuncSetAttribute(gdn2_fwd_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gdn2_fwd_simt_kernel<T><<<p.B * p.H, 256, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_fwd_simt(const FwdParams &p, int dtype, cudaStream_t stream) {
    return dtype == GDELTA_BF16 ? launch_t<__nv_bfloat16>(p, stream) : launch_t<float>(p, stream);
}

}  // namespace gdelta
