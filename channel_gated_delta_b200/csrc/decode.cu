// Single-token decode step: one CTA per (batch, head), S streamed once in and
// once out with 128-bit coalesced accesses.  Half of a thread's rows of S are
// held in registers, the other half in shared memory (loaded with cp.async),
// so that four CTAs fit on an SM: with 1024 heads that is 1.7 waves of CTAs
// instead of 3.5, and twice the bytes in flight per SM.
//
// Per head, with S_hat = Diag(alpha) S (Muir review §2.1), for every value
// column j one read pass yields
//   r_j = sum_i k_i alpha_i S_ij        (k S_hat, the erase projection)
//   a_j = sum_i q~_i alpha_i S_ij       (q~ S_hat)
// and then, with c_b = q~ . (b*k) and c_k = q~ . k,
//   o_j   = a_j - r_j c_b + (w*v)_j c_k                  (= q~ S_t)
//   S'_ij = alpha_i S_ij - (b*k)_i r_j + k_i (w*v)_j     (the GDN-2 update)
// so S is read once and written once; o is RMS-normalised over d_v and gated.
#include "common.cuh"

namespace gdelta {

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}

// kRaw: q and k need SiLU and l2 normalisation (compiled apart, so the plain
// build keeps its register allocation).
template <typename T, int DK, int DV, bool kRaw>
__global__ void __launch_bounds__(256, 4) gdn2_decode_kernel(DecodeParams p) {
    constexpr int NT = 256;
    constexpr int CPR = DV / 4;       // threads across one row (4 columns each)
    constexpr int RG = NT / CPR;      // row groups
    constexpr int RPT = DK / RG;      // rows per thread
    constexpr int RREG = RPT / 2;     // of them in registers; the rest in shared memory
    static_assert(DK % RG == 0 && RPT % 2 == 0, "row split");

    __shared__ float s_k[DK], s_kh[DK], s_ka[DK], s_qa[DK], s_alpha[DK];
    __shared__ float s_vh[DV];
    __shared__ float s_red_r[RG][DV], s_red_a[RG][DV];
    __shared__ float s_r[DV], s_o[DV];
    __shared__ float s_part[3][NT / 32];
    __shared__ float4 s_S[RPT - RREG][NT];       // this thread's shared-memory rows, [m - RREG][tid]

    const int tid = threadIdx.x;
    const int cg = tid % CPR;
    const int rg = tid / CPR;
    const int head = blockIdx.x;                  // b * H + h
    const int h = head % p.H;
    const size_t kbase = (size_t)head * DK;
    const size_t vbase = (size_t)head * DV;
    float *S = p.S + (size_t)head * DK * DV;

    // Issue the state loads first: they are the bulk of the traffic.
#pragma unroll
    for (int m = RREG; m < RPT; ++m) {
        const int i = rg + RG * m;
        cp_async16(&s_S[m - RREG][tid], S + (size_t)i * DV + 4 * cg);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    float4 Sr[RREG];
#pragma unroll
    for (int m = 0; m < RREG; ++m) {
        const int i = rg + RG * m;
        Sr[m] = *reinterpret_cast<const float4 *>(S + (size_t)i * DV + 4 * cg);
    }

    const T *q = (const T *)p.q, *k = (const T *)p.k, *z = (const T *)p.z, *b = (const T *)p.b;
    const T *v = (const T *)p.v, *w = (const T *)p.w, *beta = (const T *)p.beta;
    // raw q, k: SiLU, then 1 / ||.|| over the head's d_k channels
    float inv_k = 1.f, inv_q = 1.f;
    if (kRaw) {
        float ssk = 0.f, ssq = 0.f;
        for (int i = tid; i < DK; i += NT) {
            const float a = silu(ldf(k, kbase + i)), c = silu(ldf(q, kbase + i));
            ssk = fmaf(a, a, ssk);
            ssq = fmaf(c, c, ssq);
        }
        ssk = warp_sum(ssk);
        ssq = warp_sum(ssq);
        if ((tid & 31) == 0) {
            s_part[0][tid >> 5] = ssk;
            s_part[1][tid >> 5] = ssq;
        }
        __syncthreads();
        ssk = 0.f;
        ssq = 0.f;
#pragma unroll
        for (int u = 0; u < NT / 32; ++u) {
            ssk += s_part[0][u];
            ssq += s_part[1][u];
        }
        inv_k = rsqrtf(fmaxf(ssk, 1e-24f));
        inv_q = rsqrtf(fmaxf(ssq, 1e-24f));
        __syncthreads();                              // s_part is reused below
    }
    float cb = 0.f, ck = 0.f;
    for (int i = tid; i < DK; i += NT) {
        const float ki = kRaw ? as_dtype(silu(ldf(k, kbase + i)) * inv_k, k) : ldf(k, kbase + i);
        const float bi = beta ? ldf(beta, head) : ldf(b, kbase + i);
        const float al = expf(p.decay_tok ? p.la[head] : p.la[kbase + i]);
        const float gs = p.gs ? p.gs[(size_t)h * DK + i] : 1.f;
        const float qi = kRaw ? as_dtype(silu(ldf(q, kbase + i)) * inv_q, q) : ldf(q, kbase + i);
        const float qt = qi * gs * two_sigmoid(z ? ldf(z, kbase + i) : 0.f);
        s_k[i] = ki;
        s_kh[i] = bi * ki;
        s_alpha[i] = al;
        s_ka[i] = ki * al;
        s_qa[i] = qt * al;
        cb += qt * bi * ki;
        ck += qt * ki;
    }
    for (int j = tid; j < DV; j += NT) s_vh[j] = (beta ? ldf(beta, head) : ldf(w, vbase + j)) * ldf(v, vbase + j);
    cb = warp_sum(cb);
    ck = warp_sum(ck);
    if ((tid & 31) == 0) {
        s_part[0][tid >> 5] = cb;
        s_part[1][tid >> 5] = ck;
    }
    __syncthreads();
    cb = 0.f;
    ck = 0.f;
#pragma unroll
    for (int u = 0; u < NT / 32; ++u) {
        cb += s_part[0][u];
        ck += s_part[1][u];
    }

    // Partial column sums over this thread's rows (its own cp.async copies are
    // complete after the wait; no other thread reads them).
    asm volatile("cp.async.wait_all;" ::: "memory");
    float4 pr = make_float4(0.f, 0.f, 0.f, 0.f), pa = pr;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg + RG * m;
        const float ka = s_ka[i], qa = s_qa[i];
        const float4 x = m < RREG ? Sr[m] : s_S[m - RREG][tid];
        pr.x += ka * x.x; pr.y += ka * x.y; pr.z += ka * x.z; pr.w += ka * x.w;
        pa.x += qa * x.x; pa.y += qa * x.y; pa.z += qa * x.z; pa.w += qa * x.w;
    }
    *reinterpret_cast<float4 *>(&s_red_r[rg][4 * cg]) = pr;
    *reinterpret_cast<float4 *>(&s_red_a[rg][4 * cg]) = pa;
    __syncthreads();

    float osq = 0.f;
    for (int j = tid; j < DV; j += NT) {
        float r = 0.f, a = 0.f;
#pragma unroll
        for (int u = 0; u < RG; ++u) {
            r += s_red_r[u][j];
            a += s_red_a[u][j];
        }
        const float o = a - r * cb + s_vh[j] * ck;
        s_r[j] = r;
        s_o[j] = o;
        osq += o * o;
    }
    osq = warp_sum(osq);
    if ((tid & 31) == 0) s_part[2][tid >> 5] = osq;
    __syncthreads();
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < NT / 32; ++u) ss += s_part[2][u];
    const float inv = rsqrtf(ss / DV + p.eps);

    const T *g = (const T *)p.g;
    for (int j = tid; j < DV; j += NT) {
        const float o = s_o[j];
        stf((T *)p.y, vbase + j, ldf(g, vbase + j) * o * inv);
        if (p.o_raw) p.o_raw[vbase + j] = o;
    }

    // S' = alpha S - (b*k)^T r + k^T (w*v)
    const float4 r4 = *reinterpret_cast<const float4 *>(&s_r[4 * cg]);
    const float4 v4 = *reinterpret_cast<const float4 *>(&s_vh[4 * cg]);
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg + RG * m;
        const float al = s_alpha[i], kh = s_kh[i], ki = s_k[i];
        const float4 x = m < RREG ? Sr[m] : s_S[m - RREG][tid];
        float4 o;
        o.x = al * x.x - kh * r4.x + ki * v4.x;
        o.y = al * x.y - kh * r4.y + ki * v4.y;
        o.z = al * x.z - kh * r4.z + ki * v4.z;
        o.w = al * x.w - kh * r4.w + ki * v4.w;
        *reinterpret_cast<float4 *>(S + (size_t)i * DV + 4 * cg) = o;
    }
}

template <typename T, bool kRaw>
static cudaError_t launch_tr(const DecodeParams &p, cudaStream_t s) {
    const dim3 grid(p.B * p.H), block(256);
    if (p.dk == 128 && p.dv == 128) gdn2_decode_kernel<T, 128, 128, kRaw><<<grid, block, 0, s>>>(p);
    else if (p.dk == 128 && p.dv == 64) gdn2_decode_kernel<T, 128, 64, kRaw><<<grid, block, 0, s>>>(p);
    else if (p.dk == 64 && p.dv == 128) gdn2_decode_kernel<T, 64, 128, kRaw><<<grid, block, 0, s>>>(p);
    else if (p.dk == 64 && p.dv == 64) gdn2_decode_kernel<T, 64, 64, kRaw><<<grid, block, 0, s>>>(p);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_t(const DecodeParams &p, cudaStream_t s) {
    return p.qk_raw ? launch_tr<T, true>(p, s) : launch_tr<T, false>(p, s);
}

cudaError_t launch_decode(const DecodeParams &p, int dtype, cudaStream_t stream) {
    return dtype == GDELTA_BF16 ? launch_t<__nv_bfloat16>(p, stream) : launch_t<float>(p, stream);
}

}  // namespace gdelta
