// Shared device helpers for the gated delta-rule kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdelta.h"

namespace gdelta {

// Element loads/stores for the two token dtypes.
__device__ __forceinline__ float ldf(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void stf(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// 2 * sigmoid(z): the dynamic readout modulation in (0, 2) (Muir review §2.1).
__device__ __forceinline__ float two_sigmoid(float z) { return 2.0f / (1.0f + expf(-z)); }

// SiLU, x sigmoid(x): the key and query activation before their per-head
// l2 normalisation (Muir review §2.1).
__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

// A value as the token dtype holds it (bf16 rounding; fp32 unchanged).
__device__ __forceinline__ float as_dtype(float x, const float *) { return x; }
__device__ __forceinline__ float as_dtype(float x, const __nv_bfloat16 *) {
    return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Device status codes written by kernels that detect a run-time fault.
enum DeviceStatus : int { kDevOk = 0, kDevTimeout = 1, kDevRange = 2 };

// Gate and decay forms (gdelta.h): z may be null (read as 0); beta, when
// non-null, replaces b and w (one value per token and head); decay_tok = 1
// means log_alpha holds one value per token and head; qk_raw = 1 means q and
// k still need SiLU and per-head l2 normalisation.
struct FwdParams {
    int B, T, H, dk, dv, C;
    const void *q, *k, *z, *b, *v, *w, *g;
    const float *la, *gs, *S_in;
    float *S_out;
    void *y;
    float *o_raw;
    float eps;
    const void *beta;
    int decay_tok;
    int qk_raw;
    int *status;
    unsigned wait_limit;     // polls before a bounded wait gives up
    int stall;               // 1: the kernels first wait on a barrier nothing completes (failure-path tests)
};

struct DecodeParams {
    int B, H, dk, dv;
    const void *q, *k, *z, *b, *v, *w, *g;
    const float *la, *gs;
    float *S;
    void *y;
    float *o_raw;
    float eps;
    const void *beta;
    int decay_tok;
    int qk_raw;
};

// Backward pass (d_k = d_v = 128): forward inputs, the incoming gradients,
// the gradient outputs (fp32) and the workspace partition.
struct BwdParams {
    int B, T, H;
    const void *q, *k, *z, *b, *v, *w, *g;
    const float *la, *gs, *S_in;
    const float *dy, *dS_out;
    float eps;
    float *grad_q, *grad_k, *grad_v, *grad_b, *grad_w, *grad_z, *grad_g, *grad_la, *grad_gs, *grad_S_in;
    float *ws_ckpt, *ws_chunk, *ws_dgam, *ws_part, *ws_or;
    int *status;             // device status word (a bounded wait that ran out)
    uint32_t wait_limit;     // polls before such a wait gives up
    int stall;               // 1: wait first on a barrier nothing completes, so that the wait runs out
};

// Five-gate low-rank projection (gdelta.h, gdelta_gate_proj).
struct GateProjParams {
    int N, d;
    int ranks[5];
    const void *x, *w_down, *w_up;
    const float *bias;
    void *codes;             // workspace: [N, 2R] bf16, the codes as two parts (hi | lo)
    float *log_alpha;
    void *b, *g, *w, *z;
    int *status;
    unsigned wait_limit;
    int stall;
};

// Launchers (return cudaError_t of the launch).
cudaError_t launch_decode(const DecodeParams &p, int dtype, cudaStream_t stream);
cudaError_t launch_fwd_simt(const FwdParams &p, int dtype, cudaStream_t stream);
size_t fwd_simt_smem_bytes(int dk, int dv, int C);
int fwd_simt_chunk(int dk, int dv, int requested);
cudaError_t launch_state_init(float *S, const float *src, size_t n, cudaStream_t stream);
size_t bwd_workspace_bytes(int B, int H, int T);
cudaError_t launch_bwd(BwdParams p, void *workspace, int dtype, cudaStream_t stream);
cudaError_t launch_state_affine(float *S_out, const float *A, const float *S_in, const float *D, int BH, int dk,
                                int dv, cudaStream_t stream);
cudaError_t launch_fwd_tc(const FwdParams &p, void *workspace, cudaStream_t stream);
size_t fwd_tc_workspace_bytes(int B, int H, int T);
bool fwd_tc_supported(int dtype, int dk, int dv, int chunk);
size_t gate_proj_workspace_bytes(int N, int R);
cudaError_t launch_gate_proj(const GateProjParams &p, cudaStream_t stream);

}  // namespace gdelta
