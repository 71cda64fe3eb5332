// C ABI entry points: argument checks on the host, then kernel launches on the
// caller's stream.  Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <mutex>

#include "common.cuh"

namespace gdelta {

// Device status word (one per device that loads the library).  Kernels that
// detect a run-time fault (a bounded wait that ran out) write a nonzero code.
__device__ int g_device_status;

static int *status_ptr() {
    static std::mutex mu;
    static int *ptrs[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        ptrs[dev] = (int *)p;
    }
    return ptrs[dev];
}

// Bounded-wait limit of the tensor-core kernels and the failure-path test
// switch (gdelta_set_wait_limit, gdelta_set_wait_timeout_test).
constexpr uint32_t kDefaultWaitPolls = 1u << 20;
static std::atomic<uint32_t> g_wait_polls{kDefaultWaitPolls};
static std::atomic<int> g_stall_test{0};

static bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }
static bool dim_ok(int d) { return d == 64 || d == 128; }

// Shape/dtype/path checks, plus (for a real call) the required pointers.
static gdelta_status check_fwd(const gdelta_fwd_args *a, bool need_tensors = true) {
    if (!a) return GDELTA_ERR_INVALID_ARG;
    if (a->B < 1 || a->H < 1 || a->T < 0) return GDELTA_ERR_INVALID_ARG;
    if (!(a->eps >= 0.f) || !std::isfinite(a->eps)) return GDELTA_ERR_INVALID_ARG;
    if (a->dtype != GDELTA_F32 && a->dtype != GDELTA_BF16) return GDELTA_ERR_UNSUPPORTED;
    if (!dim_ok(a->dk) || !dim_ok(a->dv)) return GDELTA_ERR_UNSUPPORTED;
    const int C = a->chunk == 0 ? 64 : a->chunk;
    if (C != 16 && C != 32 && C != 64) return GDELTA_ERR_UNSUPPORTED;
    if (a->path < GDELTA_PATH_AUTO || a->path > GDELTA_PATH_TC) return GDELTA_ERR_INVALID_ARG;
    if ((a->qk_raw != 0 && a->qk_raw != 1) || (a->decay_per_token != 0 && a->decay_per_token != 1))
        return GDELTA_ERR_INVALID_ARG;
    if (a->beta && (a->b || a->w)) return GDELTA_ERR_INVALID_ARG;     // one gate form, not both
    if (need_tensors && a->T > 0) {
        if (!a->q || !a->k || !a->v || !a->g || !a->log_alpha || !a->y) return GDELTA_ERR_INVALID_ARG;
        if (!a->beta && (!a->b || !a->w)) return GDELTA_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {a->q, a->k, a->z, a->b, a->v, a->w, a->g, a->log_alpha, a->gamma_stat,
                          a->S_in, a->S_out, a->y, a->o_raw, a->workspace, a->beta};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDELTA_ERR_ALIGNMENT;
    return GDELTA_OK;
}

static int select_path(const gdelta_fwd_args *a) {
    const int C = a->chunk == 0 ? 64 : a->chunk;
    const bool tc_ok = fwd_tc_supported(a->dtype, a->dk, a->dv, C);
    if (a->path == GDELTA_PATH_TC) return tc_ok ? GDELTA_PATH_TC : -1;
    if (a->path == GDELTA_PATH_AUTO && tc_ok) return GDELTA_PATH_TC;
    return GDELTA_PATH_SIMT;
}

}  // namespace gdelta

using namespace gdelta;

extern "C" {

int gdelta_abi_version(void) { return GDELTA_ABI_VERSION; }

const char *gdelta_status_string(gdelta_status s) {
    switch (s) {
        case GDELTA_OK: return "ok";
        case GDELTA_ERR_INVALID_ARG: return "invalid argument";
        case GDELTA_ERR_UNSUPPORTED: return "unsupported shape, chunk, dtype or path";
        case GDELTA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case GDELTA_ERR_CUDA: return "CUDA error";
        case GDELTA_ERR_TIMEOUT: return "device-side bounded wait ran out";
        case GDELTA_ERR_WORKSPACE: return "workspace missing or too small";
        case GDELTA_ERR_RANGE: return "a value left the tensor-core path's fp16 operand range";
    }
    return "unknown status";
}

int gdelta_fwd_selected_path(const gdelta_fwd_args *args) {
    if (check_fwd(args, false) != GDELTA_OK) return -1;
    return select_path(args);
}

size_t gdelta_fwd_workspace_bytes(const gdelta_fwd_args *args) {
    if (check_fwd(args, false) != GDELTA_OK) return 0;
    if (select_path(args) == GDELTA_PATH_TC && args->T > 0) return fwd_tc_workspace_bytes(args->B, args->H, args->T);
    return 0;
}

gdelta_status gdelta_state_init(float *S, int32_t B, int32_t H, int32_t dk, int32_t dv,
                                const float *S_src, void *stream) {
    if (!S || B < 1 || H < 1) return GDELTA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return GDELTA_ERR_UNSUPPORTED;
    if (!aligned16(S) || !aligned16(S_src)) return GDELTA_ERR_ALIGNMENT;
    const size_t n = (size_t)B * H * dk * dv;
    if (S_src && S_src != S) {
        const char *a = (const char *)S, *b = (const char *)S_src;
        if (a < b + n * sizeof(float) && b < a + n * sizeof(float)) return GDELTA_ERR_INVALID_ARG;
    }
    return launch_state_init(S, S_src, n, (cudaStream_t)stream) == cudaSuccess ? GDELTA_OK
                                                                               : GDELTA_ERR_CUDA;
}

static bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b) return false;
    const char *x = (const char *)a, *y = (const char *)b;
    return x < y + nb && y < x + na;
}

gdelta_status gdelta_state_affine(float *S_out, const float *A, const float *S_in, const float *D, int32_t B,
                                  int32_t H, int32_t dk, int32_t dv, void *stream) {
    if (!S_out || !A || B < 1 || H < 1) return GDELTA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return GDELTA_ERR_UNSUPPORTED;
    if (!aligned16(S_out) || !aligned16(A) || !aligned16(S_in) || !aligned16(D)) return GDELTA_ERR_ALIGNMENT;
    const size_t ns = (size_t)B * H * dk * dv * sizeof(float), na = (size_t)B * H * dk * dk * sizeof(float);
    if (overlaps(S_out, ns, A, na) || overlaps(S_out, ns, S_in, ns)) return GDELTA_ERR_INVALID_ARG;
    if (D && D != S_out && overlaps(S_out, ns, D, ns)) return GDELTA_ERR_INVALID_ARG;
    return launch_state_affine(S_out, A, S_in, D, B * H, dk, dv, (cudaStream_t)stream) == cudaSuccess
               ? GDELTA_OK
               : GDELTA_ERR_CUDA;
}

static gdelta_status check_bwd(const gdelta_bwd_args *a) {
    if (!a) return GDELTA_ERR_INVALID_ARG;
    if (a->B < 1 || a->H < 1 || a->T < 0) return GDELTA_ERR_INVALID_ARG;
    if (!(a->eps >= 0.f) || !std::isfinite(a->eps)) return GDELTA_ERR_INVALID_ARG;
    if (a->dtype != GDELTA_F32 && a->dtype != GDELTA_BF16) return GDELTA_ERR_UNSUPPORTED;
    if (a->dk != 128 || a->dv != 128) return GDELTA_ERR_UNSUPPORTED;
    if (a->T > 0) {
        const void *req[] = {a->q, a->k, a->z, a->b, a->v, a->w, a->g, a->log_alpha, a->grad_y,
                             a->grad_q, a->grad_k, a->grad_z, a->grad_b, a->grad_log_alpha,
                             a->grad_v, a->grad_w, a->grad_g};
        for (const void *p : req)
            if (!p) return GDELTA_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {a->q, a->k, a->z, a->b, a->v, a->w, a->g, a->log_alpha, a->gamma_stat, a->S_in,
                          a->grad_y, a->grad_S_out, a->grad_q, a->grad_k, a->grad_z, a->grad_b,
                          a->grad_log_alpha, a->grad_v, a->grad_w, a->grad_g, a->grad_gamma_stat,
                          a->grad_S_in, a->workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDELTA_ERR_ALIGNMENT;
    return GDELTA_OK;
}

size_t gdelta_bwd_workspace_bytes(const gdelta_bwd_args *a) {
    if (check_bwd(a) != GDELTA_OK) return 0;
    return bwd_workspace_bytes(a->B, a->H, a->T);
}

gdelta_status gdelta_bwd(const gdelta_bwd_args *a, void *stream) {
    const gdelta_status st = check_bwd(a);
    if (st != GDELTA_OK) return st;
    if (!a->workspace || a->workspace_bytes < bwd_workspace_bytes(a->B, a->H, a->T)) return GDELTA_ERR_WORKSPACE;
    BwdParams p{};
    p.B = a->B; p.T = a->T; p.H = a->H;
    p.q = a->q; p.k = a->k; p.z = a->z; p.b = a->b; p.v = a->v; p.w = a->w; p.g = a->g;
    p.la = a->log_alpha; p.gs = a->gamma_stat; p.S_in = a->S_in;
    p.dy = a->grad_y; p.dS_out = a->grad_S_out; p.eps = a->eps;
    p.grad_q = a->grad_q; p.grad_k = a->grad_k; p.grad_v = a->grad_v; p.grad_b = a->grad_b;
    p.grad_w = a->grad_w; p.grad_z = a->grad_z; p.grad_g = a->grad_g; p.grad_la = a->grad_log_alpha;
    p.grad_gs = a->grad_gamma_stat; p.grad_S_in = a->grad_S_in;
    p.status = status_ptr();
    p.wait_limit = g_wait_polls.load(std::memory_order_relaxed);
    p.stall = g_stall_test.load(std::memory_order_relaxed);
    return launch_bwd(p, a->workspace, a->dtype, (cudaStream_t)stream) == cudaSuccess ? GDELTA_OK
                                                                                    : GDELTA_ERR_CUDA;
}

gdelta_status gdelta_fwd_chunked(const gdelta_fwd_args *a, void *stream) {
    gdelta_status st = check_fwd(a);
    if (st != GDELTA_OK) return st;
    const int path = select_path(a);
    if (path < 0) return GDELTA_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    if (a->T == 0) {
        if (!a->S_out) return GDELTA_OK;
        return launch_state_init(a->S_out, a->S_in, (size_t)a->B * a->H * a->dk * a->dv, s) ==
                       cudaSuccess
                   ? GDELTA_OK
                   : GDELTA_ERR_CUDA;
    }
    FwdParams p;
    p.B = a->B; p.T = a->T; p.H = a->H; p.dk = a->dk; p.dv = a->dv;
    p.q = a->q; p.k = a->k; p.z = a->z; p.b = a->b; p.v = a->v; p.w = a->w; p.g = a->g;
    p.la = a->log_alpha; p.gs = a->gamma_stat; p.S_in = a->S_in; p.S_out = a->S_out;
    p.y = a->y; p.o_raw = a->o_raw; p.eps = a->eps;
    p.beta = a->beta; p.decay_tok = a->decay_per_token; p.qk_raw = a->qk_raw;
    p.status = status_ptr();
    p.wait_limit = g_wait_polls.load(std::memory_order_relaxed);
    p.stall = g_stall_test.load(std::memory_order_relaxed);
    if (path == GDELTA_PATH_TC) {
        p.C = 64;
        const size_t need = fwd_tc_workspace_bytes(a->B, a->H, a->T);
        if (!a->workspace || a->workspace_bytes < need) return GDELTA_ERR_WORKSPACE;
        return launch_fwd_tc(p, a->workspace, s) == cudaSuccess ? GDELTA_OK : GDELTA_ERR_CUDA;
    }
    p.C = fwd_simt_chunk(a->dk, a->dv, a->chunk == 0 ? 64 : a->chunk);
    if (p.C == 0) return GDELTA_ERR_UNSUPPORTED;
    return launch_fwd_simt(p, a->dtype, s) == cudaSuccess ? GDELTA_OK : GDELTA_ERR_CUDA;
}

gdelta_status gdelta_decode_step(const gdelta_decode_args *a, void *stream) {
    if (!a) return GDELTA_ERR_INVALID_ARG;
    if (a->B < 1 || a->H < 1 || a->reserved != 0 || (a->qk_raw != 0 && a->qk_raw != 1))
        return GDELTA_ERR_INVALID_ARG;
    if (a->decay_per_token != 0 && a->decay_per_token != 1) return GDELTA_ERR_INVALID_ARG;
    if (a->beta ? (a->b || a->w) : (!a->b || !a->w)) return GDELTA_ERR_INVALID_ARG;
    if (!(a->eps >= 0.f) || !std::isfinite(a->eps)) return GDELTA_ERR_INVALID_ARG;
    if (a->dtype != GDELTA_F32 && a->dtype != GDELTA_BF16) return GDELTA_ERR_UNSUPPORTED;
    if (!dim_ok(a->dk) || !dim_ok(a->dv)) return GDELTA_ERR_UNSUPPORTED;
    if (!a->q || !a->k || !a->v || !a->g || !a->log_alpha || !a->S || !a->y) return GDELTA_ERR_INVALID_ARG;
    const void *ptrs[] = {a->q, a->k, a->z, a->b, a->v, a->w, a->g, a->log_alpha, a->gamma_stat,
                          a->S, a->y, a->o_raw, a->beta};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDELTA_ERR_ALIGNMENT;
    DecodeParams p;
    p.B = a->B; p.H = a->H; p.dk = a->dk; p.dv = a->dv;
    p.q = a->q; p.k = a->k; p.z = a->z; p.b = a->b; p.v = a->v; p.w = a->w; p.g = a->g;
    p.la = a->log_alpha; p.gs = a->gamma_stat; p.S = a->S; p.y = a->y; p.o_raw = a->o_raw;
    p.eps = a->eps;
    p.beta = a->beta; p.decay_tok = a->decay_per_token; p.qk_raw = a->qk_raw;
    return launch_decode(p, a->dtype, (cudaStream_t)stream) == cudaSuccess ? GDELTA_OK
                                                                           : GDELTA_ERR_CUDA;
}

static gdelta_status check_gate_proj(const gdelta_gate_proj_args *a, int *R) {
    if (!a) return GDELTA_ERR_INVALID_ARG;
    if (a->N < 1 || a->d < 256) return GDELTA_ERR_INVALID_ARG;
    if (a->d % 256 != 0) return GDELTA_ERR_UNSUPPORTED;
    int r = 0;
    for (int i = 0; i < 5; ++i) {
        if (a->ranks[i] < 64 || a->ranks[i] % 64 != 0) return GDELTA_ERR_UNSUPPORTED;
        r += a->ranks[i];
    }
    if (r % 256 != 0 || r > 2048) return GDELTA_ERR_UNSUPPORTED;
    *R = r;
    return GDELTA_OK;
}

size_t gdelta_gate_proj_workspace_bytes(const gdelta_gate_proj_args *a) {
    int R = 0;
    if (check_gate_proj(a, &R) != GDELTA_OK) return 0;
    return gate_proj_workspace_bytes(a->N, R);
}

gdelta_status gdelta_gate_proj(const gdelta_gate_proj_args *a, void *stream) {
    int R = 0;
    const gdelta_status st = check_gate_proj(a, &R);
    if (st != GDELTA_OK) return st;
    const void *req[] = {a->x, a->w_down, a->w_up, a->bias, a->log_alpha, a->b, a->g, a->w, a->z};
    for (const void *p : req)
        if (!p) return GDELTA_ERR_INVALID_ARG;
    const void *ptrs[] = {a->x, a->w_down, a->w_up, a->bias, a->log_alpha, a->b, a->g, a->w, a->z, a->workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDELTA_ERR_ALIGNMENT;
    if (!a->workspace || a->workspace_bytes < gate_proj_workspace_bytes(a->N, R)) return GDELTA_ERR_WORKSPACE;
    GateProjParams p{};
    p.N = a->N;
    p.d = a->d;
    for (int i = 0; i < 5; ++i) p.ranks[i] = a->ranks[i];
    p.x = a->x; p.w_down = a->w_down; p.w_up = a->w_up; p.bias = a->bias;
    p.codes = a->workspace;
    p.log_alpha = a->log_alpha; p.b = a->b; p.g = a->g; p.w = a->w; p.z = a->z;
    p.status = status_ptr();
    p.wait_limit = g_wait_polls.load(std::memory_order_relaxed);
    p.stall = g_stall_test.load(std::memory_order_relaxed);
    const cudaError_t e = launch_gate_proj(p, (cudaStream_t)stream);
    if (e == cudaErrorInvalidValue) return GDELTA_ERR_UNSUPPORTED;     // a tensor map was refused
    return e == cudaSuccess ? GDELTA_OK : GDELTA_ERR_CUDA;
}

gdelta_status gdelta_set_wait_limit(uint32_t polls) {
    g_wait_polls.store(polls == 0 ? kDefaultWaitPolls : polls, std::memory_order_relaxed);
    return GDELTA_OK;
}

gdelta_status gdelta_set_wait_timeout_test(int32_t on) {
    if (on != 0 && on != 1) return GDELTA_ERR_INVALID_ARG;
    g_stall_test.store(on, std::memory_order_relaxed);
    return GDELTA_OK;
}

gdelta_status gdelta_get_last_device_error(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GDELTA_ERR_CUDA;
    int *p = status_ptr();
    if (!p) return GDELTA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GDELTA_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    }
    if (v == kDevOk) return GDELTA_OK;
    return v == kDevRange ? GDELTA_ERR_RANGE : GDELTA_ERR_TIMEOUT;
}

}  // extern "C"
