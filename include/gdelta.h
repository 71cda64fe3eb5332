/*
 * gdelta.h -- C ABI of the channel-wise gated delta-rule token mixer on
 * NVIDIA B200 (sm_100a).
 *
 * The mixer (GDN-2 state update with the Muir readout).  Per head it keeps a
 * fixed d_k x d_v fp32 state S.  For every token t (row-vector convention,
 * k_t, q_t in R^{1 x d_k}, v_t in R^{1 x d_v}):
 *
 *   S_hat = Diag(alpha_t) S_{t-1},            alpha_t = exp(log_alpha_t)
 *   S_t   = S_hat - (b_t*k_t)^T (k_t S_hat) + k_t^T (w_t*v_t)
 *   o_t   = (q_t * gamma_stat * 2 sigmoid(z_t)) S_t
 *   y_t   = g_t * o_t / sqrt(mean_j o_tj^2 + eps)
 *
 * Sources: "Muir: Linear Attention with Sensitivity-Allocated Gating and
 * Matched-Filter Readout" (arXiv:2611.08376), review page §2.1 (per-channel
 * decay alpha in (0,1)^{d_k}, erase gate b in (0,2)^{d_k} on the key, write
 * gate w in (0,1)^{d_v} on the value, query-only readout gain, per-head RMSNorm
 * followed by the output gate) and §2.4 (chunked kernel); "Kimi3 = GPT2 x
 * 22580" §3-§4 (the state is the cache; read after write; chunked prefill).
 * The page elides the update's display equation; the form above is the one
 * whose special cases are KDA (b = w = beta), Gated DeltaNet (scalar alpha)
 * and DeltaNet (alpha = 1), as the ETH DeltaNet-family study states in its
 * "Gated DeltaNet-2" section.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device,
 *    owned by the caller.  The library allocates no device memory and keeps
 *    no state between calls except cached kernel attributes.
 *  - Token tensors are contiguous [B, T, H, d] (d innermost); decode tensors
 *    are [B, H, d]; states are [B, H, d_k, d_v] fp32 (d_v innermost).
 *  - Every pointer must be 16-byte aligned (GDELTA_ERR_ALIGNMENT otherwise).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  They return after the launches are queued.
 *  - Errors are return codes; nothing aborts or throws across the ABI.
 *    Argument checks run on the host before any launch.  A launch failure is
 *    GDELTA_ERR_CUDA.  Kernels that detect a fault at run time (a bounded wait
 *    that ran out) record it in a device status word that
 *    gdelta_get_last_device_error() reads.
 */
#ifndef GDELTA_H
#define GDELTA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDELTA_ABI_VERSION 4

#if defined(__GNUC__)
#define GDELTA_API __attribute__((visibility("default")))
#else
#define GDELTA_API
#endif

typedef enum gdelta_status {
    GDELTA_OK = 0,
    GDELTA_ERR_INVALID_ARG = 1,   /* null pointer where one is required, bad size */
    GDELTA_ERR_UNSUPPORTED = 2,   /* shape / chunk / dtype outside the supported set */
    GDELTA_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
    GDELTA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    GDELTA_ERR_TIMEOUT = 5,       /* a kernel's bounded wait ran out (device status) */
    GDELTA_ERR_WORKSPACE = 6,     /* workspace missing or smaller than required */
    GDELTA_ERR_RANGE = 7          /* device status: an fp16 tensor-core operand (state, erase
                                     projection or scaled key/query) exceeded 6e4 in magnitude */
} gdelta_status;

typedef enum gdelta_dtype {
    GDELTA_F32 = 0,               /* q,k,v,b,w,z,g and y are fp32 */
    GDELTA_BF16 = 1               /* q,k,v,b,w,z,g and y are bf16 */
} gdelta_dtype;

/* Kernel selection for gdelta_fwd_chunked (args.path). */
typedef enum gdelta_fwd_path {
    GDELTA_PATH_AUTO = 0,         /* tensor-core path where supported, else SIMT */
    GDELTA_PATH_SIMT = 1,         /* fp32 CUDA-core chunked kernel (any supported shape) */
    GDELTA_PATH_TC = 2            /* tcgen05 tensor-core chunked kernel (bf16, d = 128, C = 64) */
} gdelta_fwd_path;

/*
 * Chunked forward (prefill / training forward) over T tokens.
 *
 *   q, k, z, b : [B, T, H, d_k]  dtype        query, key, readout logit, erase gate
 *   v, w, g    : [B, T, H, d_v]  dtype        value, write gate, output gate
 *   log_alpha  : [B, T, H, d_k]  fp32, <= 0   log of the per-channel decay
 *                ([B, T, H] when decay_per_token is 1)
 *   z          : may be NULL: read as 0, so 2 sigmoid(z) = 1 (no dynamic
 *                readout gain, the static profile alone)
 *   beta       : [B, T, H] dtype or NULL.  When given, b and w must be NULL
 *                and b = w = beta on every channel: the KDA parameterisation,
 *                and with decay_per_token = 1 the Gated DeltaNet one (ETH study,
 *                "Gated DeltaNet-2": equal erase and write gates reduce GDN-2
 *                to KDA, a scalar decay further to Gated DeltaNet; "Kimi3 =
 *                GPT2 x 22580" §5, §6).  The kernels then read one value per
 *                token and head instead of two d-long rows.
 *   qk_raw     : 1 = q and k are given before their preprocessing; the kernels
 *                apply it as they load them: SiLU, then l2 normalisation over
 *                the head's d_k channels, x / max(||x||, 1e-12) (Muir review
 *                §2.1: keys and queries pass through SiLU and are l2-normalised
 *                per head; values are not).  The normalised q and k are held
 *                in the token dtype, as a separate normalisation would store
 *                them.  0 = q and k are used as given.
 *   gamma_stat : [H, d_k]        fp32         static readout profile; NULL = ones
 *   S_in       : [B, H, d_k, d_v] fp32        state before token 0; NULL = zeros
 *   S_out      : [B, H, d_k, d_v] fp32        state after token T-1; NULL = not
 *                                             written; may equal S_in (in place)
 *   y          : [B, T, H, d_v]  dtype        gated, normalised readout
 *   o_raw      : [B, T, H, d_v]  fp32         optional pre-norm readout o_t; NULL
 *                                             = not written
 *   chunk      : tokens per chunk; 0 = 64.  Results do not depend on it beyond
 *                rounding.  A ragged last chunk (T % chunk != 0) is handled
 *                inside the kernels.
 *   eps        : RMSNorm epsilon (the workloads use 1e-6).
 *   path       : gdelta_fwd_path.
 *   workspace  : device scratch of gdelta_fwd_workspace_bytes(args) bytes
 *                (may be NULL when that is 0).
 *
 * Supported: d_k, d_v in {64, 128}; chunk in {16, 32, 64}; B, H >= 1; T >= 0
 * (T = 0 only copies S_in to S_out).
 */
typedef struct gdelta_fwd_args {
    int32_t B, T, H, dk, dv;
    int32_t chunk;
    int32_t dtype;        /* gdelta_dtype */
    int32_t path;         /* gdelta_fwd_path */
    const void *q, *k, *z, *b;
    const void *v, *w, *g;
    const float *log_alpha;
    const float *gamma_stat;
    const float *S_in;
    float *S_out;
    void *y;
    float *o_raw;
    float eps;
    void *workspace;
    size_t workspace_bytes;
    const void *beta;           /* see above; NULL = per-channel b and w */
    int32_t decay_per_token;    /* 1: log_alpha is [B, T, H] */
    int32_t qk_raw;             /* 0 or 1, see above */
} gdelta_fwd_args;

/*
 * One decode step for B x H heads (one token each), updating S in place.
 * Same operation as one token of the chunked forward ("Kimi3 = GPT2 x 22580"
 * §1/§3: decoding reads and rewrites the fixed-size cache).
 *
 *   q, k, z, b : [B, H, d_k] dtype;  v, w, g : [B, H, d_v] dtype
 *   log_alpha  : [B, H, d_k] fp32 ([B, H] when decay_per_token is 1)
 *   gamma_stat : [H, d_k] fp32 or NULL
 *   z may be NULL; beta ([B, H] dtype) replaces b and w, and qk_raw applies
 *   the q/k preprocessing, as in gdelta_fwd_args
 *   S          : [B, H, d_k, d_v] fp32, read as S_{t-1}, overwritten with S_t
 *   y          : [B, H, d_v] dtype;  o_raw : [B, H, d_v] fp32 or NULL
 */
typedef struct gdelta_decode_args {
    int32_t B, H, dk, dv;
    int32_t dtype;        /* gdelta_dtype */
    int32_t reserved;     /* must be 0 */
    const void *q, *k, *z, *b;
    const void *v, *w, *g;
    const float *log_alpha;
    const float *gamma_stat;
    float *S;
    void *y;
    float *o_raw;
    float eps;
    const void *beta;           /* NULL = per-channel b and w */
    int32_t decay_per_token;    /* 1: log_alpha is [B, H] */
    int32_t qk_raw;             /* 0 or 1: as in gdelta_fwd_args */
} gdelta_decode_args;

/* ABI version of the loaded library (GDELTA_ABI_VERSION it was built with). */
GDELTA_API int gdelta_abi_version(void);

/* Static, never-NULL description of a status code. */
GDELTA_API const char *gdelta_status_string(gdelta_status status);

/* Bytes of device workspace gdelta_fwd_chunked needs for these arguments
 * (0 when the selected kernel needs none).  Returns 0 for invalid arguments;
 * gdelta_fwd_chunked reports those. */
GDELTA_API size_t gdelta_fwd_workspace_bytes(const gdelta_fwd_args *args);

/* Which kernel gdelta_fwd_chunked would run for these arguments
 * (GDELTA_PATH_SIMT or GDELTA_PATH_TC), or -1 if the arguments are invalid. */
GDELTA_API int gdelta_fwd_selected_path(const gdelta_fwd_args *args);

/*
 * State initialisation ("Kimi3 = GPT2 x 22580" §3: S starts at zero, or at
 * the cache a previous call returned).  S[B,H,d_k,d_v] fp32 <- 0 when S_src is
 * NULL, else <- S_src (same shape; must not overlap S unless equal).
 */
GDELTA_API gdelta_status gdelta_state_init(float *S, int32_t B, int32_t H, int32_t dk, int32_t dv,
                                const float *S_src, void *stream);

/*
 * Affine state map: S_out = A S_in + D for every (batch, head).
 *   A           : [B, H, d_k, d_k] fp32   the map's linear part
 *   S_in, D     : [B, H, d_k, d_v] fp32   either may be NULL (read as 0)
 *   S_out       : [B, H, d_k, d_v] fp32   written; may be D itself, must not
 *                 overlap A or S_in (GDELTA_ERR_INVALID_ARG otherwise)
 * Every token's update is affine in the state with a linear part that acts
 * on the key rows and is the same for every value column, so a whole segment
 * of tokens moves the state by S_end = A S_start + D ("Kimi3 = GPT2 x 22580"
 * §4: a chunk's transition is the product of its tokens' generalised
 * Householder factors plus an accumulated write; §5 and §6 add the decays).
 * A is what gdelta_fwd_chunked returns as S_out from S_in = I with v = 0 (and
 * d_v = d_k); D is its S_out from S_in = 0.  Composing the maps of
 * consecutive segments gives each segment its starting state without running
 * the segments one after another (a long sequence split over devices).
 * Asynchronous on `stream`.
 */
GDELTA_API gdelta_status gdelta_state_affine(float *S_out, const float *A, const float *S_in, const float *D,
                                             int32_t B, int32_t H, int32_t dk, int32_t dv, void *stream);

/*
 * Backward pass: gradients of a loss with respect to every input of
 * gdelta_fwd_chunked, the static readout profile and the initial state, given
 * the loss's gradient with respect to y (and optionally the final state).  The
 * per-channel GDN-2 form with preprocessed q and k (Muir review §2.1), d_k =
 * d_v = 128; the pages describe a chunked custom backward (Muir review §2.4,
 * keeping the block inverse and solutions and recomputing boundary decays);
 * this one recomputes states from checkpoints every 32 tokens instead and
 * runs the exact per-token gradient recurrence on CUDA cores, two CTAs per
 * head (one per half of the value columns).  The key-side gradients
 * (grad_q, grad_k, grad_z, grad_b, grad_log_alpha) are accumulated from the
 * two halves: they are zeroed on `stream` first, then written, and must not
 * alias any input.
 *
 *   B, T, H, dk, dv, dtype, q, k, z, b, v, w, g, log_alpha, gamma_stat,
 *   S_in, eps   : as in gdelta_fwd_args (gamma_stat, S_in may be NULL)
 *   grad_y      : [B, T, H, d_v] fp32, dL/dy
 *   grad_S_out  : [B, H, d_k, d_v] fp32 or NULL (zero), dL/dS_T
 *   grad_q, grad_k, grad_z, grad_b, grad_log_alpha : [B, T, H, d_k] fp32 out
 *   grad_v, grad_w, grad_g                         : [B, T, H, d_v] fp32 out
 *   grad_gamma_stat : [H, d_k] fp32 out (summed over batch and tokens) or NULL
 *   grad_S_in       : [B, H, d_k, d_v] fp32 out or NULL
 *   workspace       : gdelta_bwd_workspace_bytes(args) bytes of device memory
 *                     (checkpoints and one chunk of states per head and value
 *                     half, two RMS partial sums per token, head and
 *                     warp-pair, and per token, head and value half the
 *                     token's o and r on that half's columns);
 *                     GDELTA_ERR_WORKSPACE if smaller
 * Unsupported shapes return GDELTA_ERR_UNSUPPORTED.  Asynchronous on `stream`.
 */
typedef struct gdelta_bwd_args {
    int32_t B, T, H, dk, dv, dtype;
    const void *q, *k, *z, *b, *v, *w, *g;
    const float *log_alpha, *gamma_stat, *S_in;
    const float *grad_y, *grad_S_out;
    float eps;
    float *grad_q, *grad_k, *grad_z, *grad_b, *grad_log_alpha;
    float *grad_v, *grad_w, *grad_g;
    float *grad_gamma_stat, *grad_S_in;
    void *workspace;
    size_t workspace_bytes;
} gdelta_bwd_args;

/* Workspace gdelta_bwd needs for these arguments (0 if they are invalid). */
GDELTA_API size_t gdelta_bwd_workspace_bytes(const gdelta_bwd_args *args);

/* Backward pass; see gdelta_bwd_args. */
GDELTA_API gdelta_status gdelta_bwd(const gdelta_bwd_args *args, void *stream);

/* Chunked forward; see gdelta_fwd_args. */
GDELTA_API gdelta_status gdelta_fwd_chunked(const gdelta_fwd_args *args, void *stream);

/*
 * Chunked forward that allocates nothing and needs no workspace argument.
 * The pages describe nothing like it: it exists for callers that cannot
 * allocate device memory when they run the forward -- code inside a runtime
 * that plans all device memory in advance, or latency-critical code that must
 * not call cudaMalloc (it synchronises the device and can fail).  The scratch
 * the tensor-core path needs lives in a fixed 32 MiB device array inside the
 * library, which every device that loads the library holds until the process
 * exits; args->workspace and args->workspace_bytes are ignored.
 *
 *  - Limit: gdelta_fwd_workspace_bytes(args) must not exceed 32 MiB (105 KiB
 *    per 64-token window of each batch row and head, plus one int per window:
 *    312 windows, e.g. B = 1, H = 16, T <= 1216, or B * H = 8, T <= 2496).  Larger problems return
 *    GDELTA_ERR_WORKSPACE before any launch.
 *  - The first call on a device looks up the array's device address (a CUDA
 *    runtime call); make that first call before capturing any stream.
 *  - Every call uses the same array.  Each call writes every scratch entry it
 *    later reads, so nothing needs clearing between calls, but two calls
 *    whose kernels overlap on the GPU (different streams, no ordering) race
 *    on the array and give wrong results: order them on one stream.
 *  - Otherwise identical to gdelta_fwd_chunked (same arguments, results and
 *    status codes).
 */
GDELTA_API gdelta_status gdelta_fwd_chunked_noalloc(const gdelta_fwd_args *args, void *stream);

/* One decode step; see gdelta_decode_args. */
GDELTA_API gdelta_status gdelta_decode_step(const gdelta_decode_args *args, void *stream);

/*
 * Five-gate low-rank projection: the fused prologue that produces the mixer's
 * gates from the layer input (Muir review §2.3, "五门融合投影与参数再分配").
 * The decay f, erase b, output g, write w and query-gain q gates share one
 * down-projection of x whose width R is the sum of their ranks (the review's
 * main model: 64, 64, 128, 128, 128; R = 512); each gate has its own
 * up-projection back to d and a per-channel bias, which give its logits:
 *
 *   c        = x w_down                          [N, R]  (in the workspace)
 *   logit_i  = c[:, R_i] w_up[R_i, :] + bias_i   [N, d]  R_i = gate i's block of R
 *
 * and the logits are activated into the form gdelta_fwd_chunked reads (the
 * review fixes the ranges, not every activation; these are the plainest
 * readings with those ranges):
 *   log_alpha = log sigmoid(logit_f)  fp32 (alpha = sigmoid(logit_f) in (0, 1))
 *   b = 2 sigmoid(logit_b)            bf16, in (0, 2)
 *   g = sigmoid(logit_g), w = sigmoid(logit_w)   bf16, in (0, 1)
 *   z = logit_q                       bf16 (the readout applies 2 sigmoid(z))
 *
 *   N          : tokens (rows), >= 1
 *   d          : model width = H * d_head, a multiple of 256; the [N, d]
 *                outputs are the mixer's [B, T, H, d_head] tensors when
 *                N = B * T (heads contiguous, h-major)
 *   ranks      : per gate in the order f, b, g, w, q; each a multiple of 64,
 *                their sum R a multiple of 256 and at most 2048
 *   x          : [N, d] bf16
 *   w_down     : [d, R] bf16, columns grouped f | b | g | w | q
 *   w_up       : [R, d] bf16, rows grouped the same way
 *   bias       : [5, d] fp32, one row per gate in the same order
 *   log_alpha  : [N, d] fp32 out;  b, g, w, z : [N, d] bf16 out
 *   workspace  : gdelta_gate_proj_workspace_bytes(args) bytes of device memory
 *                for the codes c (GDELTA_ERR_WORKSPACE if smaller)
 * Both products run on tcgen05 tensor cores (bf16 operands, fp32
 * accumulation).  Between them the codes are held as two bf16 parts, c = hi +
 * lo, and the up-projection reads both, so the codes keep about 16 bits (one
 * bf16 part would shift the log-decay by several percent of its rms).  Asynchronous on
 * `stream`; a bounded wait that runs out is reported by
 * gdelta_get_last_device_error as GDELTA_ERR_TIMEOUT.
 */
typedef struct gdelta_gate_proj_args {
    int32_t N, d;
    int32_t ranks[5];
    const void *x;
    const void *w_down;
    const void *w_up;
    const float *bias;
    float *log_alpha;
    void *b, *g, *w, *z;
    void *workspace;
    size_t workspace_bytes;
} gdelta_gate_proj_args;

/* Workspace gdelta_gate_proj needs (0 if the arguments are invalid). */
GDELTA_API size_t gdelta_gate_proj_workspace_bytes(const gdelta_gate_proj_args *args);

/* Five-gate projection; see gdelta_gate_proj_args. */
GDELTA_API gdelta_status gdelta_gate_proj(const gdelta_gate_proj_args *args, void *stream);

/*
 * Limit of the tensor-core kernels' bounded waits (failure detection; the
 * papers specify no such limit).  Every wait of a tensor-core forward kernel on
 * another party -- an MMA completion, a window record, the other CTA of its
 * cluster, the readout warps -- polls its mbarrier at most `polls` times; when
 * the limit runs out the kernel records GDELTA_ERR_TIMEOUT in the device status
 * word, issues no further work, lets its own copies and MMAs in flight finish,
 * frees its tensor memory and returns.  polls = 0 restores the default of
 * 2^20 polls.  The setting is process-wide, read when a call is queued (calls
 * already queued keep their limit), and applies to gdelta_fwd_chunked and
 * gdelta_fwd_chunked_noalloc on the tensor-core path, to gdelta_gate_proj and
 * to gdelta_bwd (its waits for bulk copies of chunk states; a wait that runs
 * out is reported and then drained with a fixed limit); the other kernels do
 * not wait.  A limit far below the time the hardware needs turns ordinary waits
 * into timeouts: the call then reports GDELTA_ERR_TIMEOUT and its outputs are
 * unreliable, but the device stays usable.  Always returns GDELTA_OK.
 */
GDELTA_API gdelta_status gdelta_set_wait_limit(uint32_t polls);

/*
 * Failure-path test switch (no counterpart in the papers).  With on = 1 every
 * call queued afterwards that gdelta_set_wait_limit governs first waits on an
 * mbarrier that nothing ever completes, before it issues any copy or MMA; the
 * wait runs out after the set limit, the kernels skip their work and return,
 * and gdelta_get_last_device_error reports GDELTA_ERR_TIMEOUT.  The outputs of
 * such a call are not written.  on = 0 (the default) turns it
 * off.  Nothing faults or hangs: the failing wait is an ordinary bounded wait.
 * Process-wide; returns GDELTA_ERR_INVALID_ARG for values other than 0 and 1.
 */
GDELTA_API gdelta_status gdelta_set_wait_timeout_test(int32_t on);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns GDELTA_OK, GDELTA_ERR_TIMEOUT (a kernel's bounded
 * wait ran out), GDELTA_ERR_RANGE (the tensor-core path met an operand
 * outside its fp16 range; its results are unreliable, rerun with
 * GDELTA_PATH_SIMT) or GDELTA_ERR_CUDA (the synchronisation itself failed).
 */
GDELTA_API gdelta_status gdelta_get_last_device_error(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDELTA_H */
