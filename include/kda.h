/*
 * kda.h -- C ABI of the Kimi Delta Attention (KDA) library for NVIDIA B200
 * (sm_100a). Plain pointers and sizes only; no C++ or framework types.
 *
 * The operator (page "atlas_core/kimi_k3/kda.rs", module doc and
 * `kda_recurrent_step`): per sequence and head, a state S of d_k x d_v fp32
 * values (row = key channel) evolves token by token as
 *     S     <- diag(exp(g_t)) S                 (decay on the key axis)
 *     delta <- sigmoid(beta_t) (v_t - S^T k_t)  (beta_t is a logit)
 *     S     <- S + k_t delta^T
 *     o_t   <- scale S^T q_t
 * with q_t, k_t optionally L2-normalised first as x / sqrt(sum x^2 + 1e-6)
 * (same page, `l2norm_rows`, `KDA_L2_EPS`) and g_t optionally clamped from
 * below, g_t <- max(g_t, lower_bound). Optionally the kernel forms g_t itself
 * from the gate input (kda_gate_mode) and takes beta_t as a probability
 * instead of a logit (`beta_is_prob`).
 *
 * Conventions shared by every entry point:
 *  - Every buffer is caller-owned DEVICE memory, except the fields whose
 *    names end in `_host`. The library allocates nothing, frees nothing and
 *    never synchronises (except the two *_status queries, which exist to
 *    wait); work is queued on the caller's stream (a cudaStream_t passed as
 *    `void *`; NULL is the legacy default stream).
 *  - Tensors are dense, row-major, in the layouts given per field. Data
 *    pointers must be 16-byte aligned (beta: 2-byte aligned for bf16,
 *    4-byte for fp32). Outputs must not alias inputs (except where stated).
 *  - Errors: every call validates its arguments on the host first and
 *    returns a status without launching anything if they are bad. A launch
 *    failure returns KDA_ERR_CUDA; kda_last_cuda_error() then gives the CUDA
 *    error code. Nothing aborts, traps or prints.
 *  - q/k L2 normalisation uses eps = 1e-6 inside the square root; states are
 *    always fp32; inputs and the output share one dtype.
 */
#ifndef KDA_H_
#define KDA_H_

/* 0.3.0: kda_chunk_args ends with `debug_flags`; kda_chunk_fwd_status,
 * kda_chunk_fwd_noalloc_status and kda_launch_count added. 0.2.0: kda_step_args and kda_token_args
 * end with `state_out` (0.1.0 had no such field). */
#define KDA_VERSION 300

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size, bad cu_seqlens ... */
    KDA_ERR_UNSUPPORTED = 2,      /* valid request this build has no kernel for */
    KDA_ERR_CUDA = 3,             /* a CUDA call or launch failed */
    KDA_ERR_TIMEOUT = 4,          /* a bounded device-side wait gave up */
    KDA_ERR_WORKSPACE = 5         /* workspace missing or smaller than required */
} kda_status;

typedef enum {
    KDA_DTYPE_F32 = 0,
    KDA_DTYPE_BF16 = 1
} kda_dtype;

/*
 * How the kernel obtains the log-decay g from the `g` input: page
 * "atlas_core/kimi_k3/kda.rs", `bounded_gate`, and page "K3/kda/ops/api.py",
 * `use_gate_in_kernel` / `safe_gate`. With x = g_in + dt_bias[h, c] and
 * rate = exp(A_log[h]), all in fp32:
 *   KDA_GATE_LOG       g = g_in, then max(g, lower_bound) if has_lower_bound
 *   KDA_GATE_SOFTPLUS  g = -rate * softplus(x)        (has_lower_bound must be 0:
 *                                                      the unbounded form has none)
 *   KDA_GATE_SAFE      g = lower_bound * sigmoid(rate * x)  (has_lower_bound must
 *                                                      be 1, lower_bound < 0)
 * A_log: [H] fp32 device, required by the two in-kernel forms. dt_bias:
 * [H, Dk] fp32 device, NULL = zeros. Both are ignored by KDA_GATE_LOG.
 */
typedef enum {
    KDA_GATE_LOG = 0,
    KDA_GATE_SOFTPLUS = 1,
    KDA_GATE_SAFE = 2
} kda_gate_mode;

/*
 * Chunkwise forward: the `chunk_kda` boundary of page "K3/kda/ops/api.py"
 * (signature and preprocessing: q/k L2 norm, sigmoid of beta, in-kernel
 * gate, lower bound, initial_state, output_final_state, chunk_size), minus
 * its backend dispatch. The result equals the token recurrence above run
 * over each sequence; internally tokens are processed chunk_size at a time.
 * The fields after `workspace_bytes` default to the plain operator when
 * zero-initialised.
 */
typedef struct {
    kda_dtype dtype;      /* dtype of q, k, v, g, beta and o */
    int B, T, H, Dk, Dv;  /* q,k,g: [B,T,H,Dk]; v,o: [B,T,H,Dv]; beta: [B,T,H] */
    const void *q, *k, *v;
    const void *g;        /* per-channel log-decay (<= 0), or the gate input (gate_mode) */
    const void *beta;     /* logits, sigmoid applied in the kernel (or see beta_is_prob) */
    void *o;              /* output [B,T,H,Dv] */
    float scale;          /* <= 0 or NaN selects 1/sqrt(Dk) */
    const float *initial_state; /* [N,H,Dk,Dv] fp32, NULL = zeros */
    float *final_state;         /* [N,H,Dk,Dv] fp32 out, NULL = not wanted; may alias initial_state */
    /* Varlen packing: when cu_seqlens != NULL, B must be 1 and the T tokens
     * hold N sequences back to back; sequence n is tokens
     * cu_seqlens[n] .. cu_seqlens[n+1]-1 (int32, device, N+1 entries,
     * cu_seqlens[0] = 0, non-decreasing, cu_seqlens[N] = T). States never
     * cross a sequence boundary. cu_seqlens_host, when given, is a host copy
     * that is validated; without it the device copy is trusted. When
     * cu_seqlens == NULL, N must equal B (each batch row is a sequence). */
    const int32_t *cu_seqlens;
    const int32_t *cu_seqlens_host;
    int N;
    int use_qk_l2norm;    /* 1: q,k <- x / sqrt(sum x^2 + 1e-6) in the kernel */
    int has_lower_bound;  /* 1: g <- max(g, lower_bound); lower_bound must be < 0 */
    float lower_bound;
    int chunk_size;       /* 0 (default, = 64), 32 or 64 tokens per chunk; the result does
                           * not depend on it (up to rounding). 32 runs on CUDA cores only */
    void *workspace;      /* device scratch, 256-byte aligned; see kda_chunk_fwd_workspace_size */
    size_t workspace_bytes;
    kda_gate_mode gate_mode;   /* KDA_GATE_LOG (0): g is the log-decay */
    const float *A_log;        /* [H] fp32, in-kernel gate forms only */
    const float *dt_bias;      /* [H,Dk] fp32 or NULL, in-kernel gate forms only */
    int beta_is_prob;          /* 1: beta is used as given (no sigmoid) */
    unsigned int debug_flags;  /* 0 in normal use; KDA_DEBUG_* bits exercise failure paths */
} kda_chunk_args;

/* debug_flags bit for tests of the bounded device waits: the tensor-core forward
 * (bf16, Dk = Dv = 128, 64-token chunks) does not issue the first input copy of
 * its first kernel, so that kernel's first wait gives up after its 2 s limit, its
 * CTAs leave cleanly and the status word reads KDA_ERR_TIMEOUT (see
 * kda_chunk_fwd_status). The outputs of such a call are undefined. Other shapes
 * ignore the bit. */
#define KDA_DEBUG_STALL_FIRST_WAIT 1u

/* Bytes of device workspace with which kda_chunk_fwd runs its fastest kernel
 * for these arguments (may be 0). Only shapes, dtype and flags are read;
 * pointers may be NULL. For bf16 with d_k = d_v = 128 this is the two-pass
 * tensor-core kernel, whose workspace holds one 65 KiB record per (chunk, head)
 * (about 1.04 bytes per input byte of q, k, g and v); a smaller workspace of at
 * least 256 bytes runs the single-pass tensor-core kernel instead (same result
 * up to rounding), and less than that returns KDA_ERR_WORKSPACE.
 * When there are few (sequence, head) pairs and the sequences are long, the size
 * also covers cutting each sequence into segments whose states are chained
 * afterwards (a few d_k x d_v fp32 states per segment and head, plus two
 * scratch copies of the v rows); this applies to the two-pass kernel and, for
 * d_k = d_v, to the token-recurrent kernel that the other shapes run, and a
 * workspace too small for it runs the unsegmented kernel (same result up to
 * rounding). */
KDA_API kda_status kda_chunk_fwd_workspace_size(const kda_chunk_args *args, size_t *bytes);

/* Queue the chunkwise forward on `stream`. Returns KDA_OK once queued.
 *
 * Device-side failure: the tensor-core kernels (bf16, Dk = Dv = 128, 64-token
 * chunks) wait on their own copies and products with a 2 s limit per wait. A wait
 * that gives up makes its CTA drain what it has in flight, free its tensor memory
 * and leave, and sets the first int32 of the workspace to 1 (it is cleared to 0 at
 * the start of every call); o and final_state are then partly written. Because
 * kda_chunk_fwd never synchronises it cannot return KDA_ERR_TIMEOUT itself: call
 * kda_chunk_fwd_status with the same arguments to read the word. Other shapes run
 * kernels without device waits. */
KDA_API kda_status kda_chunk_fwd(const kda_chunk_args *args, void *stream);

/* Outcome of the last kda_chunk_fwd queued with these arguments on `stream`:
 * waits for the stream to drain (cudaStreamSynchronize), then returns
 * KDA_ERR_TIMEOUT if a bounded device wait gave up (the status word, the first
 * int32 of args->workspace, is non-zero), KDA_OK if it is zero or the arguments
 * select a kernel without device waits, KDA_ERR_CUDA if the copy or the
 * synchronisation failed. The one entry point that synchronises; it reads 4 bytes
 * and launches nothing. */
KDA_API kda_status kda_chunk_fwd_status(const kda_chunk_args *args, void *stream);

/*
 * One recurrent decode step for N sequences at once: the recurrence above
 * applied to one token per sequence (page "atlas_core/kimi_k3/kda.rs",
 * `kda_recurrent_step`), with the state read, updated and written back IN
 * PLACE (a read-modify-write of [N,H,Dk,Dv] fp32), or written to `state_out`
 * when that is given. The out-of-place form serves callers that keep two state
 * buffers and swap them each step, so the previous state stays intact (page
 * "memra-engine tests/kda_fixture_gpu.rs", the decode with `state` / `state_alt`).
 */
typedef struct {
    kda_dtype dtype;      /* dtype of q, k, v, g, beta and o */
    int N, H, Dk, Dv;
    const void *q, *k;    /* [N,H,Dk] */
    const void *v;        /* [N,H,Dv] */
    const void *g;        /* [N,H,Dk] log-decay, or the gate input (gate_mode) */
    const void *beta;     /* [N,H] logits (or see beta_is_prob) */
    float *state;         /* [N,H,Dk,Dv] fp32, updated in place */
    void *o;              /* [N,H,Dv] out */
    float scale;          /* <= 0 or NaN selects 1/sqrt(Dk) */
    int use_qk_l2norm;
    int has_lower_bound;
    float lower_bound;
    kda_gate_mode gate_mode;   /* as in kda_chunk_args */
    const float *A_log;        /* [H] fp32 */
    const float *dt_bias;      /* [H,Dk] fp32 or NULL */
    int beta_is_prob;
    float *state_out;          /* NULL: state updated in place. Else [N,H,Dk,Dv] fp32 out, 16-byte
                                * aligned, equal to state or not overlapping it; state is then
                                * only read */
} kda_step_args;

KDA_API kda_status kda_recurrent_step(const kda_step_args *args, void *stream);

/*
 * One serving decode token for N sequences (page "atlas_core/kimi_k3/kda.rs",
 * `kda_decode_token` followed by `full_rank_output_gate`), fused in one launch:
 *   1. causal depthwise convolution + SiLU over the pre-conv projections x,
 *      channels laid out q | k | v (H*Dk, H*Dk, H*Dv): each channel's window of
 *      the last conv_kernel inputs (oldest first) shifts one slot, x enters the
 *      last slot, y = silu(sum_t conv_w[c][t] * window[c][t]); the windows are
 *      updated IN PLACE;
 *   2. the recurrent step of kda_recurrent_step on q, k, v = y (same gate,
 *      beta, scale and L2-norm options), state updated IN PLACE;
 *   3. when g_out is given, o = sigmoid(g_out) * core / sqrt(mean(core^2) + norm_eps)
 *      per head (RMSNorm without a weight); otherwise o = core.
 * Host-side validation as for kda_recurrent_step; conv_kernel in 1..8.
 */
typedef struct {
    kda_dtype dtype;      /* dtype of x, g, beta, g_out and o */
    int N, H, Dk, Dv;     /* Dk, Dv in {32, 64, 128} */
    int conv_kernel;      /* window length K, 1..8 */
    const void *x;        /* [N, H*(2*Dk+Dv)] pre-conv q | k | v */
    const float *conv_w;  /* [H*(2*Dk+Dv), K] fp32 */
    float *conv_state;    /* [N, H*(2*Dk+Dv), K] fp32, oldest input first, updated in place */
    const void *g;        /* [N,H,Dk] log-decay, or the gate input (gate_mode) */
    const void *beta;     /* [N,H] logits (or see beta_is_prob) */
    float *state;         /* [N,H,Dk,Dv] fp32, updated in place */
    const void *g_out;    /* [N,H,Dv] output-gate input, or NULL for the ungated core output */
    float norm_eps;       /* RMSNorm epsilon of the output gate (>= 0) */
    void *o;              /* [N,H,Dv] out */
    float scale;          /* <= 0 or NaN selects 1/sqrt(Dk) */
    int use_qk_l2norm;
    int has_lower_bound;
    float lower_bound;
    kda_gate_mode gate_mode;
    const float *A_log;   /* [H] fp32, in-kernel gate forms only */
    const float *dt_bias; /* [H,Dk] fp32 or NULL */
    int beta_is_prob;
    float *state_out;     /* NULL: state updated in place; else as in kda_step_args (the conv
                           * windows are always updated in place) */
} kda_token_args;

KDA_API kda_status kda_decode_token(const kda_token_args *args, void *stream);

/*
 * Gradients of the chunkwise forward (the operator above with gate_mode
 * KDA_GATE_LOG): given the output cotangent `dout` and optionally a final-state
 * cotangent, returns dq, dk, dv, dg, dbeta and the initial-state gradient. The
 * pages give no backward formulas: these are the derivatives of the token
 * recurrence of page "atlas_core/kimi_k3/kda.rs" (through the L2 norm, the clamp
 * g <- max(g, lower_bound), whose gradient is zero where the bound is taken, and
 * the sigmoid of beta), taken in one of three forms, the first that applies:
 *   - chunked, on tensor cores: bf16, Dk = Dv = 128, has_lower_bound with
 *     lower_bound >= -5. The forward is rerun in its two-pass chunk form, saving
 *     each 64-token chunk's entering state; the state cotangent is carried back
 *     over the chunks with tcgen05 products (over the forward's segments when the
 *     (sequence, head) pairs are few), and the chunk-local gradients are formed on
 *     warp-level MMAs;
 *   - micro-chunk: bf16, Dk = 32, Dv in {32, 64}, has_lower_bound with lower_bound
 *     >= -10, at least 256 (sequence, head) pairs. The 16-token micro-chunk forward
 *     saves each micro-chunk's entering state (bf16); then one warp per (sequence,
 *     head) walks its micro-chunks from the last with the state cotangent in
 *     registers, every product a warp-level MMA;
 *   - otherwise the token recurrence: a recompute of the forward stores the state
 *     every 16 tokens; a reverse sweep reruns each 16-token stretch forward from
 *     its checkpoint and walks it back, each (sequence, head) split by value
 *     columns over a cluster of Dv/32 CTAs; CUDA cores, fp32.
 * Every form gives the same gradients up to rounding. Validation as kda_chunk_fwd
 * (q, k, v, g, dout and dq, dk, dv, dg 16-byte aligned; beta and dbeta aligned to
 * their element); g is the log-decay (the in-kernel gate forms are not covered).
 */
typedef struct {
    kda_dtype dtype;            /* of q, k, v, g, beta, dout and dq, dk, dv, dg, dbeta */
    int B, T, H, Dk, Dv;        /* as kda_chunk_args */
    const void *q, *k, *v, *g, *beta;
    const void *dout;           /* [B,T,H,Dv] cotangent of o */
    float scale;                /* <= 0 or NaN selects 1/sqrt(Dk) */
    const float *initial_state; /* [N,H,Dk,Dv] or NULL (zeros) */
    const float *dfinal_state;  /* [N,H,Dk,Dv] cotangent of the final state, or NULL */
    void *dq, *dk, *dv, *dg;    /* out, layouts of q, k, v, g */
    void *dbeta;                /* out, [B,T,H] */
    float *dinitial_state;      /* out [N,H,Dk,Dv], or NULL when not wanted */
    const int32_t *cu_seqlens;  /* as kda_chunk_args */
    const int32_t *cu_seqlens_host;
    int N;
    int use_qk_l2norm;
    int has_lower_bound;
    float lower_bound;
    int beta_is_prob;           /* 1: beta is a probability (dbeta is then d/dprob) */
    void *workspace;            /* device scratch of kda_chunk_bwd_workspace_size() bytes, 16-byte aligned
                                   (256-byte aligned for the segment form) */
    size_t workspace_bytes;
} kda_chunk_bwd_args;

/* Bytes of workspace with which kda_chunk_bwd runs its fastest form for these
 * shapes: for the chunked form, the forward's records and chunk table, a 96 KB
 * record per 64-token chunk and head (the chunk's entering state, D and the
 * cotangent chain's output) and, when the (sequence, head) pairs are few, three
 * d x d fp32 maps per segment and head; for the
 * micro-chunk form, the saved bf16 states (one d_k x d_v tile per 16 tokens and
 * head, plus one slot per sequence); for the token recurrence, the state
 * checkpoints (one d_k x d_v fp32 state per 16 tokens per head), a scratch of 16
 * states per (sequence, head) and a small header, and, when there are few
 * (sequence, head) pairs of long sequences and d_k = d_v, the buffers of its
 * segment form. Each figure is at least the plain token form's. A smaller
 * workspace (but at least the plain token form's, 256-byte aligned for the other
 * forms) runs the next form that fits (same result up to rounding); less than the
 * plain token form's returns KDA_ERR_WORKSPACE. Only shapes are read. */
KDA_API kda_status kda_chunk_bwd_workspace_size(const kda_chunk_bwd_args *args, size_t *bytes);

KDA_API kda_status kda_chunk_bwd(const kda_chunk_bwd_args *args, void *stream);

/*
 * Chunkwise forward for callers that cannot allocate device memory. This entry
 * point has no counterpart in the pages; it exists for callers that run under a
 * fixed device-memory plan and may not allocate once running (an inference
 * engine that reserves its memory at start-up, a plug-in whose host application
 * owns every device buffer, a C host with no allocator at the call site), for
 * whom kda_chunk_fwd's workspace is out of reach.
 *
 * Same arguments and result as kda_chunk_fwd; `workspace` and `workspace_bytes`
 * are ignored. The scratch it needs comes from a fixed 4096-byte array in the
 * library's own device memory (one per device, held from library load until
 * process exit); requests needing more than that return KDA_ERR_WORKSPACE (none
 * do today: the chunk kernels need at most 256 bytes). Nothing is allocated or
 * freed.
 *  - The first call on a device looks up that array's device address (a
 *    cudaGetSymbolAddress with the device current); make that first call before
 *    any stream capture.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents; the library clears what must start at zero. Calls whose work
 *    overlaps on the GPU (different streams, no ordering) race on it: order them.
 *  - The array's address is looked up on every call, so a device reset (which
 *    reloads the library's device code) does not leave a stale address behind.
 *  - The status word of the bounded device waits (see kda_chunk_fwd) lives in
 *    that array, out of the caller's reach: read it with
 *    kda_chunk_fwd_noalloc_status.
 */
KDA_API kda_status kda_chunk_fwd_noalloc(const kda_chunk_args *args, void *stream);

/* kda_chunk_fwd_status for the allocation-free entry point: synchronises
 * `stream`, then reports whether a bounded device wait of the last
 * kda_chunk_fwd_noalloc with these arguments on this device gave up
 * (KDA_ERR_TIMEOUT), or KDA_OK. Calls on other streams since then may have
 * overwritten the word. */
KDA_API kda_status kda_chunk_fwd_noalloc_status(const kda_chunk_args *args, void *stream);

/* Static, human-readable name of a status. */
KDA_API const char *kda_status_string(kda_status status);

/* CUDA error code (cudaError_t as int) of the last KDA_ERR_CUDA returned on
 * this host thread, 0 if none. */
KDA_API int kda_last_cuda_error(void);

/* Kernel launches the library has queued since it was loaded, over all host
 * threads and devices: a diagnostic for benchmarks, which read it before and
 * after a timed region. A launch recorded into a CUDA graph counts once, when it
 * is captured, not when the graph is replayed. */
KDA_API unsigned long long kda_launch_count(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH; equal to KDA_VERSION of
 * the header the library was built with. A caller built against an older header
 * passes shorter argument structs, so compare the two before calling. */
KDA_API int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
