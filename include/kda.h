/*
 * kda.h — C ABI of the B200 (sm_100a) Kimi Delta Attention layer-forward library.
 *
 * The operation (Kimi Linear report, section 3, Eq. 1; "KDA Recurrence"
 * problem page, problem statement), per batch row b and head h, with the
 * state S a D_k x D_v matrix:
 *
 *   alpha_t = exp(g_min * sigmoid(z_t))                        (decay gate)
 *   S_t     = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o~_t    = S_t^T q_t                          (read from the updated state)
 *   x_t     = RMSNorm_{D_v}(o~_t) * sigmoid(gate_t),  RMSNorm(u) = u / sqrt(mean(u^2) + eps)
 *   y_t     = concat_h(x_t) W_o^T                 (W_o is D_model x H*D_v)
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - Every tensor pointer is DEVICE memory owned by the caller, contiguous and
 *   row-major in exactly the shapes given, and aligned to its element size
 *   (workspaces: 256 bytes).  Tensor-core and vectorised paths additionally
 *   want 16-byte aligned bases; with a less aligned pointer the call takes an
 *   exact SIMT path instead (or fails with INVALID_ARG when that engine was
 *   demanded).  The library allocates nothing; scratch comes from a caller
 *   workspace whose size the matching *_workspace_size query returns.
 * - "dtype" tensors hold fp32 (KDA_F32) or bf16 (KDA_BF16) values; all inputs
 *   of one call share it.  State and log-decay tensors are always fp32.
 * - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream).  A call returns once its kernels are queued.
 * - Arguments are validated on the host before any launch; on failure nothing
 *   is launched and a status other than KDA_OK is returned.  kda_last_error()
 *   then gives a one-line message (thread-local, valid until the next call).
 * - Outputs must not overlap inputs, except where an entry point says so.
 * - Kernels never trap.  A device-side wait that runs out sets *dev_status to
 *   KDA_ERR_TIMEOUT (when the caller passed dev_status) and the kernel returns.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kda_status {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, g_min >= 0, overlap */
    KDA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement (dtype, size) */
    KDA_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than the size query's answer */
    KDA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 5       /* a device-side bounded wait expired (reported via dev_status) */
} kda_status_t;

typedef enum kda_dtype { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype_t;

/* Engine selection for kda_chunk_fwd. */
typedef enum kda_engine {
    KDA_ENGINE_AUTO = 0,   /* tensor-core engine when the shape allows it, else SIMT */
    KDA_ENGINE_SIMT = 1,   /* exact-fp32 SIMT engine (any D_k, D_v <= 128, chunk <= 64) */
    KDA_ENGINE_TC = 2      /* tcgen05 engine (bf16, D_k = D_v = 128, chunk = 64) */
} kda_engine_t;

/* Name of a status code ("KDA_OK", ...).  Never NULL. */
const char *kda_status_string(kda_status_t status);

/* Message describing the last failure on the calling thread ("" if none). */
const char *kda_last_error(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int kda_version(void);

/* Number of kernel launches this process has issued through the library so
 * far (all devices and threads).  For counting the kernels of a timed region. */
uint64_t kda_launch_count(void);

/* Number of bounded device-side waits that ran out on the current device since
 * the last reset (0 in a healthy run); reset != 0 clears it.  Synchronous. */
kda_status_t kda_device_timeouts(uint32_t *count, int reset);

/* Writes that a checked build (compiled with -DKDA_CHECKED: libkda_checked.so)
 * found outside their buffer and skipped, on the current device, since the
 * last reset; reset != 0 clears it.  *checked_build (if not NULL) is set to 1
 * in a checked build, 0 otherwise (where the count stays 0).  The checks cover
 * every global write through an offset the library computes: workspace
 * records, segment maps and entering states, checkpoints and stashes, final
 * states and staged outputs.  Synchronous. */
kda_status_t kda_device_bounds_errors(uint32_t *count, int reset, int *checked_build);

/* Self-test of the bounded-wait path the tensor-core kernels use: launches a
 * one-CTA kernel that waits on a barrier nothing completes, gives up after
 * limit_us microseconds (1 .. 1e6), writes KDA_ERR_TIMEOUT to *dev_status (a
 * device int32), counts one timeout and returns.  Nothing traps or faults and
 * the context stays usable.  Asynchronous on `stream`. */
kda_status_t kda_selftest_wait_timeout(int32_t *dev_status, uint32_t limit_us, void *stream);

/*
 * kda_gate — decay gate of the "KDA Recurrence" page:
 *   log_alpha[i] = g_min * sigmoid(z[i])   for i in [0, n)
 * so alpha = exp(log_alpha) lies in [exp(g_min), 1].
 *   z         : n values of `dtype` (the decay logits, same shape as the keys)
 *   log_alpha : n fp32 values, out
 * Errors: INVALID_ARG if n < 0, a pointer is NULL/misaligned, or g_min is not
 * a finite negative number (the page's Constraints require g_min < 0).
 */
kda_status_t kda_gate(const void *z, kda_dtype_t dtype, int64_t n, float g_min,
                      float *log_alpha, void *stream);

/*
 * kda_chunk_fwd — prefill: the Eq. 1 recurrence over whole sequences with the
 * chunkwise (gated WY / UT-transform) algorithm of the Kimi Linear report,
 * section 3.1 and appendix B (Propositions 1-2, Eqs. 16-19).  Sequences are
 * cut into chunks of `chunk` tokens; inside a chunk the rank-1 updates are
 * folded into a unit-lower-triangular solve, and the state is carried from
 * chunk to chunk.  The last chunk of a sequence may be partial.
 *
 * Layout ("KDA Recurrence" page, problem statement):
 *   q, k, z       (B, S, H, D_k)  dtype
 *   log_decay     (B, S, H, D_k)  fp32 log(alpha) in [g_min, 0] (values outside
 *                 that range are clamped to it), or NULL to use z
 *   g_min         the lower log-decay bound, finite and < 0 (always required:
 *                 with log_decay it is the caller's bound on those values)
 *   v             (B, S, H, D_v)  dtype
 *   beta          (B, S, H)       dtype, in [0, 1]
 *   initial_state (B, H, D_k, D_v) fp32, or NULL for zeros; never written
 *                 unless it is the same pointer as final_state (in-place
 *                 handoff is allowed: each sequence reads its state first)
 *   gate_logits   (B, S, H, D_v)  dtype, or NULL
 *   o             (B, S, H, D_v)  dtype, out.  With gate_logits == NULL it
 *                 receives o~_t; otherwise RMSNorm(o~_t) * sigmoid(gate_t).
 *   final_state   (B, H, D_k, D_v) fp32, out, or NULL to skip
 * S = 0 is allowed (no token: final_state = initial_state).
 * The tensor-core engine covers bf16, D_k = D_v = 128, chunk 64 and
 * g_min >= -5.5 (the bound keeps every in-chunk decay factor it forms inside
 * the fp32/bf16 exponent range); KDA_ENGINE_AUTO falls back to SIMT otherwise.
 * Errors: INVALID_ARG (see conventions), UNSUPPORTED (D_k or D_v > 128,
 * chunk > 64, or KDA_ENGINE_TC on a shape it does not cover), WORKSPACE.
 */
typedef struct kda_chunk_args {
    int64_t B, S;
    int32_t H, D_k, D_v;
    kda_dtype_t dtype;
    const void *q;
    const void *k;
    const void *v;
    const void *z;
    const float *log_decay;
    float g_min;
    const void *beta;
    const float *initial_state;
    const void *gate_logits;
    float eps;
    void *o;
    float *final_state;
    void *workspace;
    size_t workspace_bytes;
    int32_t chunk;          /* 0 = library default (64) */
    kda_engine_t engine;
    int32_t *dev_status;    /* optional device int32, 0 = fine; may be NULL */
    void *stream;
} kda_chunk_args;

/* Workspace bytes kda_chunk_fwd needs for these arguments (pointers unused).
 * The tensor-core engine's size depends on the current device's SM count (its
 * segment count does): query it with the device current that will run the
 * call.  kda_chunk_fwd re-checks the size and returns KDA_ERR_WORKSPACE if the
 * workspace is smaller. */
kda_status_t kda_chunk_workspace_size(const kda_chunk_args *args, size_t *bytes);

kda_status_t kda_chunk_fwd(const kda_chunk_args *args);

/*
 * kda_gdn_chunk_fwd — the Gated DeltaNet special case of the prefill (the
 * DPLR post's comparison of GDN with KDA: one scalar decay per token and head,
 *   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 * i.e. Eq. 1 with Diag(alpha_t) = alpha_t I), with the same chunkwise
 * algorithm, output readout (read after the update), optional fused RMSNorm
 * and sigmoid gate, and state handling as kda_chunk_fwd.  Arguments are those
 * of kda_chunk_fwd except the decay inputs, which hold one value per token
 * and head:
 *   z             (B, S, H)  dtype decay logits, alpha = exp(g_min * sigmoid(z))
 *   log_decay     (B, S, H)  fp32 log(alpha) in [g_min, 0], or NULL to use z
 * Because the decay ratio of two tokens is one number, the intra-chunk
 * products are plain products of the raw keys and queries scaled per token
 * pair: the tensor-core engine (bf16, D_k = D_v = 128, chunk 64) has no bound
 * on g_min.  Other shapes run the exact SIMT engine.
 * Errors: as kda_chunk_fwd.
 */
kda_status_t kda_gdn_chunk_workspace_size(const kda_chunk_args *args, size_t *bytes);

kda_status_t kda_gdn_chunk_fwd(const kda_chunk_args *args);

/*
 * kda_recurrent_bwd — gradient of the prefill recurrence for training: given
 * dL/do~_t for every token (o~_t = S_t^T q_t, the core output before any
 * normalisation) and dL/dS_T, the gradients with respect to q, k, v, beta,
 * the decay input (z, or log_decay when that is given) and the initial state.
 * Reverse-mode differentiation of Eq. 1 (Kimi Linear report, section 3) token
 * by token, exact fp32: the state is checkpointed every 64 tokens on a forward
 * pass and each chunk's states are recomputed from its checkpoint before its
 * tokens are differentiated in reverse order.  (The pages motivate the chunk
 * form by training; this is the recurrent form of its backward pass.)
 *   q, k, z/log_decay, v, beta, initial_state, g_min : as kda_chunk_fwd
 *   d_o           (B, S, H, D_v)  dtype: dL/do~
 *   d_final_state (B, H, D_k, D_v) fp32, or NULL for zero
 *   dq, dk, dz    (B, S, H, D_k)  fp32 out (dz is d/dz, or d/dlog_decay with
 *                 a log_decay input: zero where that input was clamped)
 *   dv            (B, S, H, D_v)  fp32 out;  dbeta (B, S, H) fp32 out
 *   d_initial_state (B, H, D_k, D_v) fp32 out, or NULL to skip
 * Outputs are overwritten (zeroed on the stream first).  D_k, D_v <= 128.
 * The workspace holds the checkpoints and a per-block stash (size query).
 * Errors: INVALID_ARG, UNSUPPORTED (D_k or D_v > 128), WORKSPACE.
 */
typedef struct kda_recurrent_bwd_args {
    int64_t B, S;
    int32_t H, D_k, D_v;
    kda_dtype_t dtype;
    const void *q;
    const void *k;
    const void *v;
    const void *z;
    const float *log_decay;
    float g_min;
    const void *beta;
    const float *initial_state;
    const void *d_o;
    const float *d_final_state;
    float *dq;
    float *dk;
    float *dv;
    float *dbeta;
    float *dz;
    float *d_initial_state;
    void *workspace;
    size_t workspace_bytes;
    void *stream;
} kda_recurrent_bwd_args;

kda_status_t kda_recurrent_bwd_workspace_size(const kda_recurrent_bwd_args *args, size_t *bytes);

kda_status_t kda_recurrent_bwd(const kda_recurrent_bwd_args *args);

/*
 * kda_chunk_bwd — the same gradients as kda_recurrent_bwd (same arguments,
 * same outputs), computed in the chunk form of the recurrence (Kimi Linear
 * report, section 3.1 and appendix B, Props. 1-2: the WY/UT representation the
 * pages motivate by training).  Chunks of 64 tokens run in parallel for the
 * per-chunk algebra (decayed K K^T and Q K^T, T = (I + A)^{-1} by forward
 * substitution, W, U, and every per-chunk gradient); only the state and its
 * gradient pass through the chunks in order (one 16-value-column slice of
 * the state per CTA).  Exact fp32 arithmetic; every decay factor is the
 * exponential of a difference <= 0, so any g_min works.  The reverse-mode
 * lines it evaluates are listed in csrc/chunk_bwd.cu.
 * Outputs are fully written (no zeroing needed).  The workspace holds one
 * record per (b, h, chunk): 4 (C (4 D_k + 3 D_v + 3 C) + 2 D_k D_v
 * + ceil(D_v / 16) D_k) bytes with C = 64, rounded up to 16 bytes (404 KB at
 * D_k = D_v = 128); query it with kda_chunk_bwd_workspace_size.
 * Errors: as kda_recurrent_bwd; UNSUPPORTED if B*H*chunks exceeds 2^31 - 1.
 */
kda_status_t kda_chunk_bwd_workspace_size(const kda_recurrent_bwd_args *args, size_t *bytes);

kda_status_t kda_chunk_bwd(const kda_recurrent_bwd_args *args);

/*
 * kda_dplr_recurrent_fwd — the general diagonal-plus-low-rank recurrence of the
 * "Diagonal-Plus-Low-Rank Matrices and Kimi Delta Attention" post (sections 1
 * and 3), the comparator of the KDA engines:
 *   S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,   o_t = S_t^T q_t
 * with free erase directions a_t, b_t and the readout from the updated state
 * (KDA's).  KDA is the case a_t = beta_t k_t, b_t = k_t * alpha_t with the
 * write key beta_t k_t; without that binding the chunkwise UT/WY form of
 * kda_chunk_fwd does not apply, and this entry point evaluates the recurrence
 * token by token, exact fp32 (kda_dplr_chunk_fwd below is its chunk form).
 *   q, k, a, b, z (B, S, H, D_k) dtype;  log_decay (B, S, H, D_k) fp32 or NULL
 *   v (B, S, H, D_v) dtype;  initial_state (B, H, D_k, D_v) fp32 or NULL
 *   o (B, S, H, D_v) dtype out;  final_state (B, H, D_k, D_v) fp32 out or NULL
 * Errors: INVALID_ARG, UNSUPPORTED (D_k or D_v > 128).
 */
typedef struct kda_dplr_args {
    int64_t B, S;
    int32_t H, D_k, D_v;
    kda_dtype_t dtype;
    const void *q;
    const void *k;
    const void *v;
    const void *a;
    const void *b;
    const void *z;
    const float *log_decay;
    float g_min;
    const float *initial_state;
    void *o;
    float *final_state;
    void *stream;
} kda_dplr_args;

kda_status_t kda_dplr_recurrent_fwd(const kda_dplr_args *args);

/*
 * kda_dplr_chunk_fwd — the same recurrence and outputs as kda_dplr_recurrent_fwd,
 * in chunk form: with y_t = b_t^T S_{t-1}, the chunk's erased rows Y solve a
 * unit-lower-triangular system (I + Ba) Y = (b * e^{G_{t-1}}) S + Bk V built
 * from decayed products of b with a and k, and the outputs and the next state
 * follow from S, V and Y (derivation in csrc/dplr_chunk.cu; the post's
 * sections 1 and 3 give the recurrence, the Kimi Linear report's appendix B
 * the same construction for KDA's binding).  Chunks of 64 tokens in parallel
 * for the per-chunk algebra; the state passes through the chunks in order (one
 * 16-value-column slice per CTA).  Exact fp32 arithmetic; any g_min.
 *   args            : as kda_dplr_recurrent_fwd
 *   workspace       : device memory, 256-byte aligned, at least the size
 *                     kda_dplr_chunk_workspace_size returns: one record per
 *                     (b, h, chunk) of 4 (D_k rounded up to 4 + C (3 D_k +
 *                     C + 2 D_v) + D_k D_v) bytes with C = 64, rounded up to
 *                     16 bytes (240.5 KB at D_k = D_v = 128)
 * Errors: as kda_dplr_recurrent_fwd; WORKSPACE; UNSUPPORTED if B*H*chunks
 * exceeds 2^31 - 1.
 */
kda_status_t kda_dplr_chunk_workspace_size(const kda_dplr_args *args, size_t *bytes);

kda_status_t kda_dplr_chunk_fwd(const kda_dplr_args *args, void *workspace, size_t workspace_bytes);

/*
 * kda_decode_step — one token of the Eq. 1 recurrence for B independent
 * sequences, fused in one pass over the fp32 state (the fused recurrent
 * form: decay the state, predict k^T S, form the residual beta (v - pred),
 * write k residual^T, read q^T S), the state updated IN PLACE: decode state
 * is owned by the caller and advanced by design.
 *   q, k, z       (B, H, D_k)  dtype;   log_decay (B, H, D_k) fp32 or NULL
 *   g_min         lower log-decay bound, finite and < 0 (always required)
 *   v             (B, H, D_v)  dtype;   beta (B, H) dtype
 *   state         (B, H, D_k, D_v) fp32, read and written
 *   gate_logits   (B, H, D_v)  dtype or NULL (as in kda_chunk_fwd)
 *   o             (B, H, D_v)  dtype, out
 * Errors: INVALID_ARG, UNSUPPORTED (D_k or D_v > 128).
 */
typedef struct kda_decode_args {
    int64_t B;
    int32_t H, D_k, D_v;
    kda_dtype_t dtype;
    const void *q;
    const void *k;
    const void *v;
    const void *z;
    const float *log_decay;
    float g_min;
    const void *beta;
    float *state;
    const void *gate_logits;
    float eps;
    void *o;
    void *stream;
} kda_decode_args;

kda_status_t kda_decode_step(const kda_decode_args *args);

/*
 * kda_norm_gate — per-head RMS normalisation over D_v then the sigmoid output
 * gate ("KDA Recurrence" page, problem statement):
 *   x[n,h,:] = o[n,h,:] / sqrt(mean_j o[n,h,j]^2 + eps) * sigmoid(gate[n,h,:])
 *   o, gate_logits, x : (N, H, D_v) dtype.  x may equal o (in place).
 */
kda_status_t kda_norm_gate(const void *o, const void *gate_logits, int64_t N,
                           int32_t H, int32_t D_v, float eps, void *x,
                           kda_dtype_t dtype, void *stream);

/*
 * kda_out_proj — head concat and output projection ("KDA Recurrence" page):
 *   y[n, m] = sum_i x[n, i] * W_o[m, i],   i = h * D_v + j
 *   x (N, K) dtype with K = H * D_v;  W_o (D_model, K) dtype;  y (N, D_model) dtype.
 * bf16 with K % 64 == 0 and D_model % 16 == 0 runs on the tcgen05 tensor
 * cores (fp32 accumulation); anything else runs an exact-fp32 SIMT GEMM.
 */
kda_status_t kda_out_proj(const void *x, const void *W_o, int64_t N, int32_t K,
                          int32_t D_model, void *y, kda_dtype_t dtype, void *stream);

/*
 * kda_out_norm_gate_proj — kda_norm_gate then kda_out_proj:
 *   y = concat_h(RMSNorm(o_h) * sigmoid(gate_h)) W_o^T
 *   o, gate_logits (N, H, D_v); W_o (D_model, H*D_v); y (N, D_model); all dtype.
 * The normalised activations go to the workspace (size query below).
 */
kda_status_t kda_out_norm_gate_proj_workspace_size(int64_t N, int32_t H, int32_t D_v,
                                                   kda_dtype_t dtype, size_t *bytes);

kda_status_t kda_out_norm_gate_proj(const void *o, const void *gate_logits,
                                    const void *W_o, int64_t N, int32_t H, int32_t D_v,
                                    int32_t D_model, float eps, void *y, kda_dtype_t dtype,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * kda_out_norm_gate_proj_noalloc — the same computation as
 * kda_out_norm_gate_proj for callers that cannot allocate device memory: an
 * integration point that passes the library only its input and output
 * buffers, or a loop that must not call cudaMalloc while it runs because the
 * call can synchronise the device.  No page describes this variant; it exists
 * for those callers only.
 *   o, gate_logits (N, H, D_v); W_o (D_model, H*D_v); y (N, D_model); all dtype.
 * The normalised activations live in a fixed 8 MiB scratch array inside the
 * library's device memory (held by every GPU that loads the library until the
 * process exits) instead of a caller workspace, so this call never allocates.
 * Limit: N * H * D_v * element_size <= 8 MiB, else KDA_ERR_UNSUPPORTED and
 * nothing is launched.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress); make that first call before any stream
 * capture.  All calls on a device share the array and it keeps the last call's
 * contents (each call writes every byte it reads, so nothing needs clearing);
 * calls whose kernels overlap on the GPU race on it and must be ordered by the
 * caller.
 */
kda_status_t kda_out_norm_gate_proj_noalloc(const void *o, const void *gate_logits,
                                            const void *W_o, int64_t N, int32_t H, int32_t D_v,
                                            int32_t D_model, float eps, void *y, kda_dtype_t dtype,
                                            void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
