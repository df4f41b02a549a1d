/*
 * libkda -- Kimi Delta Attention (KDA) forward pass on NVIDIA B200 (sm_100a).
 *
 * What is computed (Kimi K3 technical report, section 2.1.1, Eq. 1 and Eq. 5):
 * per (batch b, head h) chain a state S_t in R^{dk x dv} evolves as
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = scale * S_t^T q_t,          alpha_t = exp(g_t)  (per key channel),
 *
 * where g_t in R^{dk} is the per-channel LOG-decay (the report's lower-bounded
 * gate g = g_min * Sigmoid(e^A z), g_min = -5, keeps g in (-5, 0); the library
 * takes g as an input and relies on g <= 0 and on every 16-token window sum of
 * g staying >= -80, which that gate guarantees) and beta_t in (0, 1) is the
 * delta-rule write strength.  The output reads the post-update state.  The
 * report's Eq. 1 has no output scale; this library applies `scale` to o only
 * (default dk^-1/2), never to the state.
 *
 * Prefill evaluates the chunkwise-parallel form of the report (section 2.1.1,
 * Eqs. 3-4: cumulative decay, UT transform, intra/inter-chunk outputs, state
 * carried across chunks); decode applies Eq. 1 to one token per sequence with
 * the state updated in place (section 5.4.2).  Both are mathematically the
 * same recurrence; results differ from an exact evaluation only by rounding.
 *
 * Conventions for every entry point
 *  - All tensor arguments are DEVICE pointers to dense row-major (contiguous)
 *    arrays owned by the caller.  libkda never allocates, frees or retains
 *    them, and keeps no per-call state.  Alignment: every fp32 state pointer
 *    (h0, h_T, S) and every prefill q, k, v, g, o and workspace pointer must be
 *    16-byte aligned; beta and the decode q, k, v, g, o need only be aligned
 *    to their element size.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without synchronising.  Argument errors are
 *    detected synchronously, before anything is enqueued; a failed launch
 *    returns KDA_ERR_CUDA.  Errors raised on the device (a bounded wait that
 *    gave up) are recorded in a device status word read by
 *    kda_get_device_status().
 *  - Thread-safe: no global mutable host state besides a per-context cache of
 *    the status-word address filled on first use (a context re-created after
 *    cudaDeviceReset looks it up again).
 *  - No C++ exception crosses this interface.
 */
#ifndef LIBKDA_KDA_H_
#define LIBKDA_KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kda_stream_t; /* identical to cudaStream_t */

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1, /* NULL required pointer, bad scale, negative size */
  KDA_ERR_SHAPE = 2,       /* unsupported B/H/T/dk/dv/chunk combination */
  KDA_ERR_DTYPE = 3,       /* unknown kda_dtype_t, or dtype not supported by the requested path */
  KDA_ERR_ALIGNMENT = 4,   /* a pointer breaks the alignment rule above */
  KDA_ERR_ALIAS = 5,       /* an output overlaps an input (other than the allowed in-place cases) */
  KDA_ERR_WORKSPACE = 6,   /* workspace missing or smaller than the size query returned */
  KDA_ERR_CUDA = 7,        /* a CUDA runtime call or kernel launch failed */
  KDA_ERR_TIMEOUT = 8,     /* a bounded device-side wait gave up (see kda_get_device_status) */
  KDA_ERR_UNSUPPORTED = 9, /* device is not sm_100 / path not available */
  KDA_ERR_DEVICE = 10      /* device-side bounds check failed (see kda_get_device_status) */
} kda_status_t;

typedef enum {
  KDA_DTYPE_F32 = 0, /* fp32 q, k, v, g, beta, o */
  KDA_DTYPE_BF16 = 1 /* bf16 q, k, v, g, beta, o (state and accumulation stay fp32) */
} kda_dtype_t;

/* Kernel families selectable for prefill (see kda_chunk_fwd). */
typedef enum {
  KDA_PATH_AUTO = 0,   /* library choice */
  KDA_PATH_SIMT16 = 1, /* fp32 CUDA-core chunked kernel, 16-token chunks, any supported dtype/d */
  KDA_PATH_TC32 = 2    /* tcgen05 tensor-core chunked kernel, 32-token chunks, bf16, dk = dv = 128 */
} kda_path_t;

/* What kda_chunk_fwd will launch for a given problem (for benchmarks/tests). */
typedef struct {
  int path;         /* kda_path_t actually used */
  int chunk_size;   /* tokens per chunk of the chosen kernel */
  int segments;     /* in-device context-parallel segments per chain (1 = none) */
  int launches;     /* kernel launches per call */
  size_t workspace; /* bytes of workspace the call needs */
  int segment_tokens; /* tokens per context-parallel segment (the last may be shorter); T if unsegmented */
} kda_plan_t;

/*
 * Plan a prefill call (no device work).  chunk_size selects the kernel:
 * 0 = automatic (KDA_PATH_TC32 for bf16 with dk = dv = 128, else
 * KDA_PATH_SIMT16), 16 = KDA_PATH_SIMT16, 32 = KDA_PATH_TC32.  Returns KDA_OK and
 * fills *plan, or the error kda_chunk_fwd would return for these sizes.
 */
kda_status_t kda_chunk_fwd_plan(int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                int chunk_size, kda_plan_t *plan);

/* Workspace bytes kda_chunk_fwd needs (0 if none, (size_t)-1 on invalid sizes). */
size_t kda_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                    int chunk_size);

/*
 * Prefill / training forward over T tokens for B x H independent chains
 * (Kimi K3 report, section 2.1.1, Eqs. 1-4; in-device context parallelism of
 * section 5.1.1 for long chains).
 *
 *   q, k, g : [B, H, T, dk]  dtype         g = per-channel log-decay (<= 0)
 *   v       : [B, H, T, dv]  dtype
 *   beta    : [B, H, T]      dtype
 *   h0      : [B, H, dk, dv] fp32, or NULL for a zero initial state
 *   o       : [B, H, T, dv]  dtype (written; bf16 outputs are rounded to nearest even)
 *   h_T     : [B, H, dk, dv] fp32 final state, or NULL if not wanted.
 *             h_T == h0 (exactly the same pointer) is allowed: in-place carry.
 *   dk, dv  : each one of 16, 32, 64, 128 (KDA_PATH_TC32: both 128, bf16 only)
 *   T       : >= 0 (T = 0 copies h0, or zeros, to h_T); need not be a
 *             multiple of the chunk size
 *   chunk_size : 0, 16 or 32, as for kda_chunk_fwd_plan (the result does not
 *             depend on it beyond rounding)
 *   scale   : output scale; <= 0 selects dk^-1/2; must be finite
 *   workspace, workspace_bytes : device scratch of at least
 *             kda_chunk_fwd_workspace_size(...) bytes (may be NULL when that is 0);
 *             contents on entry are ignored, on exit undefined
 * o must not overlap any input, and
 * h_T must not overlap any input except by being identical to h0.
 */
kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, const void *g,
                           const void *beta, const float *h0, void *o, float *h_T, int B, int H,
                           int T, int dk, int dv, kda_dtype_t dtype, int chunk_size, float scale,
                           void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * One recurrent decode step, one new token per sequence (Kimi K3 report,
 * Eq. 1 applied once; section 5.4.2: the state is updated in place).
 *
 *   q, k, g : [B, H, dk] dtype;  v : [B, H, dv] dtype;  beta : [B, H] dtype
 *   S       : [B, H, dk, dv] fp32, read and overwritten in place with S_t
 *   o       : [B, H, dv] dtype (written)
 *   dk, dv  : each one of 16, 32, 64, 128;  scale as for kda_chunk_fwd.
 * o must not overlap S or any input; S must not overlap any input.
 */
kda_status_t kda_recurrent_step(const void *q, const void *k, const void *v, const void *g,
                                const void *beta, float *S, void *o, int B, int H, int dk, int dv,
                                kda_dtype_t dtype, float scale, kda_stream_t stream);

/*
 * Prefill that also emits recurrent-state checkpoints for prefix caching
 * (Kimi K3 report, section 5.4.1: after a forward pass the KDA kernel persists
 * the recurrent state at hash-block-aligned positions, so a later request that
 * shares the prefix can copy the snapshot and resume prefill at that token).
 *
 * Same arguments, layouts, alignment, aliasing rules and results as
 * kda_chunk_fwd, plus:
 *   ckpt_interval : hash-block size in tokens; a positive multiple of 64
 *   ckpt          : [B, H, T / ckpt_interval, dk, dv] fp32 (integer division),
 *                   16-byte aligned; entry j is the state after token
 *                   (j + 1) * ckpt_interval - 1, i.e. the state from which
 *                   prefill resumes at token (j + 1) * ckpt_interval (with that
 *                   snapshot as h0).  Written, never read.  May be NULL only when
 *                   T < ckpt_interval (no entry).  Must not overlap any input,
 *                   o or h_T.
 * Returns KDA_ERR_INVALID_ARG for a bad interval or a missing buffer.
 */
kda_status_t kda_chunk_fwd_ckpt(const void *q, const void *k, const void *v, const void *g,
                                const void *beta, const float *h0, void *o, float *h_T, float *ckpt,
                                int ckpt_interval, int B, int H, int T, int dk, int dv,
                                kda_dtype_t dtype, int chunk_size, float scale, void *workspace,
                                size_t workspace_bytes, kda_stream_t stream);

/*
 * Prefill with the decay gate fused into the loads (Kimi K3 report, section
 * 2.1.1, Eq. 5): instead of the log-decay g the call takes the decay logits z
 * and the log-scales A and forms, per token and key channel,
 *     g = g_min * Sigmoid(exp(A[h][c]) * z[b][h][t][c])
 * in fp32 on chip, so g never goes through memory.
 *
 * Same arguments, layouts, alignment, aliasing rules and results as
 * kda_chunk_fwd with g replaced by:
 *   z     : [B, H, T, dk] dtype (16-byte aligned)
 *   A_log : [H, dk] fp32, 4-byte aligned (a per-head scale is the same value
 *           repeated over dk); read only
 *   g_min : the lower bound of the log-decay, in [-5, 0) (the report fixes
 *           -5; a bound below -5 would break the e^{80} range the chunked
 *           kernels rely on); otherwise KDA_ERR_INVALID_ARG
 */
kda_status_t kda_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *z,
                                 const float *A_log, float g_min, const void *beta, const float *h0,
                                 void *o, float *h_T, int B, int H, int T, int dk, int dv,
                                 kda_dtype_t dtype, int chunk_size, float scale, void *workspace,
                                 size_t workspace_bytes, kda_stream_t stream);

/*
 * Output edge of a KDA layer (Kimi K3 report, section 2.1.1, Eq. 6): per-head
 * RMSNorm of the recurrent output followed by the data-dependent sigmoid gate,
 *     y[b,h,t,:] = Sigmoid(gate[b,h,t,:]) * w[h,:] * o[b,h,t,:] / sqrt(mean(o[b,h,t,:]^2) + eps)
 * The projections W_g x (giving `gate`, already split into heads) and W_o are
 * outside the call.
 *
 *   o, gate, y : [B, H, T, dv] dtype, 16-byte aligned; y == o (in place) is
 *                allowed, any other overlap of y with an input is not
 *   rms_weight : [H, dv] fp32, 16-byte aligned
 *   eps        : finite, >= 0
 *   dv         : one of 16, 32, 64, 128
 * Errors are reported like kda_chunk_fwd's; the call allocates nothing.
 */
kda_status_t kda_output_gate(const void *o, const void *gate, const float *rms_weight, float eps, void *y,
                             int B, int H, int T, int dv, kda_dtype_t dtype, kda_stream_t stream);

/*
 * Prefill with the output edge of the KDA layer fused into the output
 * epilogue (Kimi K3 report, section 2.1.1, Eq. 6, without its projections):
 *     y_t = Sigmoid(gate_t) * w_h * o_t / sqrt(mean_j(o_t[j]^2) + eps),
 * o_t being what kda_chunk_fwd would write (the RMS is per token and head,
 * over dv).  On the tensor-core path the epilogue normalises and gates each
 * output tile on chip, so o never reaches memory; on the CUDA-core path the
 * prefill writes o into y's buffer and the edge runs in place after it.
 * Arguments as for kda_chunk_fwd, with o replaced by
 *   gate       : [B, H, T, dv] in dtype (W_g x split into heads), 16-byte aligned
 *   rms_weight : [H, dv] fp32, 16-byte aligned;   eps >= 0
 *   y          : [B, H, T, dv] in dtype, written; must not overlap any input
 *                (gate and rms_weight included)
 * Same workspace size as kda_chunk_fwd.  Errors as for kda_chunk_fwd.
 */
kda_status_t kda_chunk_fwd_outgate(const void *q, const void *k, const void *v, const void *g, const void *beta,
                                   const float *h0, const void *gate, const float *rms_weight, float eps, void *y,
                                   float *h_T, int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                   int chunk_size, float scale, void *workspace, size_t workspace_bytes,
                                   kda_stream_t stream);

/*
 * Segment transition of KDA context parallelism (Kimi K3 report, section
 * 5.1.2, Eq. 17).  The recurrence is linear in its entering state: a prefill
 * of these T tokens that starts from S ends in  S~ + M S,  with
 *     M = M_T ... M_1,   M_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
 * and S~ the end state from S = 0.  This call computes both for every chain in
 * one launch, without q and without writing any output (the transition-only
 * form of the tensor-core kernel: two CTAs per chain, one carrying S~ from
 * zero, one carrying M from I with no value write), so a rank can publish its
 * pair before it knows its entering state.
 *   k, g : [B, H, T, dk]; v : [B, H, T, dv]; beta : [B, H, T]   (dtype)
 *   St   : [B, H, dk, dv] fp32, written (S~)
 *   M    : [B, H, dk, dk] fp32, written, row-major (M[i][j] multiplies S's row j)
 * bf16 with dk = dv = 128 only (KDA_ERR_DTYPE / KDA_ERR_SHAPE otherwise).
 * T = 0 gives S~ = 0 and M = I.  k, v, g, St, M 16-byte aligned; St and M must
 * not overlap each other or the inputs.  Allocates nothing.
 */
kda_status_t kda_chunk_transition(const void *k, const void *v, const void *g, const void *beta, float *St,
                                  float *M, int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                  kda_stream_t stream);

/*
 * Cross-device KDA context parallelism, prefix step (Kimi K3 report, section
 * 5.1.2, Eq. 17).  Each rank holds one segment of every chain; a segment maps
 * its entering state S to S~ + M S.  After one all-gather of the (M_r, S~_r)
 * pairs (the caller's NCCL collective), rank R composes the state entering its
 * segment,
 *     S_in = M_{R-1} (... (M_0 h0 + S~_0) ...) + S~_{R-1},
 * and runs its prefill from S_in.  (M_r, S~_r) of a segment come from
 * kda_chunk_transition (or, on the CUDA-core path, from two prefill calls on
 * it: S~ = h_T from a zero state, M = h_T from h0 = I with v = 0, dk == dv).
 *   M    : [R, B, H, dk, dk] fp32;  St : [R, B, H, dk, dv] fp32 (rank-major)
 *   h0   : [B, H, dk, dv] fp32, or NULL for a zero initial state
 *   S_in : [B, H, dk, dv] fp32, written; must not overlap the inputs
 *   R    : number of earlier segments (0 on the first rank: S_in = h0)
 * All pointers 16-byte aligned; dk, dv one of 16, 32, 64, 128.
 */
kda_status_t kda_kcp_compose(const float *M, const float *St, const float *h0, float *S_in, int R, int B,
                             int H, int dk, int dv, kda_stream_t stream);

/*
 * Speculative-decode replay and verify (Kimi K3 report, section 5.4.2): one
 * recurrent loop over a window of W tokens per sequence.  The first
 * n_replay[b] tokens are the accepted drafts of the previous verification,
 * whose projected inputs the caller cached: they advance the committed state,
 * which is written back to S after the last of them.  The remaining tokens
 * (bonus token and next draft) advance the state on chip only and write their
 * outputs o for verification; S never sees them.
 *
 *   q, k, g  : [B, H, W, dk] dtype;  v : [B, H, W, dv] dtype;  beta : [B, H, W] dtype
 *   S        : [B, H, dk, dv] fp32, 16-byte aligned, updated in place (unchanged
 *              when n_replay[b] == 0)
 *   o        : [B, H, W, dv] dtype; rows t >= n_replay[b] are written, the
 *              others are left as they were
 *   n_replay : [B] int32 in device memory; values are clamped to [0, W]
 *   dk, dv   : each one of 16, 32, 64, 128;  scale as for kda_chunk_fwd.
 * Element-aligned inputs; o must not overlap S or any input; S must not
 * overlap any input.
 */
kda_status_t kda_spec_replay_verify(const void *q, const void *k, const void *v, const void *g,
                                    const void *beta, float *S, void *o, const int *n_replay, int B,
                                    int H, int W, int dk, int dv, kda_dtype_t dtype, float scale,
                                    kda_stream_t stream);

/*
 * The replay loop with the KDA layer's gate edges folded in (Kimi K3 report,
 * section 5.4.2: one fused loop over replayed, bonus and draft tokens; the
 * gates of section 2.1.1, Eq. 5 and Eq. 6).  Same window, state and replay
 * semantics as kda_spec_replay_verify, except that
 *   z     : [B, H, W, dk] the Eq. 5 decay logits in place of g;
 *           g = g_min * Sigmoid(exp(A_log) * z) is formed on chip
 *   A_log : [H, dk] fp32;   g_min in [-5, 0)
 *   gate  : [B, H, W, dv] (dtype) the Eq. 6 output gate;  rms_weight : [H, dv] fp32;  eps >= 0
 *   y     : [B, H, W, dv] (dtype), written for the verified tokens (t >= n_replay[b]) only:
 *           y_t = Sigmoid(gate_t) * rms_weight * o_t / sqrt(mean(o_t^2) + eps)
 * dk = dv = 128 only (KDA_ERR_SHAPE otherwise).  The short convolution and
 * input normalisation of the report's loop need the layer's projection and
 * convolution weights and are not part of this call.  y, S must not overlap
 * any input (gate, A_log, rms_weight included).
 */
kda_status_t kda_spec_replay_verify_fused(const void *q, const void *k, const void *v, const void *z,
                                          const float *A_log, float g_min, const void *beta, float *S,
                                          const void *gate, const float *rms_weight, float eps, void *y,
                                          const int *n_replay, int B, int H, int W, int dk, int dv,
                                          kda_dtype_t dtype, float scale, kda_stream_t stream);

/*
 * Prefill without a caller-provided workspace, for callers that cannot
 * allocate device memory (e.g. a plugin inside a host framework that owns the
 * GPU memory pool and exposes no allocator, or a latency-critical path where
 * cudaMalloc's possible device synchronisation is not acceptable).  The
 * source report has no counterpart to this entry point: it is a packaging
 * variant of kda_chunk_fwd.
 *
 * Same arguments, layouts, alignment and aliasing rules and results as
 * kda_chunk_fwd, minus workspace/workspace_bytes: the scratch comes from one
 * fixed device array inside libkda of kda_noalloc_scratch_bytes() bytes
 * (32 MiB), held on every GPU that loads the library until the process exits.
 * Returns KDA_ERR_WORKSPACE if the call would need more scratch than that.
 * Set-up: the first call that needs scratch in a CUDA context (with its
 * device current) looks up the array's device address (cudaGetSymbolAddress)
 * and caches it for that context; make that first call before any stream
 * capture.  A context re-created after cudaDeviceReset repeats the lookup on
 * its first call.  Plans that need no scratch never touch the array.  No call
 * allocates or frees memory.  All calls share the array and nothing in it
 * needs to start at zero; calls that overlap on the GPU (different streams or
 * host threads) race on it, so serialise them.
 */
kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, const float *h0, void *o, float *h_T, int B,
                                   int H, int T, int dk, int dv, kda_dtype_t dtype, int chunk_size,
                                   float scale, kda_stream_t stream);

/* Size in bytes of the fixed scratch array kda_chunk_fwd_noalloc uses. */
size_t kda_noalloc_scratch_bytes(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status_t s);

/*
 * Synchronise `stream`, then read and clear the current device's status word
 * that kernels set when a bounded wait gives up (KDA_ERR_TIMEOUT) or a
 * device-side check fails (KDA_ERR_DEVICE).  Returns KDA_OK if nothing was
 * recorded, KDA_ERR_CUDA if synchronising failed.
 */
kda_status_t kda_get_device_status(kda_stream_t stream);

/*
 * Failure-detection testing aids (host-side fault injection; never needed in
 * production).  The tensor-core prefill kernel's cross-role waits are bounded:
 * a wait that does not complete within the limit aborts the CTA (no further
 * tensor-core work, every issued copy and MMA drained before its tensor memory
 * is released), records KDA_ERR_TIMEOUT in the device status word and returns,
 * so the context stays usable; the outputs of that call are then undefined.
 *
 * kda_debug_set_wait_limit: wall-time limit of those waits for calls enqueued
 *   afterwards, in nanoseconds (0 restores the default of 2 s).  Process-wide.
 * kda_debug_inject_stall: when on, prefill calls on the tensor-core path
 *   enqueued afterwards first wait on a barrier nothing ever arrives on, so
 *   the wait runs out after the limit above and the call aborts as described.
 *   Process-wide; turn it off again to resume normal operation.
 * Both return KDA_OK.
 */
kda_status_t kda_debug_set_wait_limit(unsigned long long ns);
kda_status_t kda_debug_inject_stall(int on);

/* Library version, e.g. 100 for 0.1.0. */
int kda_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LIBKDA_KDA_H_ */
