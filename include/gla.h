/*
 * gla.h -- C ABI of the B200 (sm_100a) chunkwise Gated Linear Attention library.
 *
 * The operation is the GLA layer of "Gated Linear Attention Transformers with
 * Hardware-Efficient Training" (Yang, Wang, Shen, Panda, Kim; arXiv:2312.06635),
 * section 4.1: for every (batch b, head h) independently, with a d_k x d_v
 * fp32 state S,
 *
 *     S_t = diag(alpha_t) S_{t-1} + k_t^T v_t ,     o_t = q_t S_t ,
 *
 * alpha_t in (0,1)^{d_k} a per-key-channel gate, given as log_alpha_t <= 0,
 * S_0 = h0 (zero when h0 == NULL), and o_t reading the state after step t's own
 * update.  gla_fwd evaluates it in the chunkwise-parallel form of sections 4.2
 * and 4.3 (chunk size `chunk`, secondary sub-chunks of `subchunk` tokens);
 * gla_bwd returns the gradients of a scalar loss L given dL/do and dL/dS_T, with
 * the gate gradient from the paper's closed form (section 4.3):
 * dlog b_t = q_t (.) dq_t - k_t (.) dk_t, dlog alpha_t = sum_{i>=t} dlog b_i.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout      contiguous row-major.  q, k, dq, dk: [B,H,T,d_k]; v, o, do, dv:
 *             [B,H,T,d_v]; log_alpha, dlog_alpha: [B,H,T,d_k] (GLA_GATE_VECTOR)
 *             or [B,H,T] (GLA_GATE_SCALAR, one gate shared by all key channels);
 *             states h0, h_final, dh0, dh_final: [B,H,d_k,d_v] fp32.
 * Dtypes      q, k, v, do and o, dq, dk, dv have the element type desc->dtype
 *             (bf16 or fp32); log_alpha, dlog_alpha and every state are fp32.
 * Ownership   the caller owns every buffer (device memory, e.g. from PyTorch).
 *             The library never allocates device memory: all scratch space comes
 *             from desc->workspace (size from gla_workspace_size).  Calls that
 *             share one workspace must not overlap on the GPU.
 * Execution   asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *             stream).  No implicit synchronisation.
 * Nullable    h0 (zero state), h_final / dh0 (not written), dh_final (zero);
 *             log_alpha / dlog_alpha must be NULL iff gate == GLA_GATE_NONE.
 * Errors      every argument is validated before anything is enqueued: a call
 *             that returns an error has launched nothing.  Errors found on the
 *             device (a bounded wait that ran out, a gate outside the supported
 *             range) are recorded in a status word inside the workspace and read
 *             by gla_poll_status.
 * Ragged T    any T >= 1.  The tail chunk is zero padded (q = k = v = 0,
 *             log_alpha = 0 beyond T), which leaves the state unchanged.
 */
#ifndef GLA_B200_GLA_H
#define GLA_B200_GLA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes (0 = success, negative = error). */
#define GLA_OK 0
#define GLA_ERR_INVALID_ARG (-1)        /* NULL where a buffer is required, bad enum, ... */
#define GLA_ERR_UNSUPPORTED_SHAPE (-2)  /* shape / chunk / dtype combination not built  */
#define GLA_ERR_MISALIGNED (-3)         /* a tensor pointer is not 16-byte aligned      */
#define GLA_ERR_WORKSPACE_TOO_SMALL (-4)
#define GLA_ERR_CUDA (-5)               /* a CUDA runtime / driver call failed          */
#define GLA_ERR_TIMEOUT (-6)            /* a device-side bounded wait ran out           */
#define GLA_ERR_GATE_RANGE (-7)         /* a gate too strong for the bf16 rescaling     */
#define GLA_ERR_NO_DEVICE (-8)          /* no sm_100 device for the bf16 tensor path    */

/* Element type of q, k, v, do and of o, dq, dk, dv. */
#define GLA_DTYPE_BF16 0
#define GLA_DTYPE_FP32 1

/* Gate parameterisation (section 4.1 and the gate ablation of section 5):
 * VECTOR  G_t = alpha_t^T 1 with alpha_t per key channel,
 * SCALAR  G_t = gamma_t 1^T 1 (one gate per token and head),
 * NONE    alpha == 1 (ungated linear attention, section 2.1). */
#define GLA_GATE_VECTOR 0
#define GLA_GATE_SCALAR 1
#define GLA_GATE_NONE 2

/* Forward variant (section 3.3, Figure 1):
 * FUSED         the state is carried on chip across the chunks of a segment;
 *               only the P segment-start states are materialised (AUTO picks P).
 * MATERIALIZED  every chunk-level state S[n] is written to the workspace in fp32
 *               first, then all chunk outputs are computed in parallel
 *               ("sequence-level chunk parallelism").
 * AUTO          FUSED with the segment count chosen to fill the GPU. */
#define GLA_VARIANT_AUTO 0
#define GLA_VARIANT_FUSED 1
#define GLA_VARIANT_MATERIALIZED 2

/* Flags (desc->flags).  Both are ignored by the fp32 path, which recomputes.
 *
 * GLA_FLAG_REUSE_PREP (gla_bwd): desc->workspace already holds the per-chunk
 * prep outputs (gate-rescaled q and k, intra-chunk scores, chunk decays) that a
 * gla_fwd call wrote into this same workspace for the same q, k, log_alpha,
 * shape, gate, segments and chunk, and nothing has written to the workspace
 * since.  The backward reads them instead of recomputing them.
 *
 * GLA_FLAG_SAVE_STATES (gla_fwd and gla_bwd): on gla_fwd, the forward also
 * stores every chunk-entry state S[n-1] in bf16 into the workspace (the bf16
 * copy the inter-chunk output term already uses); on gla_bwd, the backward
 * reads those states instead of recomputing them with a second forward walk.
 * The backward's chunk states are bf16 either way, so results are unchanged.
 * The gla_bwd call must follow a gla_fwd call with this flag on the same
 * inputs (and h0), descriptor and workspace, with nothing written to the
 * workspace in between; pass GLA_FLAG_REUSE_PREP with it to reuse the prep
 * outputs too.
 *
 * With either flag the workspace must be sized for the backward
 * (gla_workspace_size(desc, chunk, 1)) on both calls, the gla_fwd call
 * included; that size is at least the forward's.
 *
 * GLA_FLAG_REUSE_PREP also applies to gla_fwd, gla_fwd_state and gla_bwd_state:
 * the prep outputs may come from any earlier call of these four on the same
 * inputs and workspace (the sequence-parallel step runs prep once).
 *
 * GLA_FLAG_REUSE_SEGMENTS (gla_fwd, gla_bwd): the workspace holds the zero-state
 * contributions of every segment written by gla_fwd_state (for gla_fwd) or
 * gla_bwd_state (for gla_bwd) on the same inputs, descriptor and flags, and
 * nothing but those calls (and a gla_fwd / gla_bwd with this flag) has written to
 * the workspace since; the walks' pre-passes are skipped.  Ignored by the fp32
 * path and by the materialized variant. */
#define GLA_FLAG_REUSE_PREP 1
#define GLA_FLAG_SAVE_STATES 2
#define GLA_FLAG_REUSE_SEGMENTS 4

typedef struct gla_desc {
  int B, H, T;          /* batch, heads, tokens (T >= 1)                                   */
  int dk, dv;           /* key / value head dimensions                                     */
  int dtype;            /* GLA_DTYPE_*                                                     */
  int gate;             /* GLA_GATE_*                                                      */
  int subchunk;         /* secondary chunk size; 0 = 16                                    */
  int variant;          /* GLA_VARIANT_* (forward only)                                    */
  int segments;         /* segments per sequence for the FUSED variant; 0 = automatic      */
  int flags;            /* GLA_FLAG_* (0 = none)                                           */
  void *workspace;      /* device scratch owned by the caller, 256-byte aligned            */
  size_t workspace_bytes;
} gla_desc;

/* Bytes of workspace gla_fwd (for_bwd == 0) or gla_bwd (for_bwd != 0) needs for
 * this descriptor and chunk size.  Returns 0 for an invalid descriptor (call
 * gla_check to learn why).  Host-only; enqueues nothing. */
size_t gla_workspace_size(const gla_desc *desc, int chunk, int for_bwd);

/* Validate a descriptor + chunk without any pointer (GLA_OK or an error code).
 * Host-only; enqueues nothing. */
int gla_check(const gla_desc *desc, int chunk);

/* Forward (sections 4.2-4.3; Algorithms 3 and 5 of Appendix B by title).
 *   q, k [B,H,T,d_k], v [B,H,T,d_v], log_alpha (see layout), h0 [B,H,d_k,d_v] or NULL
 *   o [B,H,T,d_v] (written), h_final [B,H,d_k,d_v] or NULL (written: S_T)
 * chunk: C in {16, 32, 64, 128}.  bf16 inputs run on the tensor-core path when
 * d_k is 128 or 256, d_v a multiple of 64, C = 64 and the sub-chunk 16; every
 * other shape, and fp32 inputs, run on the CUDA-core path (fp32 arithmetic,
 * pairwise log-space intra-chunk terms; the workspace sizes follow the path).
 * Returns GLA_OK or an error code; on error nothing was enqueued. */
int gla_fwd(const gla_desc *desc, const void *q, const void *k, const void *v,
            const float *log_alpha, const float *h0, void *o, float *h_final, int chunk,
            void *stream);

/* Backward (Algorithms 4 and 6 of Appendix B by title; closed-form gate
 * gradient of section 4.3).  The chunk states are recomputed by a forward walk
 * of the backward itself, unless desc->flags has GLA_FLAG_SAVE_STATES: then they
 * are read from the workspace, where the preceding gla_fwd call with that flag
 * stored them.  The loss gradient enters through do [B,H,T,d_v] and dh_final
 * (dL/dS_T, NULL = 0).  Outputs: dq, dk [B,H,T,d_k], dv [B,H,T,d_v],
 * dlog_alpha (gate layout; NULL iff gate == NONE), dh0 (dL/dh0; NULL = not
 * written).  With a SCALAR gate dlog_alpha_t is the sum over key channels. */
int gla_bwd(const gla_desc *desc, const void *q, const void *k, const void *v,
            const float *log_alpha, const float *h0, const void *do_, const float *dh_final,
            void *dq, void *dk, void *dv, float *dlog_alpha, float *dh0, int chunk,
            void *stream);

/* ---- recurrent decode step ---------------------------------------------------
 * One token per (batch, head) in the recurrent form of section 4.1 (the form the
 * paper uses for generation), on the state the caller carries between calls:
 *     S <- diag(alpha) S + k^T v ,     o = q S   (o reads the updated state).
 *   q, k [B,H,d_k]; v, o [B,H,d_v] (element type desc->dtype); log_alpha
 *   [B,H,d_k] (GLA_GATE_VECTOR) or [B,H] (GLA_GATE_SCALAR) or NULL
 *   (GLA_GATE_NONE), fp32; state [B,H,d_k,d_v] fp32, read and overwritten in
 *   place (it must not alias q, k, v, log_alpha or o).
 * desc->T must be 1; d_k <= 4096 and d_v a multiple of 4.  desc->subchunk,
 * variant, segments, flags and the workspace are ignored (no scratch memory).
 * Every argument is validated before anything is enqueued; the call is
 * asynchronous on `stream` and bound by HBM bandwidth on the state.
 * Returns GLA_OK or an error code; on error nothing was enqueued. */
int gla_decode_step(const gla_desc *desc, const void *q, const void *k, const void *v,
                    const float *log_alpha, float *state, void *o, void *stream);

/* ---- layer epilogue -------------------------------------------------------------
 * The step after the recurrence in the GLA layer of the paper: each head's output
 * is normalised by a LayerNorm over its d_v channels and multiplied elementwise
 * by the Swish output gate r (Swish(x) = x sigmoid(x)) before the output
 * projection (not part of this library):
 *     y = (w (.) (o - mean(o)) / sqrt(var(o) + eps) + b) (.) r sigmoid(r)
 * mean and biased variance over the d_v channels of one (batch, head, token).
 *   o, r, y, dy, do, dr: [B,H,T,d_v], element type desc->dtype (r is the gate's
 *   pre-activation, given in o's layout); w, b, dw, db: [d_v] fp32, one weight and
 *   bias shared by every head (w NULL = ones, b NULL = zeros; dw / db NULL = not
 *   computed).  d_v a multiple of 8 and <= 1024; 0 < eps < 1 (the paper's layer
 *   uses the usual 1e-5).  desc->dk, subchunk, variant, segments and flags are
 *   ignored.
 * gla_epilogue_bwd returns do, dr and, when asked, dw and db; the latter are
 * summed over all rows in a fixed order (deterministic on a given GPU model)
 * through per-CTA partial sums in desc->workspace.
 *   desc->workspace: 256-byte aligned, caller-owned; at least
 *   gla_epilogue_workspace_size(desc) bytes for a backward that returns dw or db,
 *   at least 256 bytes otherwise.  Its first 256 bytes hold the status word that
 *   every call clears and that gla_poll_status(desc, stream) reads (a device-side
 *   bounded wait that ran out: GLA_ERR_TIMEOUT).  Calls that share a workspace
 *   must not overlap on the GPU.
 * Both calls validate every argument before enqueuing anything, run
 * asynchronously on `stream` and are bound by HBM bandwidth. */
size_t gla_epilogue_workspace_size(const gla_desc *desc);
int gla_epilogue_fwd(const gla_desc *desc, const void *o, const void *r, const float *w, const float *b,
                     float eps, void *y, void *stream);
int gla_epilogue_bwd(const gla_desc *desc, const void *o, const void *r, const float *w, const float *b,
                     float eps, const void *dy, void *do_, void *dr, float *dw, float *db, void *stream);

/* Forward with the layer epilogue fused into its output store ("Gated Linear
 * Attention Transformers with Hardware-Efficient Training", the GLA layer of
 * section 4.4: head-wise LayerNorm, then the Swish output gate).  Computes what
 * gla_fwd followed by gla_epilogue_fwd computes: o and h_final exactly as
 * gla_fwd, and y = (w (.) (o - mean(o)) / sqrt(var(o) + eps) + b) (.) r sigmoid(r)
 * over the d_v channels of every (batch, head, token).
 *   q, k, v, log_alpha, h0, o, h_final, chunk: as gla_fwd (o is still written:
 *   the epilogue's backward reads it);  r, y [B,H,T,d_v] of desc->dtype;
 *   w, b [d_v] fp32 or NULL (ones / zeros);  0 < eps < 1.
 *   desc->workspace: as gla_fwd (gla_workspace_size(desc, chunk, 0), or the
 *   backward size under GLA_FLAG_SAVE_STATES); GLA_FLAG_REUSE_PREP and
 *   GLA_FLAG_SAVE_STATES as for gla_fwd; GLA_FLAG_REUSE_SEGMENTS is rejected
 *   (GLA_ERR_INVALID_ARG: the fused walk may split the sequence into fewer segments).
 * On the bf16 tensor-core path with d_v a multiple of 128 up to 512 and the fused
 * variant, the statistics come from the fp32 output before its rounding to bf16:
 * the output walk's CTAs of one head and segment form a thread-block cluster and
 * exchange every token's per-tile mean and sum of squared deviations through
 * distributed shared memory.  Any other valid descriptor runs gla_fwd and then the
 * epilogue as a second pass over the bf16 o (d_v a multiple of 8, at most 1024).
 * Returns GLA_OK or an error code; on error nothing was enqueued.  The status word
 * (gla_poll_status) reports device-side errors as for gla_fwd. */
int gla_fwd_epilogue(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                     const float *h0, const void *r, const float *w, const float *b, float eps, void *o, void *y,
                     float *h_final, int chunk, void *stream);

/* ---- general gate (value-side gate beta) -------------------------------------------
 * "Gated Linear Attention Transformers with Hardware-Efficient Training",
 * appendix C: the gate G_t = alpha_t^T beta_t, an outer product of a key-side
 * gate alpha_t (per desc->gate, given as log_alpha exactly as for gla_fwd) and a
 * value-side gate beta_t in (0,1]^{d_v}:
 *     S_t = diag(alpha_t) S_{t-1} diag(beta_t) + k_t^T v_t ,   o_t = q_t S_t .
 *   log_beta / dlog_beta: [B,H,T,dv] fp32, required (log_beta = 0 gives gla_fwd's
 *   result).  Every other argument as for gla_fwd / gla_bwd.  dlog_beta is the
 *   gradient of the loss with respect to log_beta.
 * Runs on the CUDA-core path for either dtype (fp32 arithmetic, every chunk state
 * materialised, intra-chunk pairs in log space, so any gate strength is stable).
 * Workspace: gla_general_workspace_size(desc, chunk, for_bwd) bytes, 256-byte
 * aligned; desc->flags, variant and segments are ignored.  Errors as for gla_fwd. */
size_t gla_general_workspace_size(const gla_desc *desc, int chunk, int for_bwd);
int gla_fwd_general(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *log_beta, const float *h0, void *o, float *h_final, int chunk, void *stream);
int gla_bwd_general(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *log_beta, const float *h0, const void *do_, const float *dh_final, void *dq,
                    void *dk, void *dv, float *dlog_alpha, float *dlog_beta, float *dh0, int chunk, void *stream);

/* ---- sequence (context) parallelism ---------------------------------------------
 * "Gated Linear Attention Transformers with Hardware-Efficient Training",
 * sections 3.3 and 4.2: the chunk-level recurrence S_n = diag(gamma_n) S_{n-1} + dS_n
 * composes affine maps, so a sequence split into consecutive pieces (one per GPU,
 * piece r holding tokens [t_r, t_{r+1}) of every (batch, head)) needs, per piece,
 * one summary: its gate product gamma = prod_t alpha_t (per key channel) and the
 * state it produces.  One exchange of the summaries (an all-gather), a fold, and
 * every piece reruns gla_fwd / gla_bwd with its incoming state.  Each call below
 * describes one piece: desc->T is the piece's token count, the tensors hold only
 * the piece's tokens.  Tensor-core path only (fp32 descriptors, and bf16 shapes that
 * path does not take: GLA_ERR_UNSUPPORTED_SHAPE).
 *
 * gla_fwd_state: delta [B,H,dk,dv] fp32 = the state after the piece's tokens
 *   starting from h0 (NULL = zero), i.e. the h_final of gla_fwd, without computing
 *   o; gamma [B,H,dk] fp32 = prod over the piece's tokens of alpha_t (exp of the
 *   summed log_alpha; all ones for GLA_GATE_NONE, the scalar gate broadcast over
 *   dk).  Workspace: gla_workspace_size(desc, chunk, 0), or
 *   gla_workspace_size(desc, chunk, 1) when desc->flags has GLA_FLAG_SAVE_STATES
 *   (the summary then uses the backward's layout, so that a following gla_fwd
 *   with that flag finds its segment contributions); a smaller workspace is
 *   rejected with GLA_ERR_WORKSPACE_TOO_SMALL.
 * gla_bwd_state: ddelta [B,H,dk,dv] fp32 = the state adjoint before the piece's
 *   first token given dh_final (NULL = zero) after its last, i.e. the dh0 of
 *   gla_bwd, without the token gradients; gamma (NULL = not written) as above.
 *   Workspace: gla_workspace_size(desc, chunk, 1).
 * gla_state_scan: the fold over gathered summaries.  gammas [nseg][B,H,dk],
 *   deltas [nseg][B,H,dk,dv] fp32 (piece-major, as an all-gather stacks them);
 *   S = init (NULL = zero), then S <- diag(gammas[s]) S + deltas[s] for
 *   s = 0 .. seg-1 (reverse = 0: the state entering piece seg) or for
 *   s = nseg-1 down to seg+1 (reverse = 1: the adjoint leaving piece seg); out = S.
 *   Uses B, H, dk, dv of desc (dv a multiple of 4); no workspace.
 * All three validate every argument before enqueuing anything and run
 * asynchronously on `stream`; the first two report device errors through the
 * status word like gla_fwd. */
int gla_fwd_state(const gla_desc *desc, const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *h0, float *delta, float *gamma, int chunk, void *stream);
int gla_bwd_state(const gla_desc *desc, const void *q, const void *k, const float *log_alpha, const void *do_,
                  const float *dh_final, float *ddelta, float *gamma, int chunk, void *stream);
int gla_state_scan(const gla_desc *desc, int nseg, int seg, int reverse, const float *gammas, const float *deltas,
                   const float *init, float *out, void *stream);

/* ---- forward without a workspace ---------------------------------------------
 * No counterpart in the paper: this entry point exists for callers that cannot
 * allocate device memory -- a program whose device memory is all owned by
 * another allocator (a fixed arena reserved up front), or a plain C caller with
 * no device-memory management of its own -- and so cannot pass a workspace.
 * It computes exactly what gla_fwd computes (same arguments; desc->workspace
 * and desc->workspace_bytes are ignored), using as scratch a fixed array of
 * GLA_NOALLOC_SCRATCH_BYTES in the library's own device memory, which every GPU
 * that loads the library holds until the process exits.  It never allocates.
 *   - Problems whose forward workspace (gla_workspace_size(desc, chunk, 0))
 *     exceeds GLA_NOALLOC_SCRATCH_BYTES are rejected with
 *     GLA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued; other argument
 *     errors are reported as by gla_fwd.
 *   - All calls share the one array.  Calls that overlap on the GPU (on other
 *     streams or from other host threads) race on it; the caller must
 *     serialise them.  Each call clears the status word it needs zeroed.
 *   - The first call on a device looks up the array's address for that device
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - desc->flags may hold GLA_FLAG_SAVE_STATES (the workspace size is then
 *     the backward's), but not GLA_FLAG_REUSE_PREP or GLA_FLAG_REUSE_SEGMENTS:
 *     nothing leaves intermediates in this scratch for a later call to reuse,
 *     so those flags are rejected with GLA_ERR_INVALID_ARG.
 *   - Errors found on the device (a bounded wait that ran out, a gate beyond
 *     the bf16 range) are recorded in a status word at the start of the
 *     scratch, which gla_poll_status_noalloc reads and clears.
 * gla_poll_status_noalloc: like gla_poll_status, for that status word on the
 * current device: synchronises `stream`, reads and clears the word, and returns
 * GLA_OK, GLA_ERR_TIMEOUT or GLA_ERR_GATE_RANGE (GLA_ERR_CUDA if the stream
 * failed).  Its first call on a device resolves the scratch address as above. */
#define GLA_NOALLOC_SCRATCH_BYTES (64u << 20)
int gla_fwd_noalloc(const gla_desc *desc, const void *q, const void *k, const void *v,
                    const float *log_alpha, const float *h0, void *o, float *h_final, int chunk,
                    void *stream);
int gla_poll_status_noalloc(void *stream);

/* Synchronise `stream`, then read and clear the device status word kept in
 * desc->workspace.  Returns GLA_OK, GLA_ERR_TIMEOUT or GLA_ERR_GATE_RANGE (or
 * GLA_ERR_CUDA if the stream itself failed). */
int gla_poll_status(const gla_desc *desc, void *stream);

/* Human-readable text for a return code (static storage). */
const char *gla_status_string(int code);

/* ---- instrumentation (benchmarking only) ------------------------------------
 * When enabled, every kernel launch of gla_fwd / gla_bwd is bracketed by two
 * CUDA events recorded on the launch stream.  gla_timing_collect synchronises
 * those events and returns, for up to `max` launches since the last collect,
 * the kernel id and its duration in milliseconds; it returns the count.
 * Events are created by the CUDA runtime; no device memory is allocated. */
int gla_timing_enable(int on);
int gla_timing_collect(int max, int *kernel_ids, float *ms);
const char *gla_kernel_name(int kernel_id);

/* Self-test of the device-side bounded waits (no counterpart in the paper).
 * Enqueues one kernel whose single thread waits, with the same bounded wait
 * every kernel of this library uses, on an mbarrier that nothing completes; the
 * wait gives up after limit_us microseconds (1 .. 1e6) and sets the timeout bit
 * in the 4-byte device word *status_word, which gla_poll_status reads when it is
 * the first word of desc->workspace.  It faults nothing and leaves the context
 * usable; it exists so that the timeout path can be tested. */
int gla_selftest_timeout(void *status_word, unsigned limit_us, void *stream);

/* Text of the most recent CUDA runtime error behind a GLA_ERR_CUDA return of
 * any call in this process ("no error" if there was none; static storage).
 * Host-only. */
const char *gla_last_cuda_error(void);

/* Build information: a static string naming the kernels and architecture. */
const char *gla_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* GLA_B200_GLA_H */
