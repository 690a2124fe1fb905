/*
 * mtla.h — C ABI of the MTLA hot-path library (libmtla.so), sm_100a.
 *
 * Multi-head Temporal Latent Attention (Deng & Woodland, NeurIPS 2025) keeps a
 * KV cache compressed twice: in feature width (a latent c of width r plus a
 * decoupled-RoPE key of width d_R) and in time (every s adjacent steps are
 * merged by a sigmoid-gated hyper-network).  This library runs the inference
 * hot path (merge/append + absorbed decode attention), the parallel
 * training/prefill forward under the stride-aware causal mask, and the
 * training shortcut's backward pass.
 *
 * Sources (page title, section):
 *   [merge]   MTLA paper notes, "Key designs: hyper-network temporal merging":
 *             w_i = Sigmoid(Linear(c_i) ⊙ Linear(pe_j)), c_hat_j = sum_i w_i ⊙ c_i,
 *             the cache holds ceil(T/s) rows.
 *   [mask]    MTLA paper notes, "Key designs: stride-aware causal mask": query m
 *             sees column n of C_hat' iff n == m, or n < m and n mod s == 0.
 *   [rope]    MTLA paper notes, "Key designs: decoupled RoPE with temporal
 *             compression": Y = softmax((X W_Q W_K^T C_hat^T + Q^R K_hat^R^T)
 *             / sqrt(d_h)) C_hat (W_V W_O).
 *   [fig2]    arXiv 2505.13544 abstract page, Figure 2: (a) incremental
 *             inference attends a temporary c_hat'_j at steps 1, 3, 5 (s = 2);
 *             (c) training with the stride-aware mask.
 *   [train]   MTLA paper notes, "Key designs: decoupled RoPE with temporal
 *             compression": training may take the uncompressed K^R in place
 *             of the merged K_hat^R (the training shortcut).
 *
 * Conventions for every call
 *   - Time is 1-indexed as on the pages: token t of a sequence belongs to group
 *     j(t) = ceil(t/s); token t opens a new cache row iff (t-1) mod s == 0 and is
 *     added in place to the tail row otherwise.
 *   - A cache row is [c_hat (r) | k_hat^R (d_R)], D = r + d_R elements, stored
 *     in the cache dtype; consecutive rows are row_stride elements apart.
 *     Sequence b owns rows [seq_offset[b], seq_offset[b] + seq_capacity[b]) of a
 *     buffer of cache_rows rows ("paged contiguous" cache).
 *   - Softmax scale is 1/sqrt(d_h) ([rope]); values are the latent part only.
 *   - All pointers except `dims`, `merge` and the host outputs of
 *     mtla_debug_stride_mask are DEVICE pointers.  The caller owns every
 *     buffer; the library allocates no memory and never synchronises.  Every
 *     call is asynchronous on `stream` (a cudaStream_t, NULL = legacy stream).
 *   - Argument errors are reported synchronously, before any launch, as the
 *     returned status.  Conditions only the device can see are OR-ed into
 *     *dev_err (MTLA_DEVERR_* bits); the kernels then skip the offending work
 *     and never trap.  dev_err is never cleared by the library.
 *   - bf16 tensors must be 16-byte aligned and row strides multiples of 8
 *     elements; fp32 tensors 16-byte aligned.
 */
#ifndef MTLA_H
#define MTLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MTLA_OK = 0,
  MTLA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or stride */
  MTLA_ERR_UNSUPPORTED = 2,   /* dims or dtype this build has no kernel for    */
  MTLA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required    */
  MTLA_ERR_CUDA = 4           /* a CUDA runtime/driver call failed             */
} mtla_status;

typedef enum { MTLA_F32 = 0, MTLA_BF16 = 1 } mtla_dtype;

/* Problem dimensions: H heads of width d_h (sets the 1/sqrt(d_h) scale),
 * latent width r, RoPE width d_R, temporal stride s >= 1, cache dtype. */
typedef struct {
  int32_t H, d_h, r, d_R, s;
  int32_t dtype; /* mtla_dtype */
} mtla_dims;

/* Hyper-network merge inputs for ONE new token per sequence ([merge]).
 * Linear(c_t) = c_t W_c + b_c maps width r to D so that one gate covers
 * [c_t ; k^R_t]; Linear(pe_j) is precomputed by the caller as row j-1 of P. */
typedef struct {
  const void *c_new;   /* [B, r]    cache dtype: the new latents c_t            */
  const void *kR_new;  /* [B, d_R]  cache dtype: the new RoPE keys, rotated      */
  const float *W_c;    /* [r, D]    row-major                                    */
  const float *b_c;    /* [D]                                                    */
  const float *P;      /* [J_max, D] row j-1 = Linear(pe_j) for group j          */
  int32_t J_max;       /* rows of P; a token with j(t) > J_max sets PE_RANGE     */
} mtla_merge_args;

/* device error bits (OR-ed into *dev_err) */
#define MTLA_DEVERR_PE_RANGE 1   /* j(t) > J_max: merge skipped                   */
#define MTLA_DEVERR_CAPACITY 2   /* ceil(t/s) > seq_capacity, or the sequence's   */
                                 /* rows run past cache_rows: work clamped        */
#define MTLA_DEVERR_EMPTY    4   /* attention over an empty cache (t == 0)        */
#define MTLA_DEVERR_TIMEOUT  8   /* an internal bounded wait gave up              */

/*
 * mtla_merge_append — fold one new token per sequence into the cache ([merge],
 * [fig2](a)).  For each b: t = t_processed[b] + 1, j = ceil(t/s),
 * w = sigmoid((c_t W_c + b_c) ⊙ P[j-1]); the row j-1 of sequence b becomes
 * w ⊙ [c_t ; k^R_t] if (t-1) mod s == 0, else row += w ⊙ [c_t ; k^R_t]
 * (fp32 arithmetic, stored in the cache dtype).  Then t_processed[b] = t and,
 * if cache_len != NULL, cache_len[b] = j.
 *   cache           [cache_rows, row_stride] cache dtype, updated in place
 *   seq_offset, seq_capacity [B] int64, t_processed [B] int32 (in/out),
 *   cache_len [B] int32 (out, nullable), dev_err int32 (in/out).
 */
mtla_status mtla_merge_append(const mtla_dims *dims, int32_t B, const mtla_merge_args *merge,
                              void *cache, int64_t cache_rows, int64_t row_stride,
                              const int64_t *seq_offset, const int64_t *seq_capacity,
                              int32_t *t_processed, int32_t *cache_len, int32_t *dev_err,
                              void *stream);

/*
 * mtla_decode_attn — one incremental decode step ([rope], [fig2](a)).
 * If merge != NULL the new token is first merged exactly as mtla_merge_append
 * does, before the attention reads the tail row, and t_processed advances by
 * one; if merge == NULL the cache is read as it stands (t_processed
 * unchanged).  Then for every sequence b and head h, over the L = ceil(t/s)
 * cached rows (the partial tail included):
 *   score_j = (q_abs[b,h] · c_hat_j + q_rope[b,h] · k_hat^R_j) / sqrt(d_h),
 *   out[b,h,:] = sum_j softmax(score)_j c_hat_j,  lse[b,h] = ln sum_j e^score_j.
 *   q_abs [B, H, r], q_rope [B, H, d_R]   cache dtype
 *   out   [B, H, r] fp32;  lse [B, H] fp32 (nullable)
 *   workspace: mtla_workspace_bytes(dims, B, MTLA_WS_DECODE) bytes of device
 *              memory owned by the caller; it needs no initialisation (a call
 *              reads only what it wrote itself), and one workspace serves calls
 *              that run one after another on a stream (not calls that overlap).
 * Kernels: bf16 with (H, r, d_R) = (8, 256, 32) and B <= 1024 runs the
 * split-L tensor-core path as three launches on `stream`, chained by
 * programmatic dependent launch: the merge (gate, append or in-place update of
 * the tail row; only if merge != NULL), the attention over row shares, and the
 * split combine with the length update (workspace required).  Any other
 * supported dims run a one-block-per-sequence kernel (one launch, merge
 * included; workspace unused, may be NULL).
 * Supported dims everywhere: H <= 16, r <= 512, r + d_R <= 576, r and d_R
 * multiples of 8 (bf16) or 4 (fp32); otherwise MTLA_ERR_UNSUPPORTED.
 */
mtla_status mtla_decode_attn(const mtla_dims *dims, int32_t B,
                             const void *q_abs, const void *q_rope,
                             const mtla_merge_args *merge,
                             void *cache, int64_t cache_rows, int64_t row_stride,
                             const int64_t *seq_offset, const int64_t *seq_capacity,
                             int32_t *t_processed, int32_t *cache_len,
                             float *out, float *lse,
                             void *workspace, size_t workspace_bytes,
                             int32_t *dev_err, void *stream);

/*
 * mtla_decode_attn_multi — n new tokens per sequence in one call (speculative
 * or beam decode), 1 <= n <= MTLA_MAX_NEW_TOKENS ([merge], [fig2](a)).
 * Tokens t = t_processed[b] + 1 .. t_processed[b] + n of sequence b are merged
 * in order exactly as n consecutive mtla_decode_attn calls merge them (the
 * stored row is rounded to the cache dtype after every token), and query i
 * attends the cache as it stands after token i: rows 1 .. ceil(t_i / s), the
 * last one the (possibly partial) row that token i leaves.  Then
 * t_processed[b] += n and cache_len[b] = ceil(t_processed[b] / s).
 *   q_abs [B, n, H, r], q_rope [B, n, H, d_R]   cache dtype
 *   merge (required): c_new [B, n, r], kR_new [B, n, d_R]; W_c, b_c, P, J_max
 *   out [B, n, H, r] fp32;  lse [B, n, H] fp32 (nullable)
 *   workspace: mtla_decode_multi_workspace_bytes(dims, B, n) bytes; needs no
 *   initialisation.
 * A sequence whose n tokens do not fit its capacity (or P table) merges none
 * of them (MTLA_DEVERR_CAPACITY / _PE_RANGE) and its queries attend the cache
 * as it stands.  The attention runs over B n per-query sequences that share
 * their sequence's rows: on the split-L tensor-core path when B n <= 1024
 * (bf16, (H, r, d_R) = (8, 256, 32)), else one block per query.
 */
#define MTLA_MAX_NEW_TOKENS 16

mtla_status mtla_decode_attn_multi(const mtla_dims *dims, int32_t B, int32_t n,
                                   const void *q_abs, const void *q_rope,
                                   const mtla_merge_args *merge,
                                   void *cache, int64_t cache_rows, int64_t row_stride,
                                   const int64_t *seq_offset, const int64_t *seq_capacity,
                                   int32_t *t_processed, int32_t *cache_len,
                                   float *out, float *lse,
                                   void *workspace, size_t workspace_bytes,
                                   int32_t *dev_err, void *stream);

/* Workspace bytes of mtla_decode_attn_multi (0 on unsupported arguments).
 * Queries the current device. */
size_t mtla_decode_multi_workspace_bytes(const mtla_dims *dims, int32_t B, int32_t n);

/*
 * mtla_decode_attn_static — mtla_decode_attn with its scratch in a static
 * device array of this library instead of a caller-provided workspace.  The
 * MTLA paper has no counterpart: this is a library convenience, and it
 * computes exactly what mtla_decode_attn computes, through the same kernels.
 *
 * For callers that cannot allocate device memory around a decode step: for
 * example an engine that has given all free memory to its cache pages, or
 * plain C host code with no device allocator.  Nothing in the call
 * allocates.  The scratch is MTLA_DECODE_STATIC_SCRATCH_BYTES per device,
 * reserved by the driver when the library's device code is loaded.
 *
 * Arguments, layouts and device-side errors are those of mtla_decode_attn
 * without workspace / workspace_bytes.
 * Set-up: the first call on a device (with that device current) looks up the
 *   array's address and clears it on `stream`; make it before any stream
 *   capture.  The driver reserves the array when it loads this library's
 *   device code into the context: under lazy module loading (the CUDA
 *   default) that is this first call.  The address is kept for the life of
 *   the process: do not use this entry point on a device after
 *   cudaDeviceReset.
 * Limit: a call whose workspace (mtla_workspace_bytes) would exceed
 *   MTLA_DECODE_STATIC_SCRATCH_BYTES returns MTLA_ERR_WORKSPACE and runs
 *   nothing.  24 MiB covers every B <= 1024 on a 148-SM B200 (about 5.5 MB
 *   at B = 1024).
 * Sharing: all calls on a device use the one scratch, so calls that overlap
 *   (other streams, unordered threads) race; issue them one after another on
 *   one stream.
 */
#define MTLA_DECODE_STATIC_SCRATCH_BYTES (24u << 20)

mtla_status mtla_decode_attn_static(const mtla_dims *dims, int32_t B,
                                    const void *q_abs, const void *q_rope,
                                    const mtla_merge_args *merge,
                                    void *cache, int64_t cache_rows, int64_t row_stride,
                                    const int64_t *seq_offset, const int64_t *seq_capacity,
                                    int32_t *t_processed, int32_t *cache_len,
                                    float *out, float *lse,
                                    int32_t *dev_err, void *stream);

/*
 * mtla_prefill_masked_attn — the parallel (training / prefill) forward of B
 * sequences of T tokens, t = 1..T ([mask], [fig2](c)).
 *   1. c_partial[b, n] = C_hat'_n = sum_{i=(j(n)-1)s+1}^{n} w_i ⊙ [c_i ; k^R_i],
 *      w_i = sigmoid((c_i W_c + b_c) ⊙ P[j(i)-1])  (the running merge);
 *   2. out[b, m, h] = sum_{n visible} softmax(score)_n c_hat'_n with the
 *      stride-aware mask (n == m, or n < m and n mod s == 0) and the score of
 *      mtla_decode_attn against row n of C_hat'.
 *   3. if cache_out != NULL: cache_out[b, g-1] = C_hat'_{min(g s, T)},
 *      g = 1..ceil(T/s) — the decode cache after the prompt.
 *   If out == NULL only steps 1 and 3 run (building a cache from a prompt);
 *   q_abs and q_rope may then be NULL.
 *   q_abs [B, T, H, r], q_rope [B, T, H, d_R], c [B, T, r], kR [B, T, d_R]
 *   (cache dtype, contiguous); W_c, b_c, P, J_max as in mtla_merge_args
 *   (J_max >= ceil(T/s)); c_partial [B, T, D], cache_out [B, ceil(T/s), D],
 *   out [B, T, H, r] all cache dtype, contiguous, written by the call.
 * Kernels: bf16 with (H, r, d_R) = (8, 256, 32) runs the tcgen05/TMEM
 * tensor-core kernel; other supported dims run a SIMT kernel.  The running
 * merge of bf16 prompts with r = 256, d_R = 32, s <= 32 runs on the tensor
 * cores with W_c rounded to bf16 (fp32 sums; an error near the bf16 rounding
 * of C_hat' itself); other dims and strides keep fp32 W_c.  Every pointer
 * must be 16-byte aligned (MTLA_ERR_INVALID_ARG otherwise).
 */
mtla_status mtla_prefill_masked_attn(const mtla_dims *dims, int32_t B, int32_t T,
                                     const void *q_abs, const void *q_rope,
                                     const void *c, const void *kR,
                                     const float *W_c, const float *b_c,
                                     const float *P, int32_t J_max,
                                     void *c_partial, void *cache_out, void *out,
                                     int32_t *dev_err, void *stream);

/*
 * mtla_project_in — the layer's input maps for one new token per sequence,
 * with the key map absorbed into the query ([rope]; arXiv 2505.13544 abstract
 * page, Figure 1: the latent-to-KV maps are absorbed into the query and
 * output linear layers by associativity).  For every token b:
 *   [q_abs | q_rope | c_new | kR_new] = x[b] W_in^T, then RoPE at position
 *   pos[b] on q_rope (each head) and kR_new: channel pair (2k, 2k+1) rotated
 *   by pos[b] * 10000^(-2k/d_R).
 *   x      [B, d]       cache dtype (bf16: d a multiple of 64; fp32: of 4)
 *   W_in   [N_in, d]    cache dtype, row-major (one row per output feature),
 *          N_in = H (r + d_R) + r + d_R rows in this order:
 *            H r rows   row h r + i = column i of W_Q^h W_K^h^T (the absorbed
 *                       query of head h: d_h columns of W_Q^h times the
 *                       transposed key map of that head)
 *            H d_R rows row H r + h d_R + k = column k of W_QR^h
 *            r rows     the latent map W_down (c_t = x W_down)
 *            d_R rows   the RoPE key map W_KR
 *   pos    [B] int32    0-based position of each token (t - 1)
 *   q_abs [B, H, r], q_rope [B, H, d_R], c_new [B, r], kR_new [B, d_R]:
 *          written in the cache dtype, ready for mtla_decode_attn.
 *   workspace: mtla_project_workspace_bytes(dims, B, d, MTLA_PROJ_IN) bytes
 *          (fp32 partial sums; no initialisation needed).
 * bf16 runs a split-K tensor-core GEMM (tcgen05, batches of up to 256 tokens
 * per launch) and a finishing kernel; fp32 runs a SIMT kernel.
 */
mtla_status mtla_project_in(const mtla_dims *dims, int32_t B, int32_t d, const void *x, const void *W_in,
                            const int32_t *pos, void *q_abs, void *q_rope, void *c_new, void *kR_new,
                            void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream);

/*
 * mtla_project_out — the layer's output with the value map absorbed into the
 * output map ([rope]; Figure 1): y[b] = sum_h o[b,h] (W_V^h W_O^h).
 *   o      [B, H, r]    fp32 (mtla_decode_attn's out); rounded to bf16 for
 *                       the bf16 tensor-core path
 *   W_out  [d, H r]     cache dtype, row-major: row n, column h r + i is
 *                       (W_V^h W_O^h)[i, n]
 *   y      [B, d]       fp32
 *   workspace: mtla_project_workspace_bytes(dims, B, d, MTLA_PROJ_OUT) bytes.
 * bf16: H r a multiple of 64.
 */
mtla_status mtla_project_out(const mtla_dims *dims, int32_t B, int32_t d, const float *o, const void *W_out,
                             float *y, void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream);

/*
 * mtla_prefill_kv — the per-head keys and values of a prompt for the
 * un-absorbed masked forward ([mask], [rope]): for every position n of every
 * sequence, k[b, n, h] = c_hat'_n W_K^h and v[b, n, h] = c_hat'_n W_V^h, where
 * c_hat'_n is the latent part of C_hat' (mtla_prefill_masked_attn's c_partial).
 *   c_partial [B, T, r + d_R] bf16 (row stride r + d_R)
 *   W_kv      [2 H d_h, r] bf16, row-major: row h d_h + e is column e of W_K^h,
 *             row H d_h + h d_h + e is column e of W_V^h
 *   k, v      [B, T, H, d_h] bf16, written
 * bf16 with d_h = 64, d_R = 32, r a multiple of 64 up to 256, H even (a
 * tcgen05 GEMM, 128 positions x 256 features per CTA); else UNSUPPORTED.
 */
mtla_status mtla_prefill_kv(const mtla_dims *dims, int32_t B, int32_t T, const void *c_partial, const void *W_kv,
                            void *k, void *v, int32_t *dev_err, void *stream);

/*
 * mtla_prefill_unabsorbed_attn — the masked parallel forward in its
 * un-absorbed form ([mask], [rope]): per head, q_h = x W_Q^h (width d_h),
 *   score_n = (q_h . k_n,h + q_rope_h . k_hat^R'_n) / sqrt(d_h)
 * over the columns n == m and n = g s (g < ceil(m/s)), and
 *   out[b, m, h] = sum_n softmax(score)_n v_n,h   (width d_h),
 * where k_hat^R'_n is the last d_R channels of C_hat'_n.  By associativity
 * (Figure 1) out[b, m, h] = (the absorbed forward's output) W_V^h; each visible
 * pair costs 2 (d_h + d_R) + 2 d_h flops instead of 2 (r + d_R) + 2 r.
 *   q [B, T, H, d_h], q_rope [B, T, H, d_R], k, v [B, T, H, d_h] (from
 *   mtla_prefill_kv), c_partial [B, T, r + d_R]: bf16, contiguous.
 *   out [B, T, H, d_h] bf16, written.
 * Same dims as mtla_prefill_kv; any T >= 1.
 */
mtla_status mtla_prefill_unabsorbed_attn(const mtla_dims *dims, int32_t B, int32_t T, const void *q,
                                         const void *q_rope, const void *k, const void *v, const void *c_partial,
                                         void *out, int32_t *dev_err, void *stream);

/*
 * Training path ([train], [mask], [merge]).  The forward is
 *   mtla_prefill_masked_attn (cache-only: C_hat') -> mtla_prefill_kv (k, v)
 *   -> mtla_train_attn_fwd (out, lse);
 * the backward, given d_out = dL/dout, runs the same chain in reverse:
 *   mtla_train_attn_bwd (dq, dq_rope, dk, dv, dkR) -> mtla_train_kv_bwd
 *   (dL/dC_hat'_latent) -> mtla_train_merge_bwd (dc, dW_c, db_c, dP).
 * Under the shortcut only the latent channels of C_hat' reach the attention;
 * the RoPE key gradient dkR goes to the caller's K^R directly.  Gradients of
 * the caller's own maps (W_Q, W_K, W_V, the projections) are plain GEMMs on
 * these outputs and are left to the caller.  All three backward calls need
 * bf16, d_h = 64, d_R = 32, r = 256.
 */

/*
 * mtla_train_attn_fwd — the masked forward with explicit keys and values and
 * the uncompressed RoPE keys: per head,
 *   score_n = (q_h . k_n,h + q_rope_h . kR_n) / sqrt(d_h)
 * over the columns n == m and n = g s < m ([mask]), out = softmax(score) v.
 *   q, k, v [B, T, H, d_h], q_rope [B, T, H, d_R], kR [B, T, d_R] (RoPE
 *   applied): bf16, contiguous.
 *   out [B, T, H, d_h] bf16 and lse [B, T, H] fp32 (natural log of each
 *   softmax denominator, for mtla_train_attn_bwd): written.
 * Dims as mtla_prefill_unabsorbed_attn; any T >= 1.
 */
mtla_status mtla_train_attn_fwd(const mtla_dims *dims, int32_t B, int32_t T, const void *q, const void *q_rope,
                                const void *k, const void *v, const void *kR, void *out, float *lse,
                                int32_t *dev_err, void *stream);

#define MTLA_TRAIN_ATTN_BWD 1
#define MTLA_TRAIN_KV_BWD 2
#define MTLA_TRAIN_MERGE_BWD 3

/* Workspace bytes of the training backward call `which` (MTLA_TRAIN_*) for B
 * sequences of T tokens (0 on unsupported arguments). */
size_t mtla_train_workspace_bytes(const mtla_dims *dims, int32_t B, int32_t T, int32_t which);

/*
 * mtla_train_attn_bwd — gradients through mtla_train_attn_fwd given
 * d_out = dL/dout (softmax Jacobian: dS = P (d_out v^T - rowsum(d_out out))):
 *   dq, dk, dv [B, T, H, d_h] and dq_rope [B, T, H, d_R]: bf16, written;
 *   dkR [B, T, d_R] fp32, written: summed over heads (every head reads the
 *   same K^R).
 * Inputs as mtla_train_attn_fwd plus its out and lse, and d_out [B, T, H, d_h]
 * bf16.  Every output element is written by exactly one block in a fixed
 * order: the results do not depend on scheduling.
 */
mtla_status mtla_train_attn_bwd(const mtla_dims *dims, int32_t B, int32_t T, const void *q, const void *q_rope,
                                const void *k, const void *v, const void *kR, const void *out, const float *lse,
                                const void *d_out, void *dq, void *dq_rope, void *dk, void *dv, float *dkR,
                                void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream);

/*
 * mtla_train_kv_bwd — dL/dC_hat'_latent through k = C_hat'_latent W_K^h and
 * v = C_hat'_latent W_V^h: dC[b, n] = sum_h dk[b,n,h] (W_K^h)^T + dv[b,n,h] (W_V^h)^T.
 *   dk, dv [B, T, H, d_h] bf16; W_kv as in mtla_prefill_kv (read as stored).
 *   dC [B, T, r] fp32, written.  One tensor-core GEMM (K = 2 H d_h).
 *   Needs no workspace (mtla_train_workspace_bytes returns 0; NULL is fine).
 */
mtla_status mtla_train_kv_bwd(const mtla_dims *dims, int32_t B, int32_t T, const void *dk, const void *dv,
                              const void *W_kv, float *dC, void *workspace, size_t workspace_bytes,
                              int32_t *dev_err, void *stream);

/*
 * mtla_train_merge_bwd — gradients through the latent channels of the running
 * merge ([merge], [mask]): C_hat'_n = sum over tokens i <= n of n's group of
 * w_i ⊙ c_i, w_i = Sigmoid((c_i W_c + b_c) ⊙ P[j(i)-1]), given dC = dL/dC_hat'.
 *   c [B, T, r] bf16 (the latents given to the forward); W_c [r, D], b_c [D],
 *   P [J_max, D] fp32 as in mtla_merge_args; dC [B, T, r] fp32.
 *   dc [B, T, r], dW_c [r, D], db_c [D], dP [J_max, D] fp32: written in full
 *   (entries the latent merge does not reach, the RoPE gate channels and the
 *   groups past T, are zero).  J_max >= ceil(T/s).
 * The gate pre-activations are recomputed from bf16 c and W_c on the tensor
 * cores; the chain rule runs in fp32.
 */
mtla_status mtla_train_merge_bwd(const mtla_dims *dims, int32_t B, int32_t T, const void *c, const float *W_c,
                                 const float *b_c, const float *P, int32_t J_max, const float *dC, float *dc,
                                 float *dW_c, float *db_c, float *dP, void *workspace, size_t workspace_bytes,
                                 int32_t *dev_err, void *stream);

#define MTLA_WS_DECODE 0
#define MTLA_PROJ_IN 1
#define MTLA_PROJ_OUT 2

/* Workspace bytes of mtla_project_in (which = MTLA_PROJ_IN) or
 * mtla_project_out (MTLA_PROJ_OUT) for B tokens and model width d (0 on
 * unsupported arguments).  Queries the current device. */
size_t mtla_project_workspace_bytes(const mtla_dims *dims, int32_t B, int32_t d, int32_t which);

/* Bytes of workspace a call needs (0 if none).  Queries the current device. */
size_t mtla_workspace_bytes(const mtla_dims *dims, int32_t B, int32_t which);

/* Static text for a status code. */
const char *mtla_status_string(mtla_status status);

/* The kernels' own visibility predicate ([mask]) written to host_out[T*T]
 * (row m-1, column n-1, 1 = visible).  Host only; no GPU needed. */
mtla_status mtla_debug_stride_mask(int32_t s, int32_t T, uint8_t *host_out);

/* The kernels' own cache-length rule: rows after t processed tokens. */
int64_t mtla_cache_length(int64_t t, int32_t s);

#ifdef __cplusplus
}
#endif

#endif /* MTLA_H */
