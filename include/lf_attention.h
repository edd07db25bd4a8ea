/*
 * lf_attention.h -- C ABI of the B200 Longformer self-attention library.
 *
 * The library computes the Longformer attention forward on one GPU:
 * each non-global query attends to a sliding window of keys (w/2 taps per
 * side, or w taps to the left when causal), the taps spaced by a per-head
 * dilation, plus every global token; each global query attends to the whole
 * sequence through its own projections Qg, Kg, Vg; padded query rows are zero.
 *
 * Sources:
 *   "LongFormer: The Long-Document Transformer" (reading notes), sections
 *     "Sliding Window", "Dilated Sliding Window", "Global Attention", and the
 *     part on autoregressive language models;
 *   FasterTransformer Longformer Encoder guide, sections "four hard
 *     constraints" (head size 64) and "Longformer Encoder compute flow"
 *     (global-index extraction, local/global softmax, zeroed masked rows).
 *
 * Conventions for every entry point:
 *   - Device pointers point to memory of the current CUDA device; host
 *     pointers are marked "host".  The caller owns every buffer; the library
 *     allocates no memory and keeps no pointer after a call returns.
 *   - Tensors are contiguous and row-major.  Inputs are never modified.
 *   - Work is queued asynchronously on `stream` (a cudaStream_t passed as a
 *     void*, NULL = the legacy default stream).  No entry point synchronises
 *     the stream except lf_workspace_status and lf_attention_forward_host.
 *   - Host-detectable errors return a negative lf_status before anything is
 *     launched.  No C++ exception crosses this interface.
 *   - Errors found on the device (a count of global tokens above max_global,
 *     a bounded wait that ran out) are recorded in a status word inside the
 *     workspace; the output is then undefined.  Read it with
 *     lf_workspace_status.
 *   - All calls are thread-compatible: concurrent calls must use distinct
 *     workspaces and outputs.
 */
#ifndef LF_ATTENTION_H
#define LF_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LF_API __attribute__((visibility("default")))
#else
#define LF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, passed untyped so this header needs no CUDA header. */
typedef void *lf_stream_t;

typedef enum {
    LF_F32 = 0,   /* fp32 in, fp32 arithmetic, fp32 out */
    LF_F16 = 1,   /* fp16 in, fp32 accumulation, fp16 out */
    LF_BF16 = 2   /* bf16 in, fp32 accumulation, bf16 out */
} lf_dtype;

typedef enum {
    LF_OK = 0,
    LF_ERR_INVALID_ARG = -1,      /* bad size, pointer, alignment, window or dilation */
    LF_ERR_UNSUPPORTED = -2,      /* d_head != 64; causal with global tokens */
    LF_ERR_WORKSPACE = -3,        /* workspace NULL, misaligned or too small */
    LF_ERR_CUDA = -4,             /* a CUDA runtime call failed */
    LF_ERR_DEVICE_TIMEOUT = -5,   /* a bounded device-side wait ran out */
    LF_ERR_GLOBAL_OVERFLOW = -6,  /* a batch has more global tokens than max_global */
    LF_ERR_NO_DEVICE = -7,        /* no sm_100 device is current */
    LF_ERR_SCRATCH_LIMIT = -8     /* too large for the fixed scratch (lf_attention_forward_static) */
} lf_status;

/* Library version, major*10000 + minor*100 + patch. */
LF_API int lf_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
LF_API const char *lf_status_string(int status);

/*
 * Global-token index extraction (FasterTransformer Longformer Encoder guide,
 * compute flow: the global mask of each batch is compacted into the list of
 * its global positions and their count).
 *
 *   global_mask  device uint8 [B, n]; nonzero marks a global token.
 *   global_idx   device int32 [B, n]; out: row b holds the global positions of
 *                batch b in ascending order, then -1 up to n.
 *   counts       device int32 [B]; out: number of global tokens per batch.
 *
 * Returns LF_ERR_INVALID_ARG for B < 1, n < 1 or a NULL pointer.
 */
LF_API int lf_global_index(const uint8_t *global_mask, int B, int n,
                    int32_t *global_idx, int32_t *counts, lf_stream_t stream);

/*
 * Workspace bytes needed by lf_attention_prepare / lf_attention_run /
 * lf_attention_forward for these sizes (0 on invalid sizes).  The workspace
 * must be 256-byte aligned device memory; it needs no initialisation.
 * It holds the compacted global indices, per-batch validity and global
 * bitmaps, the fp32 partial results of the global rows, and a status word.
 */
LF_API size_t lf_workspace_size(int B, int H, int n, int d_head, int max_global);

/*
 * Mask preprocessing, once per set of masks (shared by every layer that uses
 * the same masks).  Compacts the global mask (as lf_global_index), builds the
 * per-batch bitmaps of valid keys and of global tokens, clears the status
 * word.
 *
 *   local_mask   device uint8 [B, n]; 1 (nonzero) = valid token, 0 = padding.
 *                NULL: every token valid.
 *   global_mask  device uint8 [B, n]; nonzero = global token.  NULL: none.
 *   max_global   host upper bound on the global tokens of any batch (sizes
 *                grids without a device-to-host copy); 0 when there are none.
 *                A batch above it sets LF_ERR_GLOBAL_OVERFLOW in the status word.
 */
LF_API int lf_attention_prepare(int B, int H, int n, int d_head,
                         const uint8_t *local_mask, const uint8_t *global_mask,
                         int max_global, void *workspace, size_t workspace_bytes,
                         lf_stream_t stream);

/*
 * The attention itself, on a workspace prepared by lf_attention_prepare with
 * the same B, H, n, d_head, max_global and masks.
 *
 *   dtype        element type of all seven tensors.  Each of the seven
 *                pointers must be 16-byte aligned (LF_ERR_INVALID_ARG).
 *   q, k, v      device [B, H, n, d_head]: the sliding-window projections.
 *   qg, kg, vg   device [B, H, n, d_head]: the global projections; qg is read
 *                only at global rows.  May alias q, k, v.
 *   window       w.  Non-causal: even, >= 2; taps i + t*dil[h] for
 *                t in [-w/2, w/2].  Causal: >= 1; taps i - t*dil[h] for
 *                t in [0, w-1].  Taps outside [0, n) are dropped.
 *   dilation     host int32 [H], every entry >= 1.  NULL: all 1.
 *   causal       0 or 1.  Causal attention takes no global tokens: with
 *                causal = 1 a max_global other than 0 is LF_ERR_UNSUPPORTED
 *                (prepare with max_global = 0 and a NULL global mask).
 *   out          device [B, H, n, d_head], same dtype.  Every row is written:
 *                padded rows with zeros.  Must not alias an input.
 *
 * Key set of a valid, non-global row i of head h in batch b:
 *   (window taps of i  UNION  global tokens of b)  INTERSECT  valid tokens of b
 * with softmax over s * <q_i, k_j>, s = 1/sqrt(d_head), applied to v_j.
 * A valid global row attends to every valid token with qg, kg, vg.
 * Inputs must be finite everywhere, padded positions included.
 */
LF_API int lf_attention_run(lf_dtype dtype, int B, int H, int n, int d_head,
                     const void *q, const void *k, const void *v,
                     const void *qg, const void *kg, const void *vg,
                     int max_global, int window, const int32_t *dilation, int causal,
                     void *out, void *workspace, size_t workspace_bytes,
                     lf_stream_t stream);

/*
 * lf_attention_prepare followed by lf_attention_run: the whole forward.
 */
LF_API int lf_attention_forward(lf_dtype dtype, int B, int H, int n, int d_head,
                         const void *q, const void *k, const void *v,
                         const void *qg, const void *kg, const void *vg,
                         const uint8_t *local_mask, const uint8_t *global_mask,
                         int max_global, int window, const int32_t *dilation, int causal,
                         void *out, void *workspace, size_t workspace_bytes,
                         lf_stream_t stream);

/*
 * lf_attention_forward for training (bf16 / fp16): also writes, for every
 * valid row, its log-sum-exp over its key set in log2 units,
 *   lse[b, h, i] = log2( sum_j 2^(s_ij * log2(e) / sqrt(d_head)) ),
 * where s_ij = <q_i, k_j> for a non-global row (window taps and global
 * tokens) and <qg_i, kg_j> for a global row (every valid key): the scores
 * of the row's softmax.  The entries of padded rows are left as they were.
 *
 *   lse          device fp32 [B, H, n], 4-byte aligned; NULL is refused.
 * lf_attention_backward_lse reads it instead of recomputing it.  fp32 inputs
 * return LF_ERR_UNSUPPORTED.  Other arguments and errors as lf_attention_forward.
 */
LF_API int lf_attention_forward_lse(lf_dtype dtype, int B, int H, int n, int d_head,
                             const void *q, const void *k, const void *v,
                             const void *qg, const void *kg, const void *vg,
                             const uint8_t *local_mask, const uint8_t *global_mask,
                             int max_global, int window, const int32_t *dilation, int causal,
                             void *out, float *lse, void *workspace, size_t workspace_bytes,
                             lf_stream_t stream);

/*
 * The whole forward from HOST buffers: copies the projections and the masks
 * from host memory (pinned memory makes the copies asynchronous) into
 * caller-provided device staging buffers, runs lf_attention_forward, copies
 * the output back to host memory and synchronises the stream.  Qg, Kg and Vg
 * are copied only when the global mask has a global position (the kernels
 * read them only then).  lf_host_copy_bytes returns the bytes copied in.
 *
 *   h_q ... h_vg    host [B, H, n, d_head] of dtype.
 *   h_local_mask, h_global_mask   host uint8 [B, n] or NULL.
 *   h_out           host [B, H, n, d_head] of dtype; out.
 *   d_staging       device buffer of lf_host_staging_size(...) bytes,
 *                   256-byte aligned, which receives the copies.
 *   workspace       as for lf_attention_forward.
 *
 * Returns the status of the run or, after the synchronisation, the status
 * word of the workspace.
 */
LF_API size_t lf_host_staging_size(lf_dtype dtype, int B, int H, int n, int d_head);
/* Host-to-device bytes lf_attention_forward_host copies for these arguments
 * (h_local_mask, h_global_mask: the host masks it will be given, or NULL);
 * 0 for unsupported sizes.  Reads the global mask on the host. */
LF_API size_t lf_host_copy_bytes(lf_dtype dtype, int B, int H, int n, int d_head,
                                 const uint8_t *h_local_mask, const uint8_t *h_global_mask);
LF_API int lf_attention_forward_host(lf_dtype dtype, int B, int H, int n, int d_head,
                              const void *h_q, const void *h_k, const void *h_v,
                              const void *h_qg, const void *h_kg, const void *h_vg,
                              const uint8_t *h_local_mask, const uint8_t *h_global_mask,
                              int max_global, int window, const int32_t *dilation,
                              int causal, void *h_out, void *d_staging,
                              size_t staging_bytes, void *workspace,
                              size_t workspace_bytes, lf_stream_t stream);

/*
 * Synchronises `stream`, then returns the device status word of `workspace`
 * (LF_OK, LF_ERR_GLOBAL_OVERFLOW or LF_ERR_DEVICE_TIMEOUT), or LF_ERR_CUDA if
 * the synchronisation or the copy failed.
 */
LF_API int lf_workspace_status(const void *workspace, lf_stream_t stream);

/*
 * Test hooks of the bf16/fp16 attention kernel's bounded waits (failure
 * detection; no counterpart in the method).  Every wait of the kernel on a
 * shared-memory barrier gives up after a time limit, records
 * LF_ERR_DEVICE_TIMEOUT in the workspace status word, lets the CTA's other
 * roles stop, waits (bounded) for its own copies and products in flight,
 * frees its tensor memory and returns.
 *
 *   wait_limit_ns   limit of every such wait, for the launches that follow
 *                   (default 1 s; 0 is refused with LF_ERR_INVALID_ARG).
 *   stall_first_q   nonzero: in later launches CTA 0 never loads the query
 *                   tile of its first item and never signals it, so the wait
 *                   for it runs out (no copy is started for it, nothing is
 *                   left in flight).  0 restores normal launches.
 *
 * Process-wide settings read at each launch; not for concurrent use.  After a
 * device-detected error the workspace must be prepared again
 * (lf_attention_prepare or lf_attention_forward) before lf_attention_run.
 */
LF_API int lf_test_forward_hooks(unsigned long long wait_limit_ns, int stall_first_q);

/*
 * Evaluates, on the device, the 2^x approximation the bf16/fp16 attention
 * kernel uses for part of its exponentials: x = j + f with j the nearest
 * integer and f in [-1/2, 1/2], 2^f from a cubic fitted for minimum maximum
 * relative error on that interval (Remez exchange), 2^j added to the
 * exponent.  Relative error below 7.5e-5 for x >= -125.5; below that the
 * result is a number in [0, 2^-124] (arguments below -126 are clamped).
 *   x, y   device [n] fp32 (y = 2^x).  stream: as elsewhere.
 * For testing the approximation against the SFU exponential and its bound.
 */
LF_API int lf_exp2_poly_eval(const float *x, float *y, int n, lf_stream_t stream);

/*
 * Projection prologue (FasterTransformer Longformer Encoder guide, "compute
 * flow": the Q, K, V, Kg, Vg products over every token, the Qg product over
 * the global tokens only, then bias add and the split into heads).  Produces
 * the six inputs of lf_attention_run / lf_attention_forward.
 *
 *   dtype        LF_BF16 or LF_F16 (fp32 accumulation, outputs rounded to the
 *                input type); LF_F32 is LF_ERR_UNSUPPORTED.
 *   x            device [B, n, H*d_head]: hidden states.
 *   w            device [5*H*d_head, H*d_head]: the Q, K, V, Kg, Vg weight
 *                matrices stacked in that order, each [out, in] (row o holds
 *                the weights of output feature o = h*d_head + e).
 *   bias         device [5*H*d_head] in the same order, or NULL (no bias).
 *   wqg, bqg     device [H*d_head, H*d_head] and [H*d_head] (bqg may be
 *                NULL): the global-query projection.  wqg = NULL or
 *                max_global = 0 skips Qg.
 *   global_idx,  device int32 [B, n] and [B] as written by lf_global_index:
 *   counts       the rows that get Qg (at most max_global per batch).
 *   q, k, v,     device [B, H, n, d_head] outputs: out[b, h, i, e] =
 *   kg, vg       sum_c x[b, i, c] * w[o, c] + bias[o], o = h*d_head + e of
 *                the projection's block.
 *   qg           device [B, H, n, d_head]: written at global positions only;
 *                other rows keep their contents.
 *   status       optional device int32: receives LF_ERR_DEVICE_TIMEOUT if a
 *                bounded device-side wait ran out (left untouched otherwise).
 * Every pointer must be 16-byte aligned.  d_head must be 64.  Outputs must
 * not alias the inputs.
 */
LF_API int lf_qkv_projection(lf_dtype dtype, int B, int n, int H, int d_head,
                      const void *x, const void *w, const void *bias,
                      const void *wqg, const void *bqg,
                      const int32_t *global_idx, const int32_t *counts, int max_global,
                      void *q, void *k, void *v, void *qg, void *kg, void *vg,
                      int32_t *status, lf_stream_t stream);

/*
 * Output layer of the attention block (FasterTransformer Longformer Encoder
 * guide, "compute flow": the heads concatenated back into [B, n, H*d_head],
 * the output projection plus bias, the layer input added back, then layer
 * normalisation):
 *   y[b, i, :] = LayerNorm(concat_h attn[b, h, i, :] . wo^T + bo + residual[b, i, :])
 * with LayerNorm(s) = (s - mean(s)) / sqrt(var(s) + eps) * gamma + beta over
 * the H*d_head features (population variance).
 *
 *   dtype        LF_BF16 or LF_F16 (fp32 accumulation and normalisation).
 *   attn         device [B, H, n, d_head]: the attention output.
 *   wo, bo       device [H*d_head, H*d_head] (rows = output features) and
 *                [H*d_head] or NULL.
 *   residual     device [B, n, H*d_head]: the layer input.
 *   gamma, beta  device [H*d_head].
 *   eps          >= 0, finite.
 *   out          device [B, n, H*d_head].
 *   workspace    device, 256-byte aligned, lf_output_workspace_size bytes:
 *                the fp32 pre-normalisation sums.
 *   status       optional device int32 (see lf_qkv_projection).
 * Every pointer must be 16-byte aligned; d_head must be 64.
 */
LF_API size_t lf_output_workspace_size(int B, int n, int H, int d_head);
LF_API int lf_output_layer(lf_dtype dtype, int B, int n, int H, int d_head,
                    const void *attn, const void *wo, const void *bo, const void *residual,
                    const void *gamma, const void *beta, float eps, void *out,
                    void *workspace, size_t workspace_bytes, int32_t *status,
                    lf_stream_t stream);

/* Size of the fixed scratch of lf_attention_forward_static: 16 MiB. */
#define LF_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * lf_attention_forward with its workspace in a fixed scratch array of
 * LF_STATIC_SCRATCH_BYTES per device, held in the library's own device
 * global memory.  The pages describe nothing like it: it has no counterpart
 * in the method and computes exactly what lf_attention_forward computes; only
 * the place of the workspace differs.
 *
 * It is for callers that cannot allocate device memory when they call: a
 * host program or plugin that receives device tensors and a stream but owns
 * no device allocator, or a latency-bound loop where cudaMalloc / cudaFree
 * are off limits because they can synchronise the device.  It allocates
 * nothing itself.
 *
 *   arguments    as lf_attention_forward, without workspace and
 *                workspace_bytes.
 *   scratch      optional (may be NULL); out: the device address of the
 *                scratch used, to pass to lf_workspace_status to read the
 *                device-side status word of the call.
 *
 * Limit: a problem with lf_workspace_size(B, H, n, d_head, max_global) above
 * LF_STATIC_SCRATCH_BYTES returns LF_ERR_SCRATCH_LIMIT before anything
 * touches the device (for example B = 1, H = 16, n = 16384 with 32 global
 * tokens needs about 4.5 MB).
 * Invalid sizes (those for which lf_workspace_size returns 0) return
 * LF_ERR_INVALID_ARG, and d_head != 64 LF_ERR_UNSUPPORTED, also before
 * anything touches the device.
 * Set-up: the first call on a device looks up the scratch address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture.  The cached address does not survive
 * cudaDeviceReset: a process that resets a device must not call this entry
 * point on that device again.
 * Concurrency: there is one scratch per device, so calls on the same device
 * that overlap in time (several streams or host threads) race on it; callers
 * serialise them.  Nothing must be cleared beforehand: each call's
 * mask-preparation step clears what has to start at zero.
 */
LF_API int lf_attention_forward_static(lf_dtype dtype, int B, int H, int n, int d_head,
                         const void *q, const void *k, const void *v,
                         const void *qg, const void *kg, const void *vg,
                         const uint8_t *local_mask, const uint8_t *global_mask,
                         int max_global, int window, const int32_t *dilation, int causal,
                         void *out, lf_stream_t stream, void **scratch);

/*
 * Backward pass of the attention: the gradients of a scalar loss with
 * respect to the six projections, given dO = dLoss/dO of the forward output.
 * ("LongFormer: The Long-Document Transformer" notes, "Sliding Window",
 * "Dilated Sliding Window", "Global Attention" define the attention; its
 * derivative is the softmax-attention chain rule.  The pages print no
 * backward of their own.)
 *
 * With s_ij = <q_i, k_j> / sqrt(d_head), p_ij = softmax over the keys of row
 * i, and D_i = <dO_i, O_i>:
 *   dv_j = sum_i p_ij dO_i,   dS_ij = p_ij (<dO_i, v_j> - D_i),
 *   dq_i = sum_j dS_ij k_j / sqrt(d_head),  dk_j = sum_i dS_ij q_i / sqrt(d_head),
 * where rows and keys run over the same sets as the forward: a valid
 * non-global row i uses Q, K, V over its window taps and the global tokens,
 * a valid global row uses Qg, Kg, Vg over every valid token.  Gradients of
 * rows and keys that take part in nothing (padded tokens; Qg rows of
 * non-global tokens; Q rows of global tokens) are written as zeros.
 *
 *   q ... vg, max_global, window, dilation, causal
 *                as passed to the forward.
 *   out          device [B, H, n, d_head]: the forward's output for these
 *                inputs (the library's, or any O within rounding of it).
 *   dout         device [B, H, n, d_head]: dLoss/dO.
 *   dq ... dvg   device [B, H, n, d_head], out: every element is written.
 *   workspace    the workspace of the forward, prepared for the same masks
 *                and max_global (lf_attention_prepare or
 *                lf_attention_forward); read only.
 *   scratch      device, 256-byte aligned, lf_backward_scratch_size bytes:
 *                per-row log-sum-exp and D between the kernels, and the fp32
 *                partial sums of the global-token parts.  Overwritten by
 *                every call; nothing needs clearing beforehand.
 * fp32 inputs: CUDA-core kernels, fp32 arithmetic.  bf16 / fp16 inputs:
 * tcgen05 kernels for the window band (P and dS rounded to the input type
 * before their products, fp32 accumulation), CUDA-core fp32 kernels for the
 * global-token parts; more than 24 (dilation, residue) classes over the heads
 * send the whole call to the CUDA-core kernels.  Part of the work runs on a
 * second, library-owned stream of the device, forked from and joined back to
 * `stream` with events (stream capture included).
 * Every tensor pointer must be 16-byte aligned.  Errors are returned before
 * anything is launched, as for lf_attention_run.  More global tokens than
 * max_global is recorded by the preparation in the workspace status word
 * (lf_workspace_status), as for the forward.
 */
LF_API size_t lf_backward_scratch_size(int B, int H, int n, int d_head, int max_global);
LF_API int lf_attention_backward(lf_dtype dtype, int B, int H, int n, int d_head,
                         const void *q, const void *k, const void *v,
                         const void *qg, const void *kg, const void *vg,
                         const void *out, const void *dout,
                         int max_global, int window, const int32_t *dilation, int causal,
                         void *dq, void *dk, void *dv, void *dqg, void *dkg, void *dvg,
                         const void *workspace, size_t workspace_bytes,
                         void *scratch, size_t scratch_bytes, lf_stream_t stream);

/*
 * lf_attention_backward (bf16 / fp16) with the rows' log-sum-exp taken from
 * lf_attention_forward_lse on the same inputs, instead of first passes over
 * the keys that recompute it (band rows and global rows).
 *
 *   lse          device fp32 [B, H, n] as lf_attention_forward_lse wrote it
 *                for these inputs, 4-byte aligned; NULL is refused.
 * fp32 inputs return LF_ERR_UNSUPPORTED.  Other arguments and errors as
 * lf_attention_backward (the CUDA-core fallback recomputes the values).
 */
LF_API int lf_attention_backward_lse(lf_dtype dtype, int B, int H, int n, int d_head,
                              const void *q, const void *k, const void *v,
                              const void *qg, const void *kg, const void *vg,
                              const void *out, const void *dout, const float *lse,
                              int max_global, int window, const int32_t *dilation, int causal,
                              void *dq, void *dk, void *dv, void *dqg, void *dkg, void *dvg,
                              const void *workspace, size_t workspace_bytes, void *scratch,
                              size_t scratch_bytes, lf_stream_t stream);

/*
 * Feed-forward block of an encoder layer (FasterTransformer Longformer
 * Encoder guide, "compute flow": intermediate product plus bias, GELU,
 * output product, then bias, residual and LayerNorm once more):
 *   act = GELU(h W1^T + b1),        GELU(x) = x * Phi(x) (the erf form)
 *   out = LayerNorm(act W2^T + b2 + h) * gamma + beta
 * Both products run on the tensor cores with fp32 accumulation; act is
 * stored in dtype, the pre-normalisation sum in fp32.
 *
 *   dtype        LF_BF16 or LF_F16 (LF_F32: LF_ERR_UNSUPPORTED).
 *   hidden       features per token; a multiple of 64.
 *   inter        intermediate features; a multiple of 64.
 *   h            device [B, n, hidden]: the block input (also the residual).
 *   w1, b1       device [inter, hidden] (rows = output features), [inter] or NULL.
 *   w2, b2       device [hidden, inter], [hidden] or NULL.
 *   gamma, beta  device [hidden]; eps >= 0 is added to the variance.
 *   out          device [B, n, hidden]; must not overlap h.
 *   workspace    device, 256-byte aligned, lf_ffn_workspace_size bytes.
 *   status       optional device int32 (see lf_qkv_projection).
 * Every pointer must be 16-byte aligned.
 */
LF_API size_t lf_ffn_workspace_size(int B, int n, int hidden, int inter);
LF_API int lf_ffn_block(lf_dtype dtype, int B, int n, int hidden, int inter, const void *h,
                        const void *w1, const void *b1, const void *w2, const void *b2,
                        const void *gamma, const void *beta, float eps, void *out,
                        void *workspace, size_t workspace_bytes, int32_t *status,
                        lf_stream_t stream);

/*
 * Device pointers of one encoder layer's weights (rows = output features,
 * hid = H * d_head).  Biases may be NULL (zero).
 */
typedef struct lf_layer_weights {
    const void *w_qkv;      /* [5*hid, hid]: Q, K, V, Kg, Vg stacked, as lf_qkv_projection */
    const void *b_qkv;      /* [5*hid] */
    const void *w_qg;       /* [hid, hid]: global queries; may be NULL when max_global = 0 */
    const void *b_qg;       /* [hid] */
    const void *w_o;        /* [hid, hid]: attention output projection */
    const void *b_o;        /* [hid] */
    const void *ln1_gamma;  /* [hid]: LayerNorm after the attention block */
    const void *ln1_beta;   /* [hid] */
    const void *w_1;        /* [inter, hid]: intermediate product */
    const void *b_1;        /* [inter] */
    const void *w_2;        /* [hid, inter]: feed-forward output product */
    const void *b_2;        /* [hid] */
    const void *ln2_gamma;  /* [hid]: LayerNorm after the feed-forward block */
    const void *ln2_beta;   /* [hid] */
} lf_layer_weights;

/*
 * A stack of Longformer encoder layers (FasterTransformer Longformer Encoder
 * guide, "compute flow"; "LongFormer: The Long-Document Transformer" notes,
 * "Sliding Window", for a window per layer).  Per layer: lf_qkv_projection,
 * lf_attention_run (non-causal), lf_output_layer with the layer input as
 * residual, lf_ffn_block.  The masks are prepared once (lf_attention_prepare)
 * for all layers.
 *
 *   dtype        LF_BF16 or LF_F16.
 *   inter        intermediate features of the feed-forward block (multiple of 64).
 *   layers       >= 1.
 *   weights      host [layers] of device pointers.
 *   windows      host [layers]: window of each layer (even, >= 2).
 *   dilations    host [layers * H] (layer-major) or NULL for all 1.
 *   x            device [B, n, H*d_head]: the stack input.
 *   local_mask, global_mask, max_global  as lf_attention_forward.
 *   eps          of both LayerNorms.
 *   out          device [B, n, H*d_head]: the last layer's output; must not
 *                overlap x.
 *   workspace    device, 256-byte aligned, lf_encoder_workspace_size bytes.
 *                It begins with the attention workspace, so
 *                lf_workspace_status(workspace) reads the one status word
 *                every step of the stack records into.
 * Errors in the arguments of any layer return before anything is launched.
 */
LF_API size_t lf_encoder_workspace_size(int B, int n, int H, int d_head, int inter,
                                        int max_global);
LF_API int lf_encoder_forward(lf_dtype dtype, int B, int n, int H, int d_head, int inter,
                              int layers, const lf_layer_weights *weights,
                              const int32_t *windows, const int32_t *dilations, const void *x,
                              const uint8_t *local_mask, const uint8_t *global_mask,
                              int max_global, float eps, void *out, void *workspace,
                              size_t workspace_bytes, lf_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LF_ATTENTION_H */
