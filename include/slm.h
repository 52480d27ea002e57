/*
 * slm.h - C ABI of the streaming LM-head loss for NVIDIA B200 (sm_100a).
 *
 * What is computed.  Hidden states H_q [N, d] are projected by the LM head W [V, d] to
 * logits z_q = H_q W^T [N, V], which are reduced to one loss per token row and to the
 * gradients dH_q [N, d] and dW [V, d], without ever storing the [N, V] logits or their
 * gradient ("Training speculative decoders: removing the logits and attention
 * bottlenecks", sections "The logits bottleneck in long-context draft-head training",
 * "Streaming Cross Entropy" and "Backward pass").
 *
 * Loss kinds ("Loss Functions", table "Available Losses"; p = softmax(H_p W^T) is the
 * target, q = softmax(H_q W^T) the draft, alpha = sum_v min(p_v, q_v)):
 *   SLM_CE         hard-label cross entropy  -log q_y       (labels required)
 *   SLM_KL         forward KL, target to draft  KL(p || q)
 *   SLM_TV         total variation  1 - alpha
 *   SLM_NLA        negative log-acceptance  -log(alpha)   (alpha clamped at 1e-30)
 *   SLM_LK_HYBRID  lambda * KL + (1 - lambda) * TV,  lambda = exp(-3 alpha) per token,
 *                  detached (no gradient through lambda)
 *   SLM_RKL        reverse KL, draft to target  KL(q || p)
 *   SLM_JSD        Jensen-Shannon divergence  (KL(p || M) + KL(q || M)) / 2, M = (p + q) / 2,
 *                  bounded by log 2
 *   SLM_CE_ARGMAX_P  cross entropy against argmax p: hard labels from the target (the
 *                  lowest vocabulary index wins a tie)
 * The target p is detached: gradients flow to H_q and to W through z_q only.
 *
 * Masking and normalisation ("Streaming Cross Entropy"; "Correctness: alignment before
 * chunking"): a row whose label equals ignore_index is masked and contributes 0 to the
 * loss and to every gradient.  The library returns the masked loss SUM and the number of
 * valid rows; the mean divides by the number of valid rows (never by a chunk count).
 * With every row masked the mean is defined as 0 and every gradient is 0.
 *
 * Conventions shared by every entry point:
 *   - Pointers to tensors are DEVICE pointers owned by the caller, on the current CUDA
 *     device.  The library never allocates device memory: scratch lives in the caller's
 *     `workspace` (size from slm_workspace_bytes, 256-byte aligned base).
 *   - bf16 tensors are passed as `const void*` and are row-major, contiguous:
 *     H_q, H_p [N, d]; W [V, d]; dH_q [N, d].  Every tensor base must be 16-byte aligned
 *     and d must be a multiple of 8 (16-byte rows for the tensor-memory-access engine).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is enqueued
 *     asynchronously on it; no entry point synchronises, except slm_device_status.
 *   - Errors found on the host (null pointer, bad shape or alignment, small workspace,
 *     wrong kind, unsupported GPU, CUDA launch error) are returned immediately and nothing
 *     is enqueued.  Errors found on the device (a label outside [0, V) that is not
 *     ignore_index, a pipeline wait that ran out of time) are recorded in the workspace
 *     status word: the affected rows are treated as masked, and slm_device_status reports
 *     the flag.  Kernels never trap.
 */
#ifndef SLM_H_
#define SLM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLM_API __attribute__((visibility("default")))
#else
#define SLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum slm_loss_kind {
  SLM_CE = 0,
  SLM_KL = 1,
  SLM_TV = 2,
  SLM_NLA = 3,
  SLM_LK_HYBRID = 4,
  SLM_RKL = 5,
  SLM_JSD = 6,
  SLM_CE_ARGMAX_P = 7
} slm_loss_kind;

typedef enum slm_status {
  SLM_OK = 0,
  SLM_ERR_NULL = 1,             /* a required pointer is NULL                          */
  SLM_ERR_SHAPE = 2,            /* N < 0, d <= 0, V <= 0, d % 8 != 0, or too large      */
  SLM_ERR_ALIGN = 3,            /* a tensor base is not 16-byte aligned                  */
  SLM_ERR_KIND = 4,             /* unknown loss kind                                     */
  SLM_ERR_WORKSPACE = 5,        /* workspace NULL, misaligned or smaller than required  */
  SLM_ERR_LABEL_RANGE = 6,      /* device: a CE label outside [0, V), row masked         */
  SLM_ERR_TIMEOUT = 7,          /* device: a pipeline wait ran out of time               */
  SLM_ERR_CUDA = 8,             /* a CUDA runtime call or launch failed                  */
  SLM_ERR_UNSUPPORTED_ARCH = 9  /* the current device is not compute capability 10.0    */
} slm_status;

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
SLM_API int slm_version(void);

/* Human-readable name of a status code (static string; never NULL). */
SLM_API const char* slm_status_string(int status);

/* Number of floats per token row of the `stats` array that slm_loss_fwd writes and
 * slm_loss_bwd reads (layout [k][N], field-major):
 *   SLM_CE: 1  (L_q = logsumexp z_q)
 *   SLM_CE_ARGMAX_P: 2  (L_q, the argmax-p target as int32 bits; ignore_index if masked)
 *   SLM_KL: 3  (L_q, L_p, KL);  SLM_RKL: 3  (L_q, L_p, RKL)
 *   SLM_TV, SLM_NLA, SLM_LK_HYBRID: 5  (L_q, L_p, KL, alpha, S = sum_{q_v < p_v} q_v)
 *   SLM_JSD: 5  (L_q, L_p, KL, JSD, T = sum_v q_v (log q_v - log M_v) / 2)
 * Returns 0 for an unknown kind. */
SLM_API size_t slm_stats_floats(int kind);

/* Bytes of workspace that slm_loss_fwd and slm_loss_bwd need for these sizes (the
 * forward alone needs no more than the value for any chunk_tokens).
 * chunk_tokens is the backward's token chunk (0 = automatic: min(N, 2d) rounded up to
 * 128); the workspace then holds one bf16 [chunk, V] logits-gradient buffer, which is the
 * streaming chunk buffer of "Backward pass".  Returns 0 on invalid arguments. */
SLM_API size_t slm_workspace_bytes(int kind, int64_t N, int64_t d, int64_t V, int64_t chunk_tokens);

/* Forward pass ("Streaming Cross Entropy"; "Available Losses").
 *   Hq      bf16 [N, d]  draft hidden states (the hidden states for SLM_CE).
 *   Hp      bf16 [N, d]  target hidden states; required for every kind but SLM_CE
 *                        (ignored for SLM_CE, may be NULL there).
 *   W       bf16 [V, d]  LM-head weight, shared by target and draft.
 *   labels  int32 [N]    SLM_CE: the target token of each row, required; a value equal
 *                        to ignore_index masks the row, any other value outside [0, V)
 *                        sets SLM_ERR_LABEL_RANGE and masks the row.
 *                        Other kinds: optional row mask (NULL = every row valid).
 *                        (SLM_CE_ARGMAX_P takes its targets from H_p; labels only mask.)
 *   loss_tok   float [N]  per-token loss (0 on masked rows); may be NULL.
 *   alpha_tok  float [N]  per-token alpha for TV / NLA / LK_HYBRID; may be NULL.
 *   loss_sum   double [1] masked loss sum; required.
 *   n_valid    int64 [1]  number of valid rows; required.
 *   loss_mean  float [1]  loss_sum / n_valid (0 when n_valid = 0); may be NULL.
 *   stats      float [slm_stats_floats(kind) * N] per-token statistics kept for the
 *                        backward (layout above); required when N > 0.
 *   workspace  device scratch of at least slm_workspace_bytes(kind, N, d, V, *) bytes.
 * SLM_CE, SLM_KL, SLM_RKL and SLM_CE_ARGMAX_P make one pass of the LM-head GEMM over the
 * vocabulary; the alpha-based kinds and SLM_JSD make two (they need the final
 * log-sum-exps). */
SLM_API int slm_loss_fwd(int kind, const void* Hq, const void* Hp, const void* W,
                 const int32_t* labels, int32_t ignore_index,
                 int64_t N, int64_t d, int64_t V,
                 float* loss_tok, float* alpha_tok, double* loss_sum, int64_t* n_valid,
                 float* loss_mean, float* stats,
                 void* workspace, size_t ws_bytes, void* stream);

/* Backward pass ("Backward pass": per token chunk, recompute the logits, form the
 * logits gradient, produce the chunk's hidden-state gradient and accumulate the LM-head
 * gradient).  The upstream gradient of token n's loss is
 *     g_n = valid_n * (grad_tok ? grad_tok[n] : 1) * (grad_scale ? *grad_scale : 1)
 *           / (n_valid ? max(*n_valid, 1) : 1)
 * so passing grad_tok = NULL, grad_scale = d(out)/d(mean) and the forward's n_valid gives
 * the gradient of the mean loss.
 *   grad_tok    float [N] or NULL;  grad_scale float [1] or NULL;  n_valid int64 [1] or NULL
 *   stats       float [k * N] written by slm_loss_fwd for the same inputs.
 *   dHq         bf16 [N, d]  overwritten with dLoss/dH_q.
 *   dW          float [V, d] dLoss/dW; overwritten when accumulate_dW == 0, else added to.
 *   chunk_tokens  token chunk of the streaming loop (0 = automatic, see above).
 * There is no gradient for Hp (the target is detached). */
SLM_API int slm_loss_bwd(int kind, const void* Hq, const void* Hp, const void* W,
                 const int32_t* labels, int32_t ignore_index,
                 int64_t N, int64_t d, int64_t V,
                 const float* grad_tok, const float* grad_scale, const int64_t* n_valid,
                 const float* stats, void* dHq, float* dW, int accumulate_dW,
                 int64_t chunk_tokens, void* workspace, size_t ws_bytes, void* stream);

/* slm_loss_bwd for data-parallel training, where dW is summed across ranks after the
 * backward ("Training speculative decoders: removing the logits and attention
 * bottlenecks", "Streaming Cross Entropy": the streaming loss is orthogonal to data
 * parallelism).  Same arguments, same results, bit for bit, plus:
 *   dw_ready_event  a cudaEvent_t created by the caller, or NULL.  It is recorded on
 *                   `stream` as soon as dW is final, before the last chunk's dH GEMM, so a
 *                   reduction of dW on another stream can wait on it and overlap that GEMM.
 *                   The caller owns the event; it is recorded once per call.
 *   reserve_sms     SMs (0..128) that the last chunk's dH GEMM leaves idle, so that the
 *                   reduction's kernels find free SMs while it runs; rounded up to whole
 *                   2-SM pairs.  0 = use them all.
 * To make this possible, the last chunk runs its dW GEMM before its dH GEMM.
 * Returns SLM_ERR_SHAPE for reserve_sms outside 0..128 and otherwise what slm_loss_bwd
 * returns. */
SLM_API int slm_loss_bwd_overlap(int kind, const void* Hq, const void* Hp, const void* W,
                 const int32_t* labels, int32_t ignore_index,
                 int64_t N, int64_t d, int64_t V,
                 const float* grad_tok, const float* grad_scale, const int64_t* n_valid,
                 const float* stats, void* dHq, float* dW, int accumulate_dW,
                 int64_t chunk_tokens, void* workspace, size_t ws_bytes, void* stream,
                 void* dw_ready_event, int reserve_sms);

/* Chunk-size rule ("Choosing the chunk size": the largest chunk that keeps the loss path's
 * memory peak below the next peak of the training step, e.g. a transformer block's).  Returns
 * the largest chunk_tokens, a multiple of 128 (of 256 with fused != 0), whose workspace
 * (slm_workspace_bytes, or slm_fused_workspace_bytes with fused != 0) fits in budget_bytes;
 * the result never exceeds N: a value equal to N means every row fits in one chunk (it is
 * then not a multiple of 128 when N is not).  Returns 0 when not even the smallest chunk
 * fits, or on invalid arguments.  Host only; no device is touched. */
SLM_API int64_t slm_chunk_for_budget(int kind, int64_t N, int64_t d, int64_t V,
                                     size_t budget_bytes, int fused);

/* Synchronises `stream`, then returns and clears the device status word of `workspace`:
 * SLM_OK, SLM_ERR_LABEL_RANGE or SLM_ERR_TIMEOUT (the first found), or SLM_ERR_CUDA if
 * the stream reported an error.  Every slm_loss_fwd / slm_loss_bwd call also clears the
 * word when it starts, so the status describes the most recent call. */
SLM_API int slm_device_status(const void* workspace, void* stream);

/* Number of valid rows, counted the way the kernels mask them ("Streaming Cross Entropy":
 * the mean divides by the number of valid, non-masked tokens of the whole batch).  A row is
 * valid when its label is not ignore_index and, for SLM_CE, lies in [0, V); with labels
 * NULL (every kind but SLM_CE) all N rows are valid.  Data-parallel training sums this
 * count over the ranks before the backward, so that each rank divides by the global count
 * and out-of-range CE labels are left out of it exactly as the kernels leave them out.
 *   labels   int32 [N] device, or NULL (required for SLM_CE when N > 0).
 *   n_valid  int64 [1] device, overwritten.
 * Asynchronous on `stream`.  Returns SLM_ERR_KIND, SLM_ERR_SHAPE (N < 0, V <= 0, or either
 * >= 2^31) or SLM_ERR_NULL on bad arguments, before anything is enqueued. */
SLM_API int slm_count_valid(int kind, const int32_t* labels, int32_t ignore_index,
                            int64_t N, int64_t V, int64_t* n_valid, void* stream);

/* Launch shape of the backward (slm_loss_bwd, slm_combo_bwd and the backward half of
 * slm_loss_fwd_bwd).  The pages' backward ("Backward pass") is, per token chunk: recompute
 * the logits, form their gradient, produce the chunk's dH, accumulate dW.
 *   mode 1 (default): each chunk is ONE persistent launch.  Its CTA pairs first compute the
 *          logits-gradient tiles, then the dH and dW tiles; a dH tile starts as soon as the
 *          logits gradient of its 256 rows is complete, a dW tile as soon as that of its 256
 *          vocabulary rows is, ordered by counters in the workspace (bounded waits: a wait
 *          that runs out records SLM_ERR_TIMEOUT).  The pairs' dW shares are sized so that
 *          every pair ends at about the same time.
 *   mode 0: three launches per chunk (logits gradient, dH, dW).
 * Both give the same results (dW bit for bit; the same arithmetic in the same order).
 * slm_loss_bwd_overlap runs its last chunk as three launches in any mode (that chunk's dW
 * must be final before its dH GEMM).
 * Process-wide; takes effect at the next call.  Returns the previous mode, or -1 for an
 * invalid mode (nothing changes). */
SLM_API int slm_set_backward_mode(int mode);

/* Kernel-class timing.  The pages define no counterpart: this is the library's own
 * measurement hook, used to report each GEMM of the path against its roofline.
 * slm_trace_enable(1) makes every following kernel launch of the library (any entry point,
 * any host thread) record a CUDA event on its stream before and after it; slm_trace_enable(0)
 * stops recording.  slm_trace_read waits for the recorded events, adds up their elapsed
 * times per kernel class and clears the record:
 *   ms[c]        milliseconds spent in class c since the last read (launch to launch end
 *                on its stream);
 *   launches[c]  number of launches of class c.
 * The classes (index c) are SLM_TRACE_*.  n_classes may be smaller than SLM_TRACE_CLASSES
 * (the rest is not reported).  The events are host-side CUDA resources created on first
 * use and reused; no device memory is allocated.  At most 65536 launches are recorded
 * between reads; further ones are dropped and slm_trace_read then returns
 * SLM_ERR_WORKSPACE (the sums cover the recorded ones).  Returns SLM_ERR_CUDA if an event
 * failed, SLM_ERR_NULL for NULL outputs.  Do not trace inside a stream capture. */
#define SLM_TRACE_FWD_GEMM 0     /* forward statistics GEMMs (pass 1, flatness)          */
#define SLM_TRACE_PASS2_GEMM 1   /* second-pass GEMMs (alpha and S, JSD halves)          */
#define SLM_TRACE_DZ_GEMM 2      /* backward logits recompute + logits-gradient GEMMs    */
#define SLM_TRACE_DH_GEMM 3      /* dH = dZ W                                            */
#define SLM_TRACE_DW_GEMM 4      /* dW (+)= dZ^T H                                       */
#define SLM_TRACE_BWD_FUSED 5    /* the persistent fused backward (dZ, dH, dW together)  */
#define SLM_TRACE_LOGITS_ROW 6   /* row kernels over kept logits (slm_loss_fwd_bwd)      */
#define SLM_TRACE_ROW 7          /* combines, reductions, counts, alignment              */
#define SLM_TRACE_CLASSES 8
SLM_API int slm_trace_enable(int on);
SLM_API int slm_trace_read(double* ms, int64_t* launches, int n_classes);

/* Fused forward + backward in one call ("Backward pass": for each token chunk, compute the
 * logits, the loss and the gradients; the chunk's logits plus gradient buffer bounds the
 * memory).  For each chunk of chunk_tokens rows (0 = automatic: 4096; rounded up to a
 * multiple of 256), the forward GEMM keeps the chunk's fp32 logits (the draft's, and the
 * target's for the distribution kinds) in the workspace, and the logits gradient (and the
 * second pass of the alpha losses and JSD) read them back instead of recomputing them:
 * 6NVd flops for CE instead of 8NVd, 8NVd for KL / RKL instead of 12NVd, 8NVd for the
 * alpha losses and JSD instead of 16NVd, at the cost of about 10 bytes of memory traffic
 * per logit and a workspace of chunk x V x (4 or 8 + 2) bytes.
 * Outputs and conventions are those of slm_loss_fwd followed by slm_loss_bwd with
 * n_valid = the forward's count: the upstream gradient of token n's loss is
 *     valid_n * (grad_tok ? grad_tok[n] : 1) * (grad_scale ? *grad_scale : 1) / max(n_valid, 1).
 * The workspace size comes from slm_fused_workspace_bytes. */
SLM_API size_t slm_fused_workspace_bytes(int kind, int64_t N, int64_t d, int64_t V,
                                         int64_t chunk_tokens);

SLM_API int slm_loss_fwd_bwd(int kind, const void* Hq, const void* Hp, const void* W,
                             const int32_t* labels, int32_t ignore_index,
                             int64_t N, int64_t d, int64_t V,
                             const float* grad_tok, const float* grad_scale,
                             float* loss_tok, float* alpha_tok, double* loss_sum,
                             int64_t* n_valid, float* loss_mean, float* stats,
                             void* dHq, float* dW, int accumulate_dW, int64_t chunk_tokens,
                             void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Weighted combinations ("Loss Functions", section "Weighted Combinations"): the loss is
 * sum_k w_k * loss_k over the kinds above, with the weights used as given (not
 * normalised); each term is also reported on its own, before its weight is applied.  Every
 * term shares the row mask and the valid count, and one logit pass: the forward makes one
 * pass over the vocabulary (two when a TV, NLA, LK_HYBRID or JSD term is present), the
 * backward one logit recompute that forms sum_k w_k dz_k, then one dH and one dW GEMM.
 *   weights  HOST float [SLM_NUM_KINDS], indexed by slm_loss_kind; 0 = term absent; at
 *            least one nonzero; no NaN or infinity (else SLM_ERR_KIND).
 *   Hp       required when any term but SLM_CE is present.
 *   labels   required when the SLM_CE term is present; otherwise an optional row mask.
 *   term_loss_tok  float [SLM_NUM_KINDS][N] per-term per-token losses before weighting
 *            (0 for absent terms and masked rows); may be NULL.
 *   term_loss_sum  double [SLM_NUM_KINDS] per-term loss sums; may be NULL.
 *   stats    float [SLM_COMBO_STATS][N]: L_q, L_p, KL, RKL, alpha, S, JSD, T, argmax-p
 *            target (int32 bits; ignore_index on masked rows).
 * Everything else is as for slm_loss_fwd / slm_loss_bwd; the workspace size comes from
 * slm_combo_workspace_bytes.
 * ------------------------------------------------------------------------------------- */
#define SLM_NUM_KINDS 8
#define SLM_COMBO_STATS 9

SLM_API size_t slm_combo_workspace_bytes(int64_t N, int64_t d, int64_t V, int64_t chunk_tokens);

SLM_API int slm_combo_fwd(const float* weights, const void* Hq, const void* Hp, const void* W,
                          const int32_t* labels, int32_t ignore_index,
                          int64_t N, int64_t d, int64_t V,
                          float* loss_tok, float* term_loss_tok, double* loss_sum,
                          double* term_loss_sum, int64_t* n_valid, float* loss_mean,
                          float* stats, void* workspace, size_t ws_bytes, void* stream);

SLM_API int slm_combo_bwd(const float* weights, const void* Hq, const void* Hp, const void* W,
                          const int32_t* labels, int32_t ignore_index,
                          int64_t N, int64_t d, int64_t V,
                          const float* grad_tok, const float* grad_scale,
                          const int64_t* n_valid, const float* stats, void* dHq, float* dW,
                          int accumulate_dW, int64_t chunk_tokens, void* workspace,
                          size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Draft-head helpers either side of the path.
 * ------------------------------------------------------------------------------------- */
/* Target alignment before chunking ("Training speculative decoders: ...", section
 * "Correctness: alignment before chunking": hidden states, targets and masks are aligned
 * for the objective first, masks applied, and only then split into chunks; each draft head
 * may predict a different future token, so the target shift depends on the head).
 *   tokens     int32 [B, S] token ids (device).
 *   loss_mask  uint8 [B, S] or NULL: 0 = this position may not be a target.
 *   seq_ids    int32 [B, S] or NULL: packed-sequence id of each position; a target never
 *              crosses into another sequence.
 *   shift      >= 0: the head predicts the token `shift` positions ahead (1 = next token).
 *   labels     int32 [B, S] out: tokens[b, t + shift] where t + shift < S and the target is
 *              unmasked and in the same sequence, else ignore_index.
 * Integer work, exact.  Returns SLM_ERR_SHAPE for negative sizes or shift. */
SLM_API int slm_align_labels(const int32_t* tokens, const uint8_t* loss_mask,
                             const int32_t* seq_ids, int64_t B, int64_t S, int32_t shift,
                             int32_t ignore_index, int32_t* labels, void* stream);

/* Per-token flatness of the target distribution p = softmax(H_p W^T) ("Flatter Tokens are
 * More Valuable for Speculative Draft Model Training": the cosine similarity of the target
 * distribution to the uniform one), which equals 1 / (sqrt(V) ||p||_2): 1 for a uniform p,
 * 1/sqrt(V) for a one-hot p.  One vocabulary-tiled GEMM pass over H_p with an online
 * sum of e^(2 (z - m)) in the epilogue; the logits are never stored.
 *   Hp    bf16 [N, d];  W bf16 [V, d];  flat  float [N] out.
 *   workspace  at least slm_flatness_workspace_bytes(N, d, V) bytes. */
SLM_API size_t slm_flatness_workspace_bytes(int64_t N, int64_t d, int64_t V);
SLM_API int slm_target_flatness(const void* Hp, const void* W, int64_t N, int64_t d, int64_t V,
                                float* flat, void* workspace, size_t ws_bytes, void* stream);

/* Test hook for the device-side failure path (not for production use).  fault_mode 1 makes
 * every following launch withhold one internal pipeline release, so that a bounded wait in
 * the kernel runs out: the kernel then records SLM_ERR_TIMEOUT in the workspace status word,
 * lets its own copies and MMAs finish, frees its tensor memory and returns; results of that
 * call are undefined.  fault_mode 2 makes the GEMMs' CTA pairs give up their loose
 * lockstep at the first wait (it only shapes performance: results must not change).
 * fault_mode 0 restores normal operation.  timeout_cycles bounds every
 * pipeline wait in SM clock cycles (0 = the default of 4e9, about 2 s).  Process-wide;
 * takes effect at the next launch.  Returns SLM_ERR_SHAPE for an invalid mode or bound. */
SLM_API int slm_debug_set(int fault_mode, long long timeout_cycles);

/* Test hook (not for production use): evaluates, for each x[i] (device float [n]), the
 * 2^x that the loss epilogues compute on the FMA pipe for part of their exponentials
 * (y_fma[i]), and CUDA's exp2f (y_mufu[i]).  The former rounds x to an integer j and
 * evaluates 2^(x - j) by a degree-5 polynomial whose coefficients this library fitted; it is
 * meant for x <= 0 and clamps x at -126.  Asynchronous on `stream`.  Returns SLM_ERR_SHAPE
 * for n < 0 or n >= 2^31, SLM_ERR_NULL for a NULL buffer when n > 0. */
SLM_API int slm_debug_exp2(const float* x, float* y_fma, float* y_mufu, int64_t n, void* stream);

/* Size of the device scratch array behind slm_loss_fwd_noalloc: 32 MiB per GPU that loads
 * the library's device code, held until the process exits. */
#define SLM_NOALLOC_SCRATCH_BYTES (32u << 20)

/* Forward pass for callers that cannot allocate device memory.  The pages have no
 * counterpart to this entry point; it exists for hosts that have no allocator of their own
 * to hand out a workspace (a plain C program linking this library), runtimes whose enqueue
 * path must not call cudaMalloc because it can synchronise the device, and processes with a
 * fixed memory budget.
 * Same arguments, outputs and results as slm_loss_fwd, without the workspace: the scratch
 * lives in a fixed __device__ array of SLM_NOALLOC_SCRATCH_BYTES.  Sizes whose forward
 * scratch exceeds it return SLM_ERR_WORKSPACE before anything is enqueued (at V = 128256
 * that is N > ~65,000 rows for SLM_CE and N > ~26,000 rows for the other kinds).
 *   device_flags  int [1] device memory or NULL: receives the device status bits of this
 *                 call (0 = none; 1 = a CE label outside [0, V); 2 = a wait ran out of time).
 * The first call on each device looks up the array's device address (and may load the
 * library's device code), so make it before any stream capture.  The address is kept per
 * device and CUDA context: after the context is torn down and re-created (cudaDeviceReset),
 * the next call looks it up again, and that call too should come before any capture.  Every call shares the one
 * array: calls that overlap on the GPU race and must be serialised by the caller.  Nothing
 * is allocated.  The backward still takes a caller workspace (slm_loss_bwd). */
SLM_API int slm_loss_fwd_noalloc(int kind, const void* Hq, const void* Hp, const void* W,
                                 const int32_t* labels, int32_t ignore_index,
                                 int64_t N, int64_t d, int64_t V,
                                 float* loss_tok, float* alpha_tok, double* loss_sum,
                                 int64_t* n_valid, float* loss_mean, float* stats,
                                 int* device_flags, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SLM_H_ */
