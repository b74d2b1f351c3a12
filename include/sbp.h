/*
 * sbp.h -- C ABI of libsbp: StreamBP's streamed exact backward on one B200 (sm_100a).
 *
 * Sources (web pages on StreamBP, arXiv 2506.03077):
 *   [skill] "StreamBP: Memory-Efficient Backpropagation" (skillsmp.com skill page)
 *   [paper] "StreamBP: Memory-Efficient Exact Backpropagation for Long Sequence Training of
 *           LLMs" (tomesphere.com), Abstract.
 *
 * What the library computes.  The backward pass of a causal decoder layer and of the LM-head
 * cross-entropy, split into D chunks along the sequence ([skill] Core Concept; [paper]
 * Abstract: a layer-wise linear decomposition of the chain rule along the sequence).  For each
 * chunk the forward is recomputed and backpropagated against the keys/values of its causal
 * prefix only ([skill] Architecture Overview, Causal Structure Exploitation); weight gradients
 * and dK/dV accumulate across chunks in fp32.  The result is the plain (unchunked) backward up
 * to fp32 summation order ([skill] Architecture Overview, Exact Gradients).
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller allocates every device buffer, including the workspace; the
 *     library allocates no device memory and never synchronises the host.  All work is queued
 *     on `stream` (a cudaStream_t passed as void*; NULL = legacy default stream).
 *   - Layout: row-major, tokens outer: activations are [batch, seq_len, features] (contiguous);
 *     weights use the nn.Linear layout [out_features, in_features].
 *   - dtype: SBP_F32 = fp32 operands and arithmetic (no TF32); SBP_BF16 = bf16 operands with
 *     fp32 accumulation.  Gradients, loss and upstream gradients are always fp32.
 *   - Accumulation: weight gradients are ACCUMULATED (+=) so that micro-batch gradient
 *     accumulation composes with chunking ([skill] Practical Guidance, Gradient Accumulation);
 *     the caller zeroes them.  Activation gradients (dx, d_hidden) and the loss are
 *     overwritten.
 *   - Errors: arguments are checked on the host before anything is queued; a bad argument
 *     returns a status and queues nothing.  Errors found on the device (a target outside
 *     [0, vocab) with a nonzero loss weight) set a status word inside the workspace that
 *     sbp_get_device_status() reads.  sbp_last_error() gives a message for the calling thread.
 *   - Alignment: every device pointer must be 16-byte aligned.
 */
#ifndef SBP_H_
#define SBP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SBP_OK = 0,
  SBP_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer, D > T, ...   */
  SBP_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. odd head_dim)            */
  SBP_ERR_WORKSPACE = 3,      /* workspace smaller than the *_workspace_size() answer     */
  SBP_ERR_CUDA = 4,           /* a CUDA runtime call failed; see sbp_last_error()         */
  SBP_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait gave up                       */
  SBP_ERR_BAD_TARGET = 6      /* device: target outside [0, vocab) with loss weight != 0  */
} sbp_status;

typedef enum { SBP_F32 = 0, SBP_BF16 = 1 } sbp_dtype;

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* sbp_last_error(void);

/* Library version string. */
const char* sbp_version(void);

/*
 * Chunk decomposition ([skill] Implementation, decompose_sequence): chunk = seq_len / D
 * (integer division); chunk i = [i*chunk, (i+1)*chunk), the last chunk ends at seq_len.
 * Writes num_chunks + 1 boundaries into the HOST array `bounds` (bounds[0] = 0,
 * bounds[D] = seq_len).  Returns SBP_ERR_INVALID_ARG unless 1 <= num_chunks <= seq_len.
 */
sbp_status sbp_chunk_bounds(int64_t seq_len, int num_chunks, int64_t* bounds);

/*
 * Reads (and clears) the device status word kept at the start of a workspace that a previous
 * call used.  Synchronises `stream`.  Returns SBP_OK, SBP_ERR_BAD_TARGET or
 * SBP_ERR_DEVICE_TIMEOUT, or SBP_ERR_CUDA if the stream itself failed.
 */
sbp_status sbp_get_device_status(void* workspace, void* stream);

/* ------------------------------------------------------------------------------------------
 * LM head + cross-entropy, streamed over chunks of rows.
 *
 * [skill] Implementation (chunked cross-entropy gradient): per row t, d loss / d logits_t =
 * w_t * (softmax(logits_t) - onehot(y_t)).  With logits = H W^T and
 *     loss = sum_t w_t * (logsumexp(logits_t) - logits_t[y_t]),
 * this computes loss, d_hidden = G W and d_weight += G^T H for G = d loss / d logits, one chunk
 * of n_tokens / num_chunks rows at a time.  The objective's normaliser (1 / #loss tokens for
 * mean-CE SFT, A_s / #tokens for GRPO) is folded into w by the caller, so the result does not
 * depend on num_chunks.  Rows with w_t == 0 are skipped (their d_hidden row is 0).  Logits are
 * formed tile by tile in on-chip memory; the only logit-sized intermediates are the bf16/fp32
 * gradient blocks G of one vocabulary block (<= rows_per_chunk x 16384 elements, two of them so
 * that one is formed while the products consume the other) in the workspace.
 *
 *   n_tokens       number of rows N (all sequences of a batch flattened)
 *   hidden         d (multiple of 8)
 *   vocab          V
 *   num_chunks     D, 1 <= D <= N
 *   dt             operand dtype of hidden_states and weight
 *   hidden_states  device [N, d], dt
 *   weight         device [V, d], dt (nn.Linear layout of the LM head)
 *   targets        device [N] int32; a row with w_t != 0 needs 0 <= y_t < V, else the device
 *                  status becomes SBP_ERR_BAD_TARGET and the row is treated as w_t = 0
 *   loss_weights   device [N] fp32 (may be negative, e.g. GRPO advantages)
 *   loss_out       device fp32 scalar, overwritten with sum_t w_t CE_t
 *   d_hidden       device [N, d] fp32, overwritten
 *   d_weight       device [V, d] fp32, accumulated (+=)
 *   workspace      device, >= sbp_lmhead_ce_workspace_size(...) bytes, 256-byte aligned
 * ------------------------------------------------------------------------------------------ */
size_t sbp_lmhead_ce_workspace_size(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                    int num_chunks, sbp_dtype dt);

sbp_status sbp_lmhead_ce_backward_stream(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                         int num_chunks, sbp_dtype dt,
                                         const void* hidden_states, const void* weight,
                                         const int32_t* targets, const float* loss_weights,
                                         float* loss_out, float* d_hidden, float* d_weight,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * The same backward with the per-token inputs in HOST memory: hidden_states_host [N, d] (dt),
 * targets_host [N] and loss_weights_host [N] are host pointers (page-locked for the copies to
 * overlap the computation; pageable memory works but serialises).  Each chunk's rows are
 * copied into one of two staging blocks of the workspace on a library side stream while the
 * previous chunk computes, so only the first chunk's copy is exposed.  weight, loss_out,
 * d_hidden, d_weight and workspace are device memory as above; the results are identical to
 * sbp_lmhead_ce_backward_stream's.  The host buffers must stay valid and unchanged until
 * `stream` has passed this call.  Workspace: sbp_lmhead_ce_workspace_size_host(...) bytes
 * (the device workspace plus two staging blocks of rows_per_chunk rows).
 */
size_t sbp_lmhead_ce_workspace_size_host(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                         int num_chunks, sbp_dtype dt);
sbp_status sbp_lmhead_ce_backward_stream_host(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                              int num_chunks, sbp_dtype dt,
                                              const void* hidden_states_host, const void* weight,
                                              const int32_t* targets_host,
                                              const float* loss_weights_host, float* loss_out,
                                              float* d_hidden, float* d_weight, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * Causal decoder layer (pre-norm Llama/Qwen block):
 *   n1 = RMSNorm(x; ln1_g);  q,k,v = n1 W_{q,k,v}^T (+ b_{q,k,v});  RoPE(q), RoPE(k)
 *   (rotate-half, absolute positions, inv_freq_j = rope_theta^(-2j/head_dim));
 *   a = causal softmax(q k^T / sqrt(head_dim)) v with GQA (query head h reads KV head
 *   h / (n_heads / n_kv_heads));  h = x + a W_o^T;  n2 = RMSNorm(h; ln2_g);
 *   y = h + (silu(n2 W_gate^T) * (n2 W_up^T)) W_down^T.
 * ------------------------------------------------------------------------------------------ */
typedef struct {
  int64_t batch, seq_len, d_model, n_heads, n_kv_heads, head_dim, ffn;
  float rms_eps;
  double rope_theta;
  int dtype;      /* sbp_dtype of x, y and every weight */
  int num_chunks; /* D, 1 <= D <= seq_len */
} sbp_layer_cfg;

typedef struct {  /* device pointers, dtype = cfg.dtype; bq/bk/bv may be NULL (no bias) */
  const void *ln1_g, *wq, *wk, *wv, *bq, *bk, *bv, *wo, *ln2_g, *w_gate, *w_up, *w_down;
} sbp_layer_weights;

typedef struct {  /* device fp32, ACCUMULATED; bq/bk/bv must be non-NULL iff the bias is */
  float *ln1_g, *wq, *wk, *wv, *bq, *bk, *bv, *wo, *ln2_g, *w_gate, *w_up, *w_down;
} sbp_layer_grads;

/* Workspace bytes for the backward (and, with the same size, the forward) of one layer. */
size_t sbp_decoder_layer_workspace_size(const sbp_layer_cfg* cfg);

/*
 * Streamed exact backward of one decoder layer ([skill] Implementation, the streamed layer
 * backward with gradient accumulation; Architecture Overview, Layer-Wise Application).
 * For each chunk i = [s_i, e_i) in order: recompute the chunk's forward with K/V of the prefix
 * [0, e_i) (appended chunk by chunk), backpropagate dy[:, s_i:e_i), add weight gradients and
 * the prefix dK/dV (fp32).  After the loop the K/V projections are backpropagated chunk by
 * chunk (RMSNorm's backward is linear in its upstream gradient, so this part may be applied
 * separately and added).
 *   x   device [batch, seq_len, d_model], dtype
 *   dy  device [batch, seq_len, d_model] fp32 (upstream gradient)
 *   dx  device [batch, seq_len, d_model] fp32, overwritten
 * Requirements: n_heads % n_kv_heads == 0; head_dim even and <= 256; d_model, n_heads*head_dim,
 * n_kv_heads*head_dim and ffn multiples of 8 for SBP_BF16.
 */
sbp_status sbp_decoder_layer_backward_stream(const sbp_layer_cfg* cfg,
                                             const sbp_layer_weights* w, const void* x,
                                             const float* dy, float* dx,
                                             const sbp_layer_grads* grads, void* workspace,
                                             size_t workspace_bytes, void* stream);

/*
 * The same backward with the chunks visited in reverse order (the pages fix the per-chunk
 * computation, not the order of the chunk loop: [skill] Implementation, the streamed layer
 * backward with gradient accumulation).  The K/V prefix of the whole sequence is computed
 * first (RMSNorm-1 and the K/V projections, chunk by chunk); then chunks D-1 .. 0 are
 * recomputed and backpropagated.  When chunk i is reached, every chunk whose queries attend to
 * its keys has been done, so its dK/dV rows are final and its K/V projection backward runs in
 * the same iteration, on the RMSNorm-1 rows already computed for its forward: no pass after
 * the loop, and one RMSNorm-1 backward per chunk.  Arguments, layouts, workspace size
 * (sbp_decoder_layer_workspace_size), accumulation and errors are those of
 * sbp_decoder_layer_backward_stream; the results are equal up to the order of fp32 sums.
 */
sbp_status sbp_decoder_layer_backward_stream_reverse(const sbp_layer_cfg* cfg,
                                                     const sbp_layer_weights* w, const void* x,
                                                     const float* dy, float* dx,
                                                     const sbp_layer_grads* grads,
                                                     void* workspace, size_t workspace_bytes,
                                                     void* stream);

/*
 * Forward of one decoder layer, chunk by chunk (activation memory O(T/D) apart from the
 * O(T * n_kv_heads * head_dim) K/V prefix).  Used to produce the layer-input checkpoints of a
 * stack ([skill] Core Concept: StreamBP is compared with, and sits on, gradient
 * checkpointing).  y: device [batch, seq_len, d_model], dtype, overwritten.
 */
sbp_status sbp_decoder_layer_forward_stream(const sbp_layer_cfg* cfg,
                                            const sbp_layer_weights* w, const void* x, void* y,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream);

/* ------------------------------------------------------------------------------------------
 * Support calls for composing a stack (embedding -> layers -> final norm -> LM head).
 * ------------------------------------------------------------------------------------------ */

/* y[r] = x[r] / sqrt(mean(x[r]^2) + eps) * g; rstd[r] = that reciprocal (fp32, may be NULL).
 * x, g, y: dtype; rows x cols. */
sbp_status sbp_rmsnorm_forward(int64_t rows, int64_t cols, sbp_dtype dt, float eps,
                               const void* x, const void* g, void* y, float* rstd,
                               void* stream);

/* Backward of sbp_rmsnorm_forward given its rstd: dx = (accumulate ? dx : 0) +
 * rstd * (g * dy - xhat * mean(xhat * g * dy)); dg += sum over rows of dy * xhat.
 * dy, dx, dg fp32; x, g dtype.  Needs `workspace` of sbp_rmsnorm_backward_workspace_size(). */
size_t sbp_rmsnorm_backward_workspace_size(int64_t rows, int64_t cols);
sbp_status sbp_rmsnorm_backward(int64_t rows, int64_t cols, sbp_dtype dt, const void* x,
                                const void* g, const float* rstd, const float* dy, float* dx,
                                int accumulate, float* dg, void* workspace,
                                size_t workspace_bytes, void* stream);

/* y[r] = table[ids[r]]; table [vocab, cols] dtype; ids int32 [rows] in [0, vocab). */
sbp_status sbp_embedding_forward(int64_t rows, int64_t cols, int64_t vocab, sbp_dtype dt,
                                 const int32_t* ids, const void* table, void* y, void* stream);

/* d_table[v] += sum of dy[r] over rows with ids[r] == v, in row order (deterministic).
 * Needs workspace of sbp_embedding_backward_workspace_size(). */
size_t sbp_embedding_backward_workspace_size(int64_t rows, int64_t vocab);
sbp_status sbp_embedding_backward(int64_t rows, int64_t cols, int64_t vocab,
                                  const int32_t* ids, const float* dy, float* d_table,
                                  void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SBP_H_ */
