/*
 * sbp_dpo.h -- the DPO objective on top of the streamed backward.
 *
 * [paper] Abstract and [skill] Core Concept ("Multiple Objectives") / Practical Guidance ("Loss
 * Objectives") name DPO among the objectives StreamBP serves and give no formula.  This library
 * takes the standard DPO loss on P pairs of sequences,
 *     loss = (1/P) sum_p -log sigmoid(beta * Delta_p),
 *     Delta_p = (logp(chosen_p) - ref(chosen_p)) - (logp(rejected_p) - ref(rejected_p)),
 * where logp(seq) = sum over the response tokens of log p(y_t) = -CE_t and ref(.) are the
 * reference model's sequence log-probabilities (an input).  DPO needs the sequence
 * log-probabilities before any gradient can be formed, so a step is: the streamed LM-head
 * forward (per-token CE), sbp_dpo_token_weights (loss and per-token loss weights
 * w_t = d loss / d CE_t), then the streamed backward (sbp_lmhead_ce_backward_stream and the
 * layers) unchanged, with those weights.  Since the loss depends on the network only through
 * the CE_t, that backward is the exact DPO gradient.
 *
 * Sequence layout: 2P sequences of seq_len tokens, [chosen_0, rejected_0, chosen_1, ...],
 * flattened row-major (token t of sequence b is row b * seq_len + t).
 */
#ifndef SBP_DPO_H_
#define SBP_DPO_H_

#include "sbp.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Streamed LM-head forward: per-token cross-entropy CE_t = logsumexp(h_t W^T) - (h_t W^T)[y_t]
 * for every row with loss_weights[t] != 0 (0 elsewhere), chunk by chunk as in
 * sbp_lmhead_ce_backward_stream (same arguments, same workspace size, logits never leave
 * on-chip memory).
 *   token_ce   device [n_tokens] fp32, overwritten
 *   loss_out   device fp32 scalar or NULL; if given, overwritten with sum_t w_t CE_t
 * Errors as sbp_lmhead_ce_backward_stream.
 */
sbp_status sbp_lmhead_ce_forward_stream(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                        int num_chunks, sbp_dtype dt, const void* hidden_states,
                                        const void* weight, const int32_t* targets,
                                        const float* loss_weights, float* token_ce,
                                        float* loss_out, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* Workspace bytes of sbp_dpo_token_weights (0 if n_pairs < 1). */
size_t sbp_dpo_workspace_size(int64_t n_pairs);

/*
 * DPO loss and per-token loss weights from per-token CE.
 *   n_pairs        P >= 1
 *   seq_len        tokens per sequence >= 1
 *   token_ce       device [2P * seq_len] fp32 (e.g. from sbp_lmhead_ce_forward_stream)
 *   response_mask  device [2P * seq_len] fp32, 1 on the tokens whose log-probability counts
 *                  (the response predictions), 0 elsewhere (other values weight the token)
 *   ref_logp       device [2P] fp32, the reference model's sequence log-probabilities
 *   beta           DPO temperature (> 0)
 *   loss_out       device fp32 scalar, overwritten with the DPO loss
 *   seq_logp       device [2P] fp32 or NULL; if given, overwritten with logp(seq)
 *   weights        device [2P * seq_len] fp32, overwritten with
 *                  w = response_mask * (+1 chosen / -1 rejected) * beta * sigmoid(-beta Delta_p) / P
 *   workspace      device, >= sbp_dpo_workspace_size(n_pairs) bytes, 256-byte aligned
 * Sums are taken in a fixed order (deterministic).  Returns SBP_ERR_INVALID_ARG for NULL
 * required pointers, non-positive sizes or beta, SBP_ERR_WORKSPACE for a short workspace.
 */
sbp_status sbp_dpo_token_weights(int64_t n_pairs, int64_t seq_len, const float* token_ce,
                                 const float* response_mask, const float* ref_logp, float beta,
                                 float* loss_out, float* seq_logp, float* weights,
                                 void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SBP_DPO_H_ */
