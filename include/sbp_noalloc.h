/*
 * sbp_noalloc.h -- an LM-head cross-entropy backward for callers that cannot allocate device
 * memory.  The paper has no counterpart: this is a deployment convenience of this library.
 *
 * Who needs it: code that may not call cudaMalloc (or any allocating routine) where it runs the
 * backward -- a plug-in inside a framework that owns all device memory through its own pool and
 * hands it only tensors, or an embedded runtime with a memory budget fixed in advance.  Such a
 * caller can pass inputs and outputs but no workspace.
 */
#ifndef SBP_NOALLOC_H_
#define SBP_NOALLOC_H_

#include "sbp.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Same computation, arguments, layouts and accumulate rules as sbp_lmhead_ce_backward_stream,
 * without the workspace: the scratch is a 32 MiB array inside the library (a static device
 * array; a GPU holds it from the first call made on it until the process exits).  Nothing is
 * allocated: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 *   - Size limit: sizes whose sbp_lmhead_ce_workspace_size() exceeds 32 MiB are rejected with
 *     SBP_ERR_WORKSPACE and a message in sbp_last_error(); raise num_chunks to shrink the
 *     per-chunk scratch (it scales with n_tokens / num_chunks), or use the workspace entry.
 *   - First call on a device does one-time set-up there, with that device current: it looks
 *     up the device address of the scratch, which also makes the CUDA runtime load the module
 *     holding the array (the driver reserves its 32 MiB at that moment, not when the library
 *     is opened), and, like the first call of any libsbp entry point on a device, it creates
 *     the library's side streams and events.
 *   - Invalid sizes (n_tokens, hidden or vocab <= 0, num_chunks outside [1, n_tokens]) return
 *     SBP_ERR_INVALID_ARG before any device work or set-up.
 *   - Shared scratch: every call on a device uses the same scratch, which keeps the last call's
 *     contents; the call clears what must start at zero.  Calls whose GPU work overlaps
 *     (different streams or threads) race on it -- serialise them on one stream.
 *   - Device-side errors (a target outside [0, vocab) with a nonzero weight) are handled as in
 *     the workspace entry (the row is skipped) but cannot be read back through this call.
 */
sbp_status sbp_lmhead_ce_backward_noalloc(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                          int num_chunks, sbp_dtype dt,
                                          const void* hidden_states, const void* weight,
                                          const int32_t* targets, const float* loss_weights,
                                          float* loss_out, float* d_hidden, float* d_weight,
                                          void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SBP_NOALLOC_H_ */
