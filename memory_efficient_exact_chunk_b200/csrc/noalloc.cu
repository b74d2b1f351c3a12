// sbp_lmhead_ce_backward_noalloc: the streamed LM-head cross-entropy backward for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point where they run
// the backward: code inside a framework that owns every device allocation through its own
// pool and hands plug-ins only tensors, or embedded runtimes with a fixed memory budget
// decided before they start.  Such callers can
// still pass their inputs and outputs, but not a workspace.  This entry point therefore keeps
// its scratch in a fixed-size array that belongs to the library: every GPU that loads the
// library holds kNoAllocScratchBytes of device memory for it until the process exits.
//
// The scratch is shared by every call on a device and keeps the last call's contents; the
// library clears what must start at zero (its status word) at the start of each call.  The
// array lives in this file's module, which the CUDA runtime loads lazily: the driver reserves
// its 32 MiB on a device at the first call there (the symbol lookup below), not when the
// library is opened.  Two
// calls whose GPU work overlaps (different streams, or different host threads) race on the
// scratch: serialise them on one stream.
#include <cstdio>
#include <mutex>

#include "sbp.h"
#include "sbp_internal.cuh"
#include "sbp_noalloc.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" {

sbp_status sbp_lmhead_ce_backward_noalloc(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                          int num_chunks, sbp_dtype dt,
                                          const void* hidden_states, const void* weight,
                                          const int32_t* targets, const float* loss_weights,
                                          float* loss_out, float* d_hidden, float* d_weight,
                                          void* stream) {
  const size_t need = sbp_lmhead_ce_workspace_size(n_tokens, hidden, vocab, num_chunks, dt);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "sbp_lmhead_ce_backward_noalloc: these sizes need %zu bytes of scratch but the "
             "library's static scratch holds %zu; use more chunks or the workspace entry point",
             need, kNoAllocScratchBytes);
    sbp::set_last_error(msg);
    return SBP_ERR_WORKSPACE;
  }
  if (need == 0) {
    // invalid sizes: reported before any device or symbol lookup, so that even a first call
    // on a device returns the argument error itself
    sbp::set_last_error(
        "sbp_lmhead_ce_backward_noalloc: invalid sizes (n_tokens, hidden and vocab must be "
        "positive and 1 <= num_chunks <= n_tokens)");
    return SBP_ERR_INVALID_ARG;
  }
  // Set-up, once per device, with that device current: the device address of the scratch.
  // (The array's name in host code is only a host-side stand-in, never a device address.)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    sbp::set_last_error("sbp_lmhead_ce_backward_noalloc: no usable current CUDA device");
    return SBP_ERR_CUDA;
  }
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        sbp::set_last_error("sbp_lmhead_ce_backward_noalloc: cudaGetSymbolAddress failed");
        return SBP_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    ptr = g_scratch_ptr[dev];
  }
  return sbp_lmhead_ce_backward_stream(n_tokens, hidden, vocab, num_chunks, dt, hidden_states,
                                       weight, targets, loss_weights, loss_out, d_hidden,
                                       d_weight, ptr, kNoAllocScratchBytes, stream);
}

}  // extern "C"
