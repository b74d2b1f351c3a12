// Side streams: per device, a few streams on which the library runs independent work of one
// call next to the caller's stream.  Work is forked from and joined back into the caller's
// stream with events, so a call stays ordered on the caller's stream.  Created on the first
// call on a device, kept until exit.
#include <mutex>

#include "sbp_internal.cuh"

namespace sbp {

namespace {
std::mutex g_mu;
SidePool g_pools[64];
}  // namespace

SidePool* side_pool() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  SidePool& P = g_pools[dev];
  if (!P.ok) {
    bool good = true;
    for (auto& st : P.s) good &= cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) == cudaSuccess;
    for (auto& e : P.ev) good &= cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    P.ok = good;
    if (!good) return nullptr;
  }
  return &P;
}

}  // namespace sbp
