// Launch accounting and GEMM timing (the C interface is in include/sbp_profile.h).
// While profiling is on, each GEMM / attention call is bracketed by two CUDA events on its own
// stream; sbp_profile_end() synchronises, sums the elapsed times per kernel kind, measures the
// union of each kind's intervals (calls on side streams overlap) and recycles the events.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "sbp_internal.cuh"
#include "sbp_profile.h"

namespace sbp {

namespace {
std::atomic<long long> g_launches{0};
std::atomic<bool> g_on{false};
std::mutex g_mu;
struct Mark {
  int kind;
  cudaEvent_t a, b;
};
std::vector<Mark> g_marks;
std::vector<cudaEvent_t> g_pool;
thread_local cudaEvent_t tl_open = nullptr;

cudaEvent_t get_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

void prof_count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
bool prof_enabled() { return g_on.load(std::memory_order_relaxed); }

void prof_mark_begin(int kind, cudaStream_t st) {
  (void)kind;
  if (!prof_enabled()) return;
  std::lock_guard<std::mutex> lk(g_mu);
  tl_open = get_event();
  if (tl_open) cudaEventRecord(tl_open, st);
}

void prof_mark_end(int kind, cudaStream_t st) {
  if (!prof_enabled() || !tl_open) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t b = get_event();
  if (!b) return;
  cudaEventRecord(b, st);
  g_marks.push_back({kind, tl_open, b});
  tl_open = nullptr;
}

}  // namespace sbp

using namespace sbp;

extern "C" {

long long sbp_launch_count(void) { return g_launches.load(); }

sbp_status sbp_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_marks.clear();
  g_on.store(true);
  return SBP_OK;
}

sbp_status sbp_profile_end(sbp_profile* out) {
  g_on.store(false);
  std::lock_guard<std::mutex> lk(g_mu);
  if (out) {
    for (int k = 0; k < PROF_KINDS; ++k) {
      out->launches[k] = 0;
      out->ms[k] = 0.0;
      out->busy_ms[k] = 0.0;
    }
  }
  sbp_status st = SBP_OK;
  // intervals on one time axis: milliseconds from the first mark's start (may be negative
  // for a call on another stream that started earlier)
  std::vector<std::pair<double, double>> iv[PROF_KINDS];
  for (const Mark& m : g_marks) {
    float ms = 0.f, t0 = 0.f;
    if (cudaEventSynchronize(m.b) != cudaSuccess ||
        cudaEventElapsedTime(&ms, m.a, m.b) != cudaSuccess ||
        cudaEventElapsedTime(&t0, g_marks.front().a, m.a) != cudaSuccess)
      st = SBP_ERR_CUDA;
    if (out && m.kind >= 0 && m.kind < PROF_KINDS) {
      out->launches[m.kind] += 1;
      out->ms[m.kind] += ms;
      iv[m.kind].push_back({(double)t0, (double)t0 + (double)ms});
    }
  }
  if (out) {
    for (int k = 0; k < PROF_KINDS; ++k) {
      std::sort(iv[k].begin(), iv[k].end());
      double busy = 0.0, lo = 0.0, hi = 0.0;
      bool open = false;
      for (const auto& x : iv[k]) {
        if (open && x.first <= hi) {
          hi = std::max(hi, x.second);
          continue;
        }
        if (open) busy += hi - lo;
        lo = x.first;
        hi = x.second;
        open = true;
      }
      if (open) busy += hi - lo;
      out->busy_ms[k] = busy;
    }
  }
  for (const Mark& m : g_marks) {
    g_pool.push_back(m.a);
    g_pool.push_back(m.b);
  }
  g_marks.clear();
  return st;
}

}  // extern "C"
