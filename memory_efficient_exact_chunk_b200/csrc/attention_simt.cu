// Causal GQA attention of one query chunk against its key prefix, on the CUDA cores.
// One warp per (query row, head) for the forward and dQ; one warp per (key row, KV head) for
// dK/dV, which makes each dK/dV row single-owner (deterministic fp32 accumulation).
// Keys are visited in increasing order starting at 0, so a query's result does not depend on
// how the sequence was chunked.
#include "sbp_internal.cuh"

namespace sbp {

namespace {

constexpr int kMaxPerLane = 8;  // head_dim <= 256

template <typename T>
__device__ __forceinline__ void load_row(const T* p, int hd, int lane, float (&v)[kMaxPerLane]) {
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < hd) ? ld_f(p, e) : 0.f;
  }
}

template <typename T>
__device__ __forceinline__ float dot_row(const T* p, int hd, int lane,
                                         const float (&a)[kMaxPerLane]) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < hd) s = fmaf(a[i], ld_f(p, e), s);
  }
  return warp_sum(s);
}

template <typename T>
__global__ void attn_fwd_kernel(int64_t B, int64_t T_, int64_t Tc, int64_t s, int64_t H,
                                int64_t Hkv, int hd, const T* __restrict__ q,
                                const T* __restrict__ Kp, const T* __restrict__ Vp,
                                T* __restrict__ o, float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= B * Tc * H) return;
  const int64_t h = wid % H, r = wid / H;
  const int64_t b = r / Tc, t = s + r % Tc;
  const int64_t g = h / (H / Hkv);
  const float scale = rsqrtf((float)hd);
  float qv[kMaxPerLane], acc[kMaxPerLane];
  load_row(q + (r * H + h) * hd, hd, lane, qv);
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) { qv[i] *= scale; acc[i] = 0.f; }
  float m = -INFINITY, l = 0.f;
  for (int64_t u = 0; u <= t; ++u) {
    const int64_t kvo = ((b * T_ + u) * Hkv + g) * hd;
    const float sc = dot_row(Kp + kvo, hd, lane, qv);
    const float mn = fmaxf(m, sc);
    const float corr = expf(m - mn);
    const float p = expf(sc - mn);
    l = l * corr + p;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      const float vv = (e < hd) ? ld_f(Vp + kvo, e) : 0.f;
      acc[i] = acc[i] * corr + p * vv;
    }
    m = mn;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < hd) st_f(o + (r * H + h) * hd, e, acc[i] * inv);
  }
  if (lane == 0) lse[r * H + h] = m + logf(l);
}

// dQ and delta = rowsum(dO * O)
template <typename T>
__global__ void attn_bwd_dq_kernel(int64_t B, int64_t T_, int64_t Tc, int64_t s, int64_t H,
                                   int64_t Hkv, int hd, const T* __restrict__ q,
                                   const T* __restrict__ Kp, const T* __restrict__ Vp,
                                   const T* __restrict__ o, const T* __restrict__ dO,
                                   const float* __restrict__ lse, float* __restrict__ delta,
                                   float* __restrict__ dq) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= B * Tc * H) return;
  const int64_t h = wid % H, r = wid / H;
  const int64_t b = r / Tc, t = s + r % Tc;
  const int64_t g = h / (H / Hkv);
  const float scale = rsqrtf((float)hd);
  float qv[kMaxPerLane], dov[kMaxPerLane], ov[kMaxPerLane], acc[kMaxPerLane];
  const int64_t ro = (r * H + h) * hd;
  load_row(q + ro, hd, lane, qv);
  load_row(dO + ro, hd, lane, dov);
  load_row(o + ro, hd, lane, ov);
  float dl = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) { dl = fmaf(dov[i], ov[i], dl); qv[i] *= scale; acc[i] = 0.f; }
  dl = warp_sum(dl);
  const float L = lse[r * H + h];
  for (int64_t u = 0; u <= t; ++u) {
    const int64_t kvo = ((b * T_ + u) * Hkv + g) * hd;
    const float sc = dot_row(Kp + kvo, hd, lane, qv);
    const float dp = dot_row(Vp + kvo, hd, lane, dov);
    const float p = expf(sc - L);
    const float ds = p * (dp - dl);
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      const float kv = (e < hd) ? ld_f(Kp + kvo, e) : 0.f;
      acc[i] = fmaf(ds, kv, acc[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < hd) dq[ro + e] = acc[i] * scale;
  }
  if (lane == 0) delta[r * H + h] = dl;
}

// dK/dV for keys u in [0, s + Tc) of sequence b, KV head g: sum over the group's query heads
// and the chunk's queries t >= u.  Adds into the fp32 prefix accumulators.
template <typename T>
__global__ void attn_bwd_dkv_kernel(int64_t B, int64_t T_, int64_t Tc, int64_t s, int64_t H,
                                    int64_t Hkv, int hd, const T* __restrict__ q,
                                    const T* __restrict__ Kp, const T* __restrict__ Vp,
                                    const T* __restrict__ dO, const float* __restrict__ lse,
                                    const float* __restrict__ delta, float* __restrict__ dKp,
                                    float* __restrict__ dVp) {
  const int lane = threadIdx.x & 31;
  const int64_t e_ = s + Tc;
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= B * e_ * Hkv) return;
  const int64_t g = wid % Hkv;
  const int64_t u = (wid / Hkv) % e_;
  const int64_t b = wid / (Hkv * e_);
  const int64_t grp = H / Hkv;
  const float scale = rsqrtf((float)hd);
  const int64_t kvo = ((b * T_ + u) * Hkv + g) * hd;
  float kv[kMaxPerLane], vv[kMaxPerLane], dk[kMaxPerLane], dv[kMaxPerLane];
  load_row(Kp + kvo, hd, lane, kv);
  load_row(Vp + kvo, hd, lane, vv);
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) { kv[i] *= scale; dk[i] = 0.f; dv[i] = 0.f; }
  const int64_t t0 = u > s ? u : s;
  for (int64_t hh = g * grp; hh < (g + 1) * grp; ++hh) {
    for (int64_t t = t0; t < e_; ++t) {
      const int64_t r = b * Tc + (t - s);
      const int64_t ro = (r * H + hh) * hd;
      const float sc = dot_row(q + ro, hd, lane, kv);
      const float dp = dot_row(dO + ro, hd, lane, vv);
      const float p = expf(sc - lse[r * H + hh]);
      const float ds = p * (dp - delta[r * H + hh]);
#pragma unroll
      for (int i = 0; i < kMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        if (e < hd) {
          dv[i] = fmaf(p, ld_f(dO + ro, e), dv[i]);
          dk[i] = fmaf(ds, ld_f(q + ro, e), dk[i]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < hd) {
      dKp[kvo + e] += dk[i] * scale;
      dVp[kvo + e] += dv[i];
    }
  }
}

inline unsigned warps_blocks(int64_t warps) { return (unsigned)((warps * 32 + 255) / 256); }

}  // namespace

cudaError_t attn_fwd(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                     int64_t hd, int dt, const void* q, const void* Kp, const void* Vp, void* o,
                     float* lse, const AttnFwdSplit& sc, cudaStream_t st, int path) {
  const int64_t w = B * Tc * H;
  if (w <= 0) return cudaSuccess;
  if (path != 1 && attn_tc_supported(hd, dt, q, Kp, Vp, o)) {
    prof_mark_begin(PROF_ATTN_FWD, st);
    const cudaError_t e = attn_fwd_tc(B, T, Tc, s, H, Hkv, q, Kp, Vp, o, lse, sc, status_word(), st);
    prof_mark_end(PROF_ATTN_FWD, st);
    return e;
  }
  if (path == 2) return cudaErrorNotSupported;
  prof_mark_begin(PROF_ATTN_FWD, st);
  if (dt == DT_BF16)
    launch(attn_fwd_kernel<__nv_bfloat16>, warps_blocks(w), 256, 0, st, 
        B, T, Tc, s, H, Hkv, (int)hd, (const __nv_bfloat16*)q, (const __nv_bfloat16*)Kp,
        (const __nv_bfloat16*)Vp, (__nv_bfloat16*)o, lse);
  else
    launch(attn_fwd_kernel<float>, warps_blocks(w), 256, 0, st, 
        B, T, Tc, s, H, Hkv, (int)hd, (const float*)q, (const float*)Kp, (const float*)Vp,
        (float*)o, lse);
  prof_mark_end(PROF_ATTN_FWD, st);
  return cudaGetLastError();
}

template <typename T>
static void attn_bwd_launch(int64_t B, int64_t Tn, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                            int64_t hd, const void* q, const void* Kp, const void* Vp,
                            const void* o, const void* dO, const float* lse, float* delta,
                            float* dq, float* dKp, float* dVp, cudaStream_t st) {
  const int64_t w = B * Tc * H;
  const int64_t w2 = B * (s + Tc) * Hkv;
  launch(attn_bwd_dq_kernel<T>, warps_blocks(w), 256, 0, st, 
      B, Tn, Tc, s, H, Hkv, (int)hd, (const T*)q, (const T*)Kp, (const T*)Vp, (const T*)o,
      (const T*)dO, lse, delta, dq);
  launch(attn_bwd_dkv_kernel<T>, warps_blocks(w2), 256, 0, st, 
      B, Tn, Tc, s, H, Hkv, (int)hd, (const T*)q, (const T*)Kp, (const T*)Vp, (const T*)dO, lse,
      delta, dKp, dVp);
}

cudaError_t attn_bwd(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                     int64_t hd, int dt, const void* q, const void* Kp, const void* Vp,
                     const void* o, const void* dO, const float* lse, float* delta, float* dq,
                     float* dKp, float* dVp, cudaStream_t st, int path) {
  if (B * Tc * H <= 0) return cudaSuccess;
  if (path != 1 && attn_bwd_tc_supported(hd, dt, q, Kp, Vp, o, dO, dq)) {
    prof_mark_begin(PROF_ATTN_BWD, st);
    const cudaError_t e = attn_bwd_tc(B, T, Tc, s, H, Hkv, q, Kp, Vp, o, dO, lse, delta, dq, dKp,
                                      dVp, status_word(), st);
    prof_mark_end(PROF_ATTN_BWD, st);
    return e;
  }
  if (path == 2) return cudaErrorNotSupported;
  prof_mark_begin(PROF_ATTN_BWD, st);
  if (dt == DT_BF16)
    attn_bwd_launch<__nv_bfloat16>(B, T, Tc, s, H, Hkv, hd, q, Kp, Vp, o, dO, lse, delta, dq, dKp,
                                   dVp, st);
  else
    attn_bwd_launch<float>(B, T, Tc, s, H, Hkv, hd, q, Kp, Vp, o, dO, lse, delta, dq, dKp, dVp,
                           st);
  prof_mark_end(PROF_ATTN_BWD, st);
  return cudaGetLastError();
}

}  // namespace sbp
