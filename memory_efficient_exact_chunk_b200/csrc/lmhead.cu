// LM-head cross-entropy helpers around the GEMMs: loss-row compaction and gather, the
// log-sum-exp combine with the loss reduction.  The logits themselves only ever exist inside
// GEMM tiles (see the EPI_LSE / EPI_CEGRAD epilogues).
#include "sbp_internal.cuh"

namespace sbp {

namespace {

// Stable compaction with one CTA: thread i owns the contiguous row range [b_i, e_i).
__global__ void __launch_bounds__(1024)
ce_compact_kernel(int64_t s, int64_t e, int64_t V, const int* __restrict__ tgt,
                  const float* __restrict__ w, int* __restrict__ idx, int* __restrict__ count,
                  int* __restrict__ status) {
  __shared__ int part[1024];
  const int64_t n = e - s;
  const int64_t per = (n + blockDim.x - 1) / blockDim.x;
  const int64_t b = s + threadIdx.x * per;
  const int64_t en = imin(e, b + per);
  int c = 0;
  bool bad = false;
  for (int64_t r = b; r < en; ++r) {
    if (w[r] != 0.f) {
      const int y = tgt[r];
      if (y >= 0 && (int64_t)y < V) ++c; else bad = true;
    }
  }
  if (bad) atomicExch(status, DEV_BAD_TARGET);
  part[threadIdx.x] = c;
  __syncthreads();
  // inclusive scan (Hillis-Steele)
  for (int o = 1; o < (int)blockDim.x; o <<= 1) {
    const int v = (threadIdx.x >= (unsigned)o) ? part[threadIdx.x - o] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int pos = part[threadIdx.x] - c;
  for (int64_t r = b; r < en; ++r) {
    if (w[r] != 0.f) {
      const int y = tgt[r];
      if (y >= 0 && (int64_t)y < V) idx[pos++] = (int)r;
    }
  }
  if (threadIdx.x == blockDim.x - 1) count[0] = part[threadIdx.x];
}

__global__ void ce_gather_kernel(int64_t d, int dt, const void* __restrict__ h,
                                 const int* __restrict__ idx, const int* __restrict__ count,
                                 const int* __restrict__ tgt, const float* __restrict__ w,
                                 void* __restrict__ hc, int* __restrict__ yc,
                                 float* __restrict__ wc, float* __restrict__ zy,
                                 float* __restrict__ lse) {
  const int64_t r = blockIdx.x;
  const int n = count[0];
  const bool valid = r < n;
  const int64_t src = valid ? (int64_t)idx[r] : 0;
  if (dt == DT_BF16) {
    const __nv_bfloat16* hs = static_cast<const __nv_bfloat16*>(h) + src * d;
    __nv_bfloat16* hd = static_cast<__nv_bfloat16*>(hc) + r * d;
    for (int64_t c = threadIdx.x; c < d; c += blockDim.x)
      hd[c] = valid ? hs[c] : __float2bfloat16_rn(0.f);
  } else {
    const float* hs = static_cast<const float*>(h) + src * d;
    float* hd = static_cast<float*>(hc) + r * d;
    for (int64_t c = threadIdx.x; c < d; c += blockDim.x) hd[c] = valid ? hs[c] : 0.f;
  }
  if (threadIdx.x == 0) {
    yc[r] = valid ? tgt[src] : -1;
    wc[r] = valid ? w[src] : 0.f;
    zy[r] = 0.f;
    lse[r] = 0.f;
  }
}

// one warp per row: combine the per-tile (max, sum-exp) pairs
__global__ void ce_lse_kernel(int64_t Rmax, int64_t tiles, const float* __restrict__ pmax,
                              const float* __restrict__ psum, int64_t pld,
                              const int* __restrict__ count, const float* __restrict__ wc,
                              const float* __restrict__ zy, float* __restrict__ lse,
                              float* __restrict__ row_loss) {
  const int lane = threadIdx.x & 31;
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (r >= Rmax) return;
  if (r >= count[0]) {
    if (lane == 0) row_loss[r] = 0.f;
    return;
  }
  float m = -INFINITY;
  for (int64_t j = lane; j < tiles; j += 32) m = fmaxf(m, pmax[r * pld + j]);
  m = warp_max(m);
  float sum = 0.f;
  for (int64_t j = lane; j < tiles; j += 32) sum += psum[r * pld + j] * expf(pmax[r * pld + j] - m);
  sum = warp_sum(sum);
  if (lane == 0) {
    const float l = m + logf(sum);
    lse[r] = l;
    row_loss[r] = wc[r] * (l - zy[r]);
  }
}

// deterministic sum of row_loss[0 .. count) with one CTA
__global__ void ce_loss_kernel(const int* __restrict__ count, const float* __restrict__ row_loss,
                               float* __restrict__ loss, int first) {
  __shared__ float red[32];
  const int n = count[0];
  float s = 0.f;
  for (int r = threadIdx.x; r < n; r += blockDim.x) s += row_loss[r];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    loss[0] = first ? t : loss[0] + t;
  }
}

__global__ void ce_token_scatter_kernel(int64_t Rmax, const int* __restrict__ idx,
                                        const int* __restrict__ count,
                                        const float* __restrict__ lse,
                                        const float* __restrict__ zy, float* __restrict__ token_ce) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= Rmax || r >= count[0]) return;
  token_ce[idx[r]] = lse[r] - zy[r];
}

}  // namespace

cudaError_t ce_token_scatter(int64_t s, int64_t e, int64_t Rmax, const int* idx, const int* count,
                             const float* lse, const float* zy, float* token_ce, cudaStream_t st) {
  if (e <= s) return cudaSuccess;
  cudaError_t err = cudaMemsetAsync(token_ce + s, 0, sizeof(float) * (size_t)(e - s), st);
  if (err != cudaSuccess || Rmax <= 0) return err;
  launch(ce_token_scatter_kernel, (unsigned)((Rmax + 255) / 256), 256, 0, st, Rmax, idx, count,
         lse, zy, token_ce);
  return cudaGetLastError();
}

cudaError_t ce_compact(int64_t s, int64_t e, int64_t V, const int* tgt, const float* w, int* idx,
                       int* count, int* status, cudaStream_t st) {
  launch(ce_compact_kernel, 1, 1024, 0, st, s, e, V, tgt, w, idx, count, status);
  return cudaGetLastError();
}

cudaError_t ce_gather(int64_t Rmax, int64_t d, int dt, const void* h, const int* idx,
                      const int* count, const int* tgt, const float* w, void* hc, int* yc,
                      float* wc, float* zy, float* lse, cudaStream_t st) {
  if (Rmax <= 0) return cudaSuccess;
  launch(ce_gather_kernel, (unsigned)Rmax, 256, 0, st, d, dt, h, idx, count, tgt, w, hc, yc, wc, zy,
                                                   lse);
  return cudaGetLastError();
}

cudaError_t ce_finish(int64_t Rmax, int64_t tiles, const float* pmax, const float* psum,
                      int64_t pld, const int* count, const float* wc, const float* zy,
                      float* lse, float* row_loss, float* loss, int first, cudaStream_t st) {
  if (Rmax > 0)
    launch(ce_lse_kernel, (unsigned)((Rmax * 32 + 255) / 256), 256, 0, st, 
        Rmax, tiles, pmax, psum, pld, count, wc, zy, lse, row_loss);
  launch(ce_loss_kernel, 1, 1024, 0, st, count, row_loss, loss, first);
  return cudaGetLastError();
}

cudaError_t zero_rows(int64_t s, int64_t e, int64_t d, float* dh, cudaStream_t st) {
  if (e <= s) return cudaSuccess;
  return cudaMemsetAsync(dh + s * d, 0, sizeof(float) * (size_t)(e - s) * d, st);
}

}  // namespace sbp
