// DPO objective on top of the streamed backward (the C interface is in include/sbp_dpo.h):
// sequence log-probabilities from per-token cross-entropy, the loss
// (1/P) sum_p -log sigmoid(beta Delta_p) and the per-token loss weights
// w_t = d loss / d CE_t = mask_t * (+1 chosen / -1 rejected) * beta * sigmoid(-beta Delta_p) / P.
// The pages ("StreamBP: Memory-Efficient Exact Backpropagation ...", Abstract; "StreamBP:
// Memory-Efficient Backpropagation", Core Concept and Practical Guidance, Loss Objectives) name
// DPO among the supported objectives; the formula is the standard DPO loss.
// Every sum is taken in a fixed order, so the results are deterministic.
#include "sbp_internal.cuh"

namespace sbp {

namespace {

__device__ __forceinline__ float softplus(float x) {     // log(1 + e^x), stable
  return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid(float x) {      // stable on both sides
  if (x >= 0.f) return 1.f / (1.f + expf(-x));
  const float e = expf(x);
  return e / (1.f + e);
}
__device__ __forceinline__ float pair_delta(const float* logp, const float* ref, int64_t p) {
  return (logp[2 * p] - ref[2 * p]) - (logp[2 * p + 1] - ref[2 * p + 1]);
}

// one CTA per sequence: logp[b] = -sum_t mask * ce
__global__ void __launch_bounds__(256) dpo_seq_logp_kernel(int64_t T, const float* __restrict__ ce,
                                                           const float* __restrict__ mask,
                                                           float* __restrict__ logp) {
  __shared__ float red[8];
  const int64_t b = blockIdx.x;
  const float* c = ce + b * T;
  const float* m = mask + b * T;
  float s = 0.f;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) s = fmaf(m[t], c[t], s);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int i = 0; i < 8; ++i) tot += red[i];
    logp[b] = -tot;
  }
}

__global__ void dpo_terms_kernel(int64_t P, const float* __restrict__ logp,
                                 const float* __restrict__ ref, float beta,
                                 float* __restrict__ terms) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= P) return;
  terms[p] = softplus(-beta * pair_delta(logp, ref, p)) / (float)P;
}

// deterministic sum of the P loss terms with one CTA
__global__ void __launch_bounds__(1024) dpo_loss_kernel(int64_t P, const float* __restrict__ terms,
                                                        float* __restrict__ loss) {
  __shared__ float red[32];
  float s = 0.f;
  for (int64_t p = threadIdx.x; p < P; p += blockDim.x) s += terms[p];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    loss[0] = t;
  }
}

// grid (ceil(T / 256), 2P)
__global__ void dpo_token_weights_kernel(int64_t P, int64_t T, const float* __restrict__ mask,
                                         const float* __restrict__ logp,
                                         const float* __restrict__ ref, float beta,
                                         float* __restrict__ w) {
  const int64_t b = blockIdx.y;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int64_t p = b >> 1;
  const float coef = beta * sigmoid(-beta * pair_delta(logp, ref, p)) / (float)P;
  const float sign = (b & 1) ? -1.f : 1.f;
  w[b * T + t] = mask[b * T + t] * sign * coef;
}

}  // namespace

cudaError_t dpo_weights(int64_t P, int64_t T, const float* token_ce, const float* mask,
                        const float* ref_logp, float beta, float* seq_logp, float* terms,
                        float* loss, float* weights, cudaStream_t st) {
  launch(dpo_seq_logp_kernel, (unsigned)(2 * P), 256, 0, st, T, token_ce, mask, seq_logp);
  launch(dpo_terms_kernel, (unsigned)((P + 255) / 256), 256, 0, st, P, seq_logp, ref_logp, beta,
         terms);
  launch(dpo_loss_kernel, 1, 1024, 0, st, P, terms, loss);
  launch(dpo_token_weights_kernel, dim3((unsigned)((T + 255) / 256), (unsigned)(2 * P)), dim3(256),
         0, st, P, T, mask, seq_logp, ref_logp, beta, weights);
  return cudaGetLastError();
}

}  // namespace sbp
