// Generic strided GEMM on the CUDA cores (fp32 FFMA, no TF32).  It serves the fp32 path, any
// bf16 GEMM whose layout the tensor-core kernel does not take, and the fused cross-entropy
// epilogues.  Tile 64 x 64 x 16, 256 threads, 4 x 4 outputs per thread.
#include "sbp_internal.cuh"

namespace sbp {

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename TA, typename TB>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float St[BM][BN + 1];

  const int64_t M = g.dynM ? (int64_t)*g.dynM : g.M;
  const int64_t K = g.dynK ? (int64_t)*g.dynK : g.K;
  const int64_t N = g.N;
  const int64_t m0 = (int64_t)blockIdx.y * BM;
  const int64_t n0 = (int64_t)blockIdx.x * BN;
  if (m0 >= (g.epi == EPI_CEGRAD ? g.M : M)) return;
  if (K <= 0 && g.epi == EPI_ACC && !g.bias) return;     // C += 0: C stays as it is

  const TA* A = static_cast<const TA*>(g.A);
  const TB* B = static_cast<const TB*>(g.B);
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const bool a_kmajor = (g.sak == 1);
  const bool b_nmajor = (g.sbn == 1);

  float acc[4][4], tot[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = tot[i][j] = 0.f;

  for (int64_t k0 = 0; k0 < K; k0 += BK) {
    // A tile [BM x BK]
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int mm, kk;
      if (a_kmajor) { mm = tid / 4; kk = (tid % 4) * 4 + e; }
      else          { kk = tid / 16; mm = (tid % 16) * 4 + e; }
      const int64_t m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < M && k < K) v = ld_f(A, m * g.sam + k * g.sak);
      As[kk][mm] = v;
    }
    // B tile [BK x BN]
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int nn, kk;
      if (b_nmajor) { kk = tid / 16; nn = (tid % 16) * 4 + e; }
      else          { nn = tid / 4; kk = (tid % 4) * 4 + e; }
      const int64_t n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < N && k < K) v = ld_f(B, k * g.sbk + n * g.sbn);
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
    // K blocks (kblk, a multiple of BK): partial sums restart at each block boundary
    if (g.kblk > 0 && ((k0 + BK) % g.kblk == 0 || k0 + BK >= K)) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { tot[i][j] += acc[i][j]; acc[i][j] = 0.f; }
    }
  }
  if (g.kblk > 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = tot[i][j];
  }

  if (g.epi == EPI_STORE || g.epi == EPI_ACC) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t m = m0 + ty + 16 * i;
      if (m >= M) continue;
      const int64_t row = g.crow ? (int64_t)g.crow[m] : m;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t n = n0 + tx + 16 * j;
        if (n >= N) continue;
        float v = g.alpha * acc[i][j];
        if (g.bias) v += ld_dt(g.bias, g.bias_dt, n);
        const int64_t off = row * g.ldc + n;
        if (g.epi == EPI_ACC) v += ld_dt(g.C, g.cdt, off);
        st_dt(g.C, g.cdt, off, v);
      }
    }
    return;
  }
  if (g.epi == EPI_SWIGLU_BWD) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t m = m0 + ty + 16 * i;
      if (m >= M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t n = n0 + tx + 16 * j;
        if (n >= N) continue;
        const float dm = g.alpha * acc[i][j];
        const float gv = ld_dt(g.aux, g.cdt, m * g.aux_ld + n);
        const float uv = ld_dt(g.aux, g.cdt, m * g.aux_ld + g.aux_off + n);
        const float sg = 1.f / (1.f + expf(-gv));
        st_dt(g.C, g.cdt, m * g.ldc + n, dm * uv * sg * (1.f + gv * (1.f - sg)));
        st_dt(g.C, g.cdt, m * g.ldc + g.aux_off + n, dm * gv * sg);
      }
    }
    return;
  }
  if (g.epi == EPI_CEGRAD) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t m = m0 + ty + 16 * i;
      if (m >= g.M) continue;
      const float w = g.wt[m];
      const float l = g.lse[m];
      const int y = g.tgt[m];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t n = n0 + tx + 16 * j;
        if (n >= N) continue;
        float p = expf(acc[i][j] - l);
        if (g.col0 + n == (int64_t)y) p -= 1.f;
        st_dt(g.C, g.cdt, m * g.ldc + n, w * p);
      }
    }
    return;
  }
  // EPI_LSE: reduce the tile's columns per row
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) St[ty + 16 * i][tx + 16 * j] = acc[i][j];
  __syncthreads();
  if (tid < BM) {
    const int64_t m = m0 + tid;
    if (m < M) {
      const int ncols = (int)imin(BN, N - n0);
      float mx = -INFINITY;
      for (int j = 0; j < ncols; ++j) mx = fmaxf(mx, St[tid][j]);
      float s = 0.f;
      for (int j = 0; j < ncols; ++j) s += expf(St[tid][j] - mx);
      g.pmax[m * g.pld + blockIdx.x] = mx;
      g.psum[m * g.pld + blockIdx.x] = s;
      const int64_t y = (int64_t)g.tgt[m] - g.col0 - n0;
      if (y >= 0 && y < ncols) g.zy[m] = St[tid][y];
    }
  }
}

}  // namespace

int64_t gemm_lse_tiles(int64_t N) { return (N + BN - 1) / BN; }

cudaError_t gemm_simt(const GemmDesc& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  dim3 grid((unsigned)((g.N + BN - 1) / BN), (unsigned)((g.M + BM - 1) / BM));
  if (grid.y > 65535u) return cudaErrorInvalidValue;
  if (g.adt == DT_F32 && g.bdt == DT_F32)
    launch(gemm_simt_kernel<float, float>, grid, 256, 0, st, g);
  else if (g.adt == DT_BF16 && g.bdt == DT_BF16)
    launch(gemm_simt_kernel<__nv_bfloat16, __nv_bfloat16>, grid, 256, 0, st, g);
  else if (g.adt == DT_F32 && g.bdt == DT_BF16)
    launch(gemm_simt_kernel<float, __nv_bfloat16>, grid, 256, 0, st, g);
  else
    launch(gemm_simt_kernel<__nv_bfloat16, float>, grid, 256, 0, st, g);
  return cudaGetLastError();
}

}  // namespace sbp
