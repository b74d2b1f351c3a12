// Row-wise and element-wise kernels of the decoder layer: RMSNorm forward/backward, RoPE,
// SwiGLU, chunk gather/scatter, deterministic column sums, embedding.  All are HBM-bound:
// coalesced accesses along the feature dimension, one CTA per row (or grid-stride), fp32
// arithmetic, warp-shuffle reductions.
#include "sbp_internal.cuh"

namespace sbp {

namespace {

constexpr int kRowThreads = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = 0.f;
  const int nw = blockDim.x >> 5;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

// ---------------------------------------------------------------- 8-wide vector access
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = q;
}

// RMSNorm forward, 8 columns per access (cols % 8 == 0, 16-byte aligned rows)
template <typename TX, typename TG, typename TY>
__global__ void rmsnorm_fwd_vec_kernel(int64_t cols, const TX* __restrict__ x,
                                       const TG* __restrict__ g, TY* __restrict__ y,
                                       float* __restrict__ rstd, float eps) {
  __shared__ float red[32];
  const int64_t r = blockIdx.x;
  const TX* xr = x + r * cols;
  float ss = 0.f;
  for (int64_t c = 8 * threadIdx.x; c < cols; c += 8 * blockDim.x) {
    float v[8];
    load8(xr + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(v[i], v[i], ss);
  }
  ss = block_sum(ss, red);
  const float rs = rsqrtf(ss / (float)cols + eps);
  for (int64_t c = 8 * threadIdx.x; c < cols; c += 8 * blockDim.x) {
    float v[8], gv[8];
    load8(xr + c, v);
    load8(g + c, gv);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = v[i] * rs * gv[i];
    store8(y + r * cols + c, v);
  }
  if (rstd && threadIdx.x == 0) rstd[r] = rs;
}

// RMSNorm forward with the row held in registers (NCH 8-column chunks per thread): x and g are
// read once, all loads of a thread in flight together; the sum of squares and the products
// are formed in the same order as in rmsnorm_fwd_vec_kernel, so the results are identical.
template <typename TX, typename TG, typename TY, int NCH>
__global__ void __launch_bounds__(kRowThreads)
rmsnorm_fwd_reg_kernel(int64_t rows, int64_t cols, const TX* __restrict__ x,
                       const TG* __restrict__ g, TY* __restrict__ y, float* __restrict__ rstd,
                       float eps) {
  __shared__ float red[32];
  float gv[NCH][8];
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
    if (c < cols) load8(g + c, gv[k]);
  }
  // a few CTAs per SM take the rows in turn (block_sum synchronises before reusing red)
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const TX* xr = x + r * cols;
    float v[NCH][8];
  #pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
      if (c < cols) load8(xr + c, v[k]);
    }
    float ss = 0.f;
  #pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
      if (c < cols) {
  #pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(v[k][i], v[k][i], ss);
      }
    }
    ss = block_sum(ss, red);
    const float rs = rsqrtf(ss / (float)cols + eps);
  #pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
      if (c < cols) {
  #pragma unroll
        for (int i = 0; i < 8; ++i) v[k][i] = v[k][i] * rs * gv[k][i];
        store8(y + r * cols + c, v[k]);
      }
    }
    if (rstd && threadIdx.x == 0) rstd[r] = rs;
  }
}

// RMSNorm backward, 8 columns per access; each thread keeps the dg partial of its columns in
// registers (NCH <= kVecChunks 8-column chunks per thread, sized to the row so that three CTAs
// fit on an SM).
constexpr int kVecChunks = 4;
template <typename TX, typename TG, int NCH>
__global__ void __launch_bounds__(256, NCH <= 2 ? 3 : 2)
rmsnorm_bwd_vec_kernel(int64_t rows, int64_t cols, const TX* __restrict__ x,
                       const TG* __restrict__ g, const float* __restrict__ rstd,
                       const float* __restrict__ dy, const float* __restrict__ base,
                       float* __restrict__ out, int accumulate, float* __restrict__ partial) {
  __shared__ float red[32];
  float dg[NCH][8];
  float gv[NCH][8];
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
#pragma unroll
    for (int i = 0; i < 8; ++i) dg[k][i] = 0.f;
    if (c < cols) load8(g + c, gv[k]);
  }
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t o = r * cols;
    const float rs = rstd[r];
    float xh[NCH][8], u[NCH][8];
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
      if (c >= cols) continue;
      float xv[8], dv[8];
      load8(x + o + c, xv);
      load8(dy + o + c, dv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        xh[k][i] = xv[i] * rs;
        u[k][i] = dv[i] * gv[k][i];
        dot = fmaf(xh[k][i], u[k][i], dot);
        dg[k][i] = fmaf(dv[i], xh[k][i], dg[k][i]);
      }
    }
    dot = block_sum(dot, red) / (float)cols;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
      if (c >= cols) continue;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = rs * (u[k][i] - xh[k][i] * dot);
      if (base) {
        float b[8];
        load8(base + o + c, b);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] += b[i];
      }
      if (accumulate) {
        float b[8];
        load8(out + o + c, b);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] += b[i];
      }
      store8(out + o + c, v);
    }
  }
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int64_t c = 8 * (threadIdx.x + (int64_t)k * blockDim.x);
    if (c < cols) store8(partial + (int64_t)blockIdx.x * cols + c, dg[k]);
  }
}

// y = x (cast), 8 per thread
template <typename TS, typename TD>
__global__ void copy_cast_vec_kernel(int64_t n8, const TS* __restrict__ src, TD* __restrict__ dst) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  float v[8];
  load8(src + 8 * i, v);
  store8(dst + 8 * i, v);
}

// hi = bf16(v), lo = bf16(v - hi) of four values, stored as 4 + 4 bf16 (8-byte aligned)
__device__ __forceinline__ void split4_store(__nv_bfloat16* hi, __nv_bfloat16* lo, float4 v) {
  const float f[4] = {v.x, v.y, v.z, v.w};
  float h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    h[k] = __bfloat162float(__float2bfloat16_rn(f[k]));
    l[k] = f[k] - h[k];
  }
  __nv_bfloat162 hh[2] = {__floats2bfloat162_rn(h[0], h[1]), __floats2bfloat162_rn(h[2], h[3])};
  __nv_bfloat162 ll[2] = {__floats2bfloat162_rn(l[0], l[1]), __floats2bfloat162_rn(l[2], l[3])};
  *reinterpret_cast<uint2*>(hi) = *reinterpret_cast<const uint2*>(hh);
  *reinterpret_cast<uint2*>(lo) = *reinterpret_cast<const uint2*>(ll);
}

// hi + lo split of the chunk's rows of a [B, T, cols] fp32 prefix: row r of hi / lo is row
// (r / Tc) T + s + r % Tc of src (8 values per thread; cols % 8 == 0, 16-byte aligned rows)
__global__ void gather_split_bf16_kernel(int64_t n8, int64_t cols8, int64_t Tc, int64_t s,
                                         int64_t T, const float* __restrict__ src,
                                         __nv_bfloat16* __restrict__ hi,
                                         __nv_bfloat16* __restrict__ lo) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const int64_t r = i / cols8, c8 = i - r * cols8;
  const int64_t srow = (r / Tc) * T + s + r % Tc;
  float v[8], h[8], l[8];
  load8(src + (srow * cols8 + c8) * 8, v);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    h[k] = __bfloat162float(__float2bfloat16_rn(v[k]));
    l[k] = v[k] - h[k];
  }
  store8(hi + i * 8, h);
  store8(lo + i * 8, l);
}

__global__ void split_bf16_vec_kernel(int64_t n8, const float* __restrict__ x,
                                      __nv_bfloat16* __restrict__ hi,
                                      __nv_bfloat16* __restrict__ lo) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  float v[8], h[8], l[8];
  load8(x + 8 * i, v);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    h[k] = __bfloat162float(__float2bfloat16_rn(v[k]));
    l[k] = v[k] - h[k];
  }
  store8(hi + 8 * i, h);
  store8(lo + 8 * i, l);
}

__global__ void swiglu_fwd_vec_kernel(int64_t R, int64_t f, const __nv_bfloat16* __restrict__ gu,
                                      __nv_bfloat16* __restrict__ m) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // 8-column group
  const int64_t f8 = f / 8;
  if (i >= R * f8) return;
  const int64_t r = i / f8, c = 8 * (i % f8);
  float gv[8], uv[8], o[8];
  load8(gu + r * 2 * f + c, gv);
  load8(gu + r * 2 * f + f + c, uv);
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] = gv[k] / (1.f + expf(-gv[k])) * uv[k];
  store8(m + r * f + c, o);
}

inline bool al16p(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- RMSNorm forward
__global__ void rmsnorm_fwd_kernel(int64_t cols, int xdt, const void* __restrict__ x, int gdt,
                                   const void* __restrict__ g, int ydt, void* __restrict__ y,
                                   float* __restrict__ rstd, float eps) {
  __shared__ float red[32];
  const int64_t r = blockIdx.x;
  const int64_t base = r * cols;
  float ss = 0.f;
  for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
    const float v = ld_dt(x, xdt, base + c);
    ss = fmaf(v, v, ss);
  }
  ss = block_sum(ss, red);
  const float rs = rsqrtf(ss / (float)cols + eps);
  for (int64_t c = threadIdx.x; c < cols; c += blockDim.x)
    st_dt(y, ydt, base + c, ld_dt(x, xdt, base + c) * rs * ld_dt(g, gdt, c));
  if (rstd && threadIdx.x == 0) rstd[r] = rs;
}

// ---------------------------------------------------------------- RMSNorm backward
// Each CTA handles rows r = blockIdx.x, blockIdx.x + gridDim.x, ...; its dg partial goes to
// partial[blockIdx.x, :] and a second kernel sums the partials in a fixed order.
constexpr int kBwdBlocks = 444;   // 3 per SM

__global__ void rmsnorm_bwd_kernel(int64_t rows, int64_t cols, int xdt,
                                   const void* __restrict__ x, int gdt,
                                   const void* __restrict__ g, const float* __restrict__ rstd,
                                   const float* __restrict__ dy, const float* __restrict__ base,
                                   float* __restrict__ out, int accumulate,
                                   float* __restrict__ partial) {
  __shared__ float red[32];
  extern __shared__ float dgs[];  // [cols]
  for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) dgs[c] = 0.f;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t o = r * cols;
    const float rs = rstd[r];
    float dot = 0.f;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
      const float xh = ld_dt(x, xdt, o + c) * rs;
      const float u = dy[o + c] * ld_dt(g, gdt, c);
      dot = fmaf(xh, u, dot);
    }
    dot = block_sum(dot, red) / (float)cols;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
      const float xh = ld_dt(x, xdt, o + c) * rs;
      const float d = dy[o + c];
      const float u = d * ld_dt(g, gdt, c);
      float v = rs * (u - xh * dot);
      if (base) v += base[o + c];
      if (accumulate) v += out[o + c];
      out[o + c] = v;
      dgs[c] = fmaf(d, xh, dgs[c]);
    }
  }
  __syncthreads();
  for (int64_t c = threadIdx.x; c < cols; c += blockDim.x)
    partial[(int64_t)blockIdx.x * cols + c] = dgs[c];
}

// dst[c] += sum_p partial[p, c].  A CTA of 1024 threads takes 32 columns; its 32 warps sum
// interleaved 32nds of the partial rows (a dozen independent loads per thread for the 444
// partial rows of the RMSNorm backward), and warp 0 adds the 32 sums in a fixed order.
constexpr int kColsumCols = 32, kColsumGroups = 32;
__global__ void __launch_bounds__(kColsumCols * kColsumGroups)
colsum_partials_kernel(int64_t nparts, int64_t cols, const float* __restrict__ partial,
                       float* __restrict__ dst) {
  __shared__ float red[kColsumGroups][kColsumCols];
  const int lc = threadIdx.x % kColsumCols, grp = threadIdx.x / kColsumCols;
  const int64_t c = (int64_t)blockIdx.x * kColsumCols + lc;
  float s = 0.f;
  if (c < cols) {
#pragma unroll 4
    for (int64_t p = grp; p < nparts; p += kColsumGroups) s += __ldg(partial + p * cols + c);
  }
  red[grp][lc] = s;
  __syncthreads();
  if (grp == 0 && c < cols) {
    float t = red[0][lc];
#pragma unroll
    for (int g2 = 1; g2 < kColsumGroups; ++g2) t += red[g2][lc];
    dst[c] += t;
  }
}

// column partial sums of a [rows, cols] fp32 matrix: CTA b sums rows b, b + grid, ...
__global__ void colsum_stage1_kernel(int64_t rows, int64_t cols, const float* __restrict__ src,
                                     float* __restrict__ partial) {
  const int64_t c = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float s = 0.f;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) s += src[r * cols + c];
  partial[(int64_t)blockIdx.x * cols + c] = s;
}
constexpr int kColsumParts = 64;

// ---------------------------------------------------------------- RoPE
__global__ void rope_table_kernel(int64_t T, int64_t half, double theta, float* cosb,
                                  float* sinb) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * half) return;
  const int64_t t = i / half, j = i % half;
  const double inv_freq = pow(theta, -(2.0 * (double)j) / (double)(2 * half));
  const double a = (double)t * inv_freq;
  cosb[i] = (float)cos(a);
  sinb[i] = (float)sin(a);
}

// One CTA per row r (token s + r % Tc of sequence r / Tc); its threads stride over the
// (head, pair j) slots of heads h_lo .. h_lo + nh - 1 of the combined q | k | v head index and
// rotate (x_j, x_{j+half}) of q and k; v is copied.  Per-element index math is 32-bit.
__global__ void qkv_post_kernel(int64_t Tc, int64_t s, int64_t T, int H, int Hkv, int hd,
                                int h_lo, int nh, const float* __restrict__ qkv, int dt,
                                void* __restrict__ q, void* __restrict__ Kp,
                                void* __restrict__ Vp, const float* __restrict__ cosb,
                                const float* __restrict__ sinb) {
  const int64_t r = blockIdx.x;
  const int half = hd / 2;
  const int heads = H + 2 * Hkv;
  const int64_t b = r / Tc, t = s + r % Tc;
  const float* row = qkv + r * (int64_t)heads * hd;
  const float* cr = cosb + t * half;
  const float* sr = sinb + t * half;
  const int64_t qo = r * (int64_t)H * hd;               // this row in q [R, H * hd]
  const int64_t ko = (b * T + t) * (int64_t)Hkv * hd;   // this token in the K/V prefix
  const int n = nh * half;
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int hq = p / half;
    const int j = p - hq * half;
    const int hh = h_lo + hq;
    const float x1 = row[hh * hd + j], x2 = row[hh * hd + j + half];
    if (hh < H + Hkv) {
      const float c = cr[j], sn = sr[j];
      const float y1 = x1 * c - x2 * sn;
      const float y2 = x2 * c + x1 * sn;
      if (hh < H) {
        st_dt(q, dt, qo + hh * hd + j, y1);
        st_dt(q, dt, qo + hh * hd + j + half, y2);
      } else {
        st_dt(Kp, dt, ko + (hh - H) * hd + j, y1);
        st_dt(Kp, dt, ko + (hh - H) * hd + j + half, y2);
      }
    } else {
      st_dt(Vp, dt, ko + (hh - H - Hkv) * hd + j, x1);
      st_dt(Vp, dt, ko + (hh - H - Hkv) * hd + j + half, x2);
    }
  }
}

// inverse rotation (transpose): (d1, d2) -> (d1 c + d2 s, d2 c - d1 s).  One CTA per row r
// of x [R, heads, hd] (position s + r % Tc); threads stride over its (head, pair) slots.
__global__ void rope_inv_kernel(int64_t Tc, int64_t s, int heads, int hd, float* __restrict__ x,
                                const float* __restrict__ cosb, const float* __restrict__ sinb) {
  const int64_t r = blockIdx.x;
  const int half = hd / 2;
  const int64_t t = s + r % Tc;
  float* row = x + r * (int64_t)heads * hd;
  const float* cr = cosb + t * half;
  const float* sr = sinb + t * half;
  const int n = heads * half;
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int hh = p / half;
    const int j = p - hh * half;
    float* o = row + hh * hd;
    const float d1 = o[j], d2 = o[j + half];
    const float c = cr[j], sn = sr[j];
    o[j] = d1 * c + d2 * sn;
    o[j + half] = d2 * c - d1 * sn;
  }
}

// dst row r [heads, hd] = inverse rotation of src [B, T, heads, hd] at (r / Tc, s + r % Tc)
__global__ void gather_rope_inv_kernel(int64_t T, int64_t Tc, int64_t s, int heads, int hd,
                                       const float* __restrict__ src, float* __restrict__ dst,
                                       const float* __restrict__ cosb,
                                       const float* __restrict__ sinb) {
  const int64_t r = blockIdx.x;
  const int half = hd / 2;
  const int64_t b = r / Tc, t = s + r % Tc;
  const float* srow = src + (b * T + t) * (int64_t)heads * hd;
  float* drow = dst + r * (int64_t)heads * hd;
  const float* cr = cosb + t * half;
  const float* sr = sinb + t * half;
  const int n = heads * half;
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int hh = p / half;
    const int j = p - hh * half;
    const float d1 = srow[hh * hd + j], d2 = srow[hh * hd + j + half];
    const float c = cr[j], sn = sr[j];
    drow[hh * hd + j] = d1 * c + d2 * sn;
    drow[hh * hd + j + half] = d2 * c - d1 * sn;
  }
}

// The same inverse rotation with 16-byte accesses (hd % 8 == 0, rows and tables 16-byte
// aligned): a thread rotates four consecutive pairs (x_j..x_j+3, x_j+half..x_j+half+3) of one
// head.  dst row r = rotation of src row (r / Tc) T + s + r % Tc when gather, else of src row r
// (in place when src == dst).
__global__ void rope_inv_vec_kernel(int64_t T, int64_t Tc, int64_t s, int heads, int hd,
                                    int gather, const float* src, float* dst,
                                    const float* __restrict__ cosb,
                                    const float* __restrict__ sinb,
                                    __nv_bfloat16* __restrict__ hi,
                                    __nv_bfloat16* __restrict__ lo) {
  const int64_t r = blockIdx.x;
  const int half = hd / 2, q4 = half / 4;
  const int64_t b = r / Tc, t = s + r % Tc;
  const float* srow = src + (gather ? b * T + t : r) * (int64_t)heads * hd;
  float* drow = dst + r * (int64_t)heads * hd;
  const float4* cr = reinterpret_cast<const float4*>(cosb + t * half);
  const float4* sr = reinterpret_cast<const float4*>(sinb + t * half);
  const int n = heads * q4;
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int hh = p / q4;
    const int j4 = p - hh * q4;
    const int o1 = hh * hd + 4 * j4, o2 = o1 + half;
    const float4 a = *reinterpret_cast<const float4*>(srow + o1);
    const float4 e = *reinterpret_cast<const float4*>(srow + o2);
    const float4 c = cr[j4], sn = sr[j4];
    float4 u, w;
    u.x = a.x * c.x + e.x * sn.x;  w.x = e.x * c.x - a.x * sn.x;
    u.y = a.y * c.y + e.y * sn.y;  w.y = e.y * c.y - a.y * sn.y;
    u.z = a.z * c.z + e.z * sn.z;  w.z = e.z * c.z - a.z * sn.z;
    u.w = a.w * c.w + e.w * sn.w;  w.w = e.w * c.w - a.w * sn.w;
    if (hi) {
      // the rotated values go out as their hi + lo bf16 split (the fp32 row is not stored)
      const int64_t ro = r * (int64_t)heads * hd;
      split4_store(hi + ro + o1, lo + ro + o1, u);
      split4_store(hi + ro + o2, lo + ro + o2, w);
    } else {
      *reinterpret_cast<float4*>(drow + o1) = u;
      *reinterpret_cast<float4*>(drow + o2) = w;
    }
  }
}

// ---------------------------------------------------------------- SwiGLU
__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + expf(-x)); }

__global__ void swiglu_fwd_kernel(int64_t R, int64_t f, int dt, const void* __restrict__ gu,
                                  void* __restrict__ m) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * f) return;
  const int64_t r = i / f, c = i % f;
  const float gv = ld_dt(gu, dt, r * 2 * f + c);
  const float uv = ld_dt(gu, dt, r * 2 * f + f + c);
  st_dt(m, dt, i, gv * sigmoidf_(gv) * uv);
}

__global__ void swiglu_bwd_kernel(int64_t R, int64_t f, int dt, const void* __restrict__ gu,
                                  const float* __restrict__ dm, void* __restrict__ dgu) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * f) return;
  const int64_t r = i / f, c = i % f;
  const float gv = ld_dt(gu, dt, r * 2 * f + c);
  const float uv = ld_dt(gu, dt, r * 2 * f + f + c);
  const float sg = sigmoidf_(gv);
  const float d = dm[i];
  st_dt(dgu, dt, r * 2 * f + c, d * uv * sg * (1.f + gv * (1.f - sg)));
  st_dt(dgu, dt, r * 2 * f + f + c, d * gv * sg);
}

// ---------------------------------------------------------------- gather / scatter
__global__ void gather_chunk_kernel(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols,
                                    int dt, const void* __restrict__ src, void* __restrict__ dst) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * Tc * cols) return;
  const int64_t c = i % cols, r = i / cols;
  const int64_t b = r / Tc, t = s + r % Tc;
  const int64_t so = (b * T + t) * cols + c;
  if (dt == DT_BF16)
    static_cast<__nv_bfloat16*>(dst)[i] = static_cast<const __nv_bfloat16*>(src)[so];
  else
    static_cast<float*>(dst)[i] = static_cast<const float*>(src)[so];
}

// Row copy between the chunk buffer [B * Tc, cols] and the sequence layout [B, T, cols] in
// 16-byte units: one CTA per chunk row (token s + r % Tc of sequence r / Tc), threads over the
// row's units.  to_seq: chunk -> sequence (optionally adding fp32 rows), else sequence -> chunk.
__global__ void chunk_rows_vec_kernel(int64_t Tc, int64_t s, int64_t T, int units,
                                      const uint4* __restrict__ src, uint4* __restrict__ dst,
                                      int to_seq, int accumulate_f32) {
  const int64_t r = blockIdx.x;
  const int64_t srow = (r / Tc) * T + s + r % Tc;
  const uint4* sp = src + (to_seq ? r : srow) * units;
  uint4* dp = dst + (to_seq ? srow : r) * units;
  for (int u = threadIdx.x; u < units; u += blockDim.x) {
    uint4 v = sp[u];
    if (accumulate_f32) {
      const uint4 o = dp[u];
      v.x = __float_as_uint(__uint_as_float(v.x) + __uint_as_float(o.x));
      v.y = __float_as_uint(__uint_as_float(v.y) + __uint_as_float(o.y));
      v.z = __float_as_uint(__uint_as_float(v.z) + __uint_as_float(o.z));
      v.w = __float_as_uint(__uint_as_float(v.w) + __uint_as_float(o.w));
    }
    dp[u] = v;
  }
}

__global__ void scatter_chunk_kernel(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols,
                                     int dt, const void* __restrict__ src, void* __restrict__ dst,
                                     int accumulate) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * Tc * cols) return;
  const int64_t c = i % cols, r = i / cols;
  const int64_t b = r / Tc, t = s + r % Tc;
  const int64_t o = (b * T + t) * cols + c;
  if (dt == DT_BF16) {
    static_cast<__nv_bfloat16*>(dst)[o] = static_cast<const __nv_bfloat16*>(src)[i];
  } else {
    const float v = static_cast<const float*>(src)[i];
    float* d = static_cast<float*>(dst);
    d[o] = accumulate ? d[o] + v : v;
  }
}

__global__ void add_residual_kernel(int64_t n, int xdt, const void* __restrict__ x,
                                    const float* __restrict__ z, int ydt, void* __restrict__ y) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  st_dt(y, ydt, i, ld_dt(x, xdt, i) + z[i]);
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi): a 16-bit-mantissa operand for the tensor
// cores, used where a value's fp32 rounding depends on the chunking (the fp32 dK/dV sums)
__global__ void split_bf16_kernel(int64_t n, const float* __restrict__ x,
                                  __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = x[i];
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi[i] = h;
  lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
}

__global__ void copy_cast_kernel(int64_t n, int sdt, const void* __restrict__ src, int ddt,
                                 void* __restrict__ dst) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  st_dt(dst, ddt, i, ld_dt(src, sdt, i));
}

// ---------------------------------------------------------------- embedding
// ids outside [0, vocab) produce a zero row (and are skipped by the backward)
__global__ void embed_fwd_kernel(int64_t rows, int64_t cols, int64_t vocab, int dt,
                                 const int* __restrict__ ids, const void* __restrict__ table,
                                 void* __restrict__ y) {
  const int64_t r = blockIdx.x;
  const int64_t v = ids[r];
  const bool ok = v >= 0 && v < vocab;
  for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
    if (dt == DT_BF16)
      static_cast<__nv_bfloat16*>(y)[r * cols + c] =
          ok ? static_cast<const __nv_bfloat16*>(table)[v * cols + c] : __float2bfloat16_rn(0.f);
    else
      static_cast<float*>(y)[r * cols + c] = ok ? static_cast<const float*>(table)[v * cols + c]
                                                : 0.f;
  }
}

// Deterministic embedding backward: counting sort of rows by id (stable), then one CTA per
// distinct id sums its rows in row order.
__global__ void embed_count_kernel(int64_t rows, int64_t vocab, const int* __restrict__ ids,
                                   int* cnt) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r < rows && ids[r] >= 0 && ids[r] < vocab) atomicAdd(&cnt[ids[r]], 1);
}
// exclusive scan of cnt[0..vocab) into off (single CTA, 1024 threads, sequential chunks)
__global__ void scan_kernel(int64_t n, const int* __restrict__ cnt, int* __restrict__ off) {
  __shared__ int part[1024];
  const int64_t per = (n + blockDim.x - 1) / blockDim.x;
  const int64_t b = threadIdx.x * per, e = imin(n, b + per);
  int s = 0;
  for (int64_t i = b; i < e; ++i) s += cnt[i];
  part[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0;
    for (int i = 0; i < (int)blockDim.x; ++i) { const int t = part[i]; part[i] = a; a += t; }
  }
  __syncthreads();
  int a = part[threadIdx.x];
  for (int64_t i = b; i < e; ++i) { off[i] = a; a += cnt[i]; }
}
// rows of each id land in their segment in arbitrary order (atomics); the accumulate kernel
// restores row order inside the segment before summing, so the sum is deterministic.
__global__ void embed_place_kernel(int64_t rows, int64_t vocab, const int* __restrict__ ids,
                                   int* __restrict__ pos, int* __restrict__ order) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r < rows && ids[r] >= 0 && ids[r] < vocab) order[atomicAdd(&pos[ids[r]], 1)] = (int)r;
}
constexpr int kSegSort = 2048;
__global__ void embed_accum_kernel(int64_t rows, int64_t cols, const int* __restrict__ ids,
                                   const int* __restrict__ off0, const int* __restrict__ cnt,
                                   const int* __restrict__ order, const float* __restrict__ dy,
                                   float* __restrict__ dtable) {
  __shared__ int seg[kSegSort];
  __shared__ int srt[kSegSort];
  const int64_t v = blockIdx.x;
  const int n = cnt[v];
  if (n == 0) return;
  if (n <= kSegSort) {
    const int o = off0[v];
    for (int i = threadIdx.x; i < n; i += blockDim.x) seg[i] = order[o + i];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      int rank = 0;
      const int a = seg[i];
      for (int j = 0; j < n; ++j) rank += (seg[j] < a);
      srt[rank] = a;
    }
    __syncthreads();
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) {
      float s = 0.f;
      for (int k = 0; k < n; ++k) s += dy[(int64_t)srt[k] * cols + c];
      dtable[v * cols + c] += s;
    }
  } else {
    // very frequent id: walk all rows in order
    for (int64_t c0 = 0; c0 < cols; c0 += blockDim.x) {
      const int64_t c = c0 + threadIdx.x;
      float s = 0.f;
      for (int64_t r = 0; r < rows; ++r)
        if (ids[r] == (int)v && c < cols) s += dy[r * cols + c];
      if (c < cols) dtable[v * cols + c] += s;
    }
  }
}

inline unsigned nblk(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace

cudaError_t rmsnorm_fwd(int64_t rows, int64_t cols, int xdt, const void* x, int gdt,
                        const void* g, int ydt, void* y, float* rstd, float eps,
                        cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (cols % 8 == 0 && gdt == DT_BF16 && ydt == DT_BF16 && al16p(x) && al16p(g) && al16p(y)) {
    const auto* gb = static_cast<const __nv_bfloat16*>(g);
    auto* yb = static_cast<__nv_bfloat16*>(y);
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    const auto* xf = static_cast<const float*>(x);
    const int64_t nch = (cols + 8 * kRowThreads - 1) / (8 * kRowThreads);
    const dim3 grid((unsigned)rows), block(kRowThreads);
    const int64_t rcap = (int64_t)sm_count() * 8;   // 8 CTAs of 256 threads per SM
    const dim3 rgrid((unsigned)(rows < rcap ? rows : rcap));
    if (nch > 4) {
      if (xdt == DT_BF16)
        launch(rmsnorm_fwd_vec_kernel<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>, grid, block,
               0, st, cols, xb, gb, yb, rstd, eps);
      else
        launch(rmsnorm_fwd_vec_kernel<float, __nv_bfloat16, __nv_bfloat16>, grid, block, 0, st,
               cols, xf, gb, yb, rstd, eps);
    } else if (xdt == DT_BF16) {
      if (nch == 1)
        launch(rmsnorm_fwd_reg_kernel<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16, 1>, rgrid, block, 0, st, rows, cols, xb, gb, yb, rstd, eps);
      else if (nch == 2)
        launch(rmsnorm_fwd_reg_kernel<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16, 2>, rgrid, block, 0, st, rows, cols, xb, gb, yb, rstd, eps);
      else
        launch(rmsnorm_fwd_reg_kernel<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16, 4>, rgrid, block, 0, st, rows, cols, xb, gb, yb, rstd, eps);
    } else {
      if (nch == 1)
        launch(rmsnorm_fwd_reg_kernel<float, __nv_bfloat16, __nv_bfloat16, 1>, rgrid, block, 0, st, rows, cols, xf, gb, yb, rstd, eps);
      else if (nch == 2)
        launch(rmsnorm_fwd_reg_kernel<float, __nv_bfloat16, __nv_bfloat16, 2>, rgrid, block, 0, st, rows, cols, xf, gb, yb, rstd, eps);
      else
        launch(rmsnorm_fwd_reg_kernel<float, __nv_bfloat16, __nv_bfloat16, 4>, rgrid, block, 0, st, rows, cols, xf, gb, yb, rstd, eps);
    }
    return cudaGetLastError();
  }
  launch(rmsnorm_fwd_kernel, (unsigned)rows, kRowThreads, 0, st, cols, xdt, x, gdt, g, ydt, y, rstd,
                                                             eps);
  return cudaGetLastError();
}

size_t rmsnorm_bwd_partial_floats(int64_t cols) { return (size_t)kBwdBlocks * cols; }

cudaError_t rmsnorm_bwd(int64_t rows, int64_t cols, int xdt, const void* x, int gdt,
                        const void* g, const float* rstd, const float* dy, const float* base,
                        float* out, int accumulate, float* dg, float* partial,
                        cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (cols % 8 == 0 && cols <= 8 * kRowThreads * kVecChunks && gdt == DT_BF16 && al16p(x) &&
      al16p(g) && al16p(dy) && al16p(out) && (!base || al16p(base))) {
    const auto* gb = static_cast<const __nv_bfloat16*>(g);
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    const auto* xf = static_cast<const float*>(x);
    const dim3 grid(kBwdBlocks), block(kRowThreads);
    const int nch = (int)((cols + 8 * kRowThreads - 1) / (8 * kRowThreads));
    if (xdt == DT_BF16) {
      if (nch <= 1)
        launch(rmsnorm_bwd_vec_kernel<__nv_bfloat16, __nv_bfloat16, 1>, grid, block, 0, st, rows,
               cols, xb, gb, rstd, dy, base, out, accumulate, partial);
      else if (nch == 2)
        launch(rmsnorm_bwd_vec_kernel<__nv_bfloat16, __nv_bfloat16, 2>, grid, block, 0, st, rows,
               cols, xb, gb, rstd, dy, base, out, accumulate, partial);
      else
        launch(rmsnorm_bwd_vec_kernel<__nv_bfloat16, __nv_bfloat16, kVecChunks>, grid, block, 0,
               st, rows, cols, xb, gb, rstd, dy, base, out, accumulate, partial);
    } else {
      if (nch <= 1)
        launch(rmsnorm_bwd_vec_kernel<float, __nv_bfloat16, 1>, grid, block, 0, st, rows, cols,
               xf, gb, rstd, dy, base, out, accumulate, partial);
      else if (nch == 2)
        launch(rmsnorm_bwd_vec_kernel<float, __nv_bfloat16, 2>, grid, block, 0, st, rows, cols,
               xf, gb, rstd, dy, base, out, accumulate, partial);
      else
        launch(rmsnorm_bwd_vec_kernel<float, __nv_bfloat16, kVecChunks>, grid, block, 0, st,
               rows, cols, xf, gb, rstd, dy, base, out, accumulate, partial);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !dg) return e;
    launch(colsum_partials_kernel, dim3(nblk(cols, kColsumCols)),
           dim3(kColsumCols * kColsumGroups), 0, st, (int64_t)kBwdBlocks,
           cols, (const float*)partial, dg);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)cols * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(rmsnorm_bwd_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  launch(rmsnorm_bwd_kernel, kBwdBlocks, kRowThreads, smem, st, rows, cols, xdt, x, gdt, g, rstd, dy,
                                                            base, out, accumulate, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (dg) {
    launch(colsum_partials_kernel, nblk(cols, kColsumCols), kColsumCols * kColsumGroups, 0, st,
           kBwdBlocks, cols, partial, dg);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t rope_table(int64_t T, int64_t hd, double theta, float* cosb, float* sinb,
                       cudaStream_t st) {
  const int64_t n = T * (hd / 2);
  if (n <= 0) return cudaSuccess;
  launch(rope_table_kernel, nblk(n, 256), 256, 0, st, T, hd / 2, theta, cosb, sinb);
  return cudaGetLastError();
}

cudaError_t qkv_post(int64_t R, int64_t Tc, int64_t s, int64_t T, int64_t H, int64_t Hkv,
                     int64_t hd, const float* qkv, int dt, void* q, void* Kp, void* Vp,
                     const float* cosb, const float* sinb, cudaStream_t st, int part) {
  const int64_t h_lo = part == QKV_KV ? H : 0;
  const int64_t h_hi = part == QKV_Q ? H : H + 2 * Hkv;
  if (R <= 0 || h_hi <= h_lo || hd < 2) return cudaSuccess;
  launch(qkv_post_kernel, dim3((unsigned)R), dim3(256), 0, st, Tc, s, T, (int)H, (int)Hkv,
         (int)hd, (int)h_lo, (int)(h_hi - h_lo), qkv, dt, q, Kp, Vp, cosb, sinb);
  return cudaGetLastError();
}

cudaError_t rope_inv_f32(int64_t R, int64_t Tc, int64_t s, int64_t heads, int64_t hd, float* x,
                         const float* cosb, const float* sinb, cudaStream_t st) {
  if (R <= 0 || heads <= 0 || hd < 2) return cudaSuccess;
  if (hd % 8 == 0 && al16p(x) && al16p(cosb) && al16p(sinb)) {
    launch(rope_inv_vec_kernel, dim3((unsigned)R), dim3(128), 0, st, (int64_t)0, Tc, s,
           (int)heads, (int)hd, 0, (const float*)x, x, cosb, sinb,
           static_cast<__nv_bfloat16*>(nullptr), static_cast<__nv_bfloat16*>(nullptr));
    return cudaGetLastError();
  }
  launch(rope_inv_kernel, dim3((unsigned)R), dim3(256), 0, st, Tc, s, (int)heads, (int)hd, x,
         cosb, sinb);
  return cudaGetLastError();
}

cudaError_t gather_rope_inv(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t heads,
                            int64_t hd, const float* src, float* dst, const float* cosb,
                            const float* sinb, cudaStream_t st) {
  const int64_t R = B * Tc;
  if (R <= 0 || heads <= 0 || hd < 2) return cudaSuccess;
  if (hd % 8 == 0 && al16p(src) && al16p(dst) && al16p(cosb) && al16p(sinb)) {
    launch(rope_inv_vec_kernel, dim3((unsigned)R), dim3(128), 0, st, T, Tc, s, (int)heads,
           (int)hd, 1, src, dst, cosb, sinb, static_cast<__nv_bfloat16*>(nullptr),
           static_cast<__nv_bfloat16*>(nullptr));
    return cudaGetLastError();
  }
  launch(gather_rope_inv_kernel, dim3((unsigned)R), dim3(256), 0, st, T, Tc, s, (int)heads,
         (int)hd, src, dst, cosb, sinb);
  return cudaGetLastError();
}

bool gather_split_ok(int64_t hd, int64_t cols, const void* src, const void* hi, const void* lo,
                     const float* cosb, const float* sinb) {
  return hd % 8 == 0 && cols % 8 == 0 && al16p(src) && al16p(hi) && al16p(lo) && al16p(cosb) &&
         al16p(sinb);
}

cudaError_t gather_rope_inv_split(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t heads,
                                  int64_t hd, const float* src, void* hi, void* lo,
                                  const float* cosb, const float* sinb, cudaStream_t st) {
  const int64_t R = B * Tc;
  if (R <= 0 || heads <= 0) return cudaSuccess;
  launch(rope_inv_vec_kernel, dim3((unsigned)R), dim3(128), 0, st, T, Tc, s, (int)heads, (int)hd,
         1, src, static_cast<float*>(nullptr), cosb, sinb, static_cast<__nv_bfloat16*>(hi),
         static_cast<__nv_bfloat16*>(lo));
  return cudaGetLastError();
}

cudaError_t gather_split_bf16(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols,
                              const float* src, void* hi, void* lo, cudaStream_t st) {
  const int64_t n8 = B * Tc * cols / 8;
  if (n8 <= 0) return cudaSuccess;
  launch(gather_split_bf16_kernel, dim3(nblk(n8, 256)), dim3(256), 0, st, n8, cols / 8, Tc, s, T,
         src, static_cast<__nv_bfloat16*>(hi), static_cast<__nv_bfloat16*>(lo));
  return cudaGetLastError();
}

cudaError_t swiglu_fwd(int64_t R, int64_t f, int dt, const void* gu, void* m, cudaStream_t st) {
  if (R * f <= 0) return cudaSuccess;
  if (dt == DT_BF16 && f % 8 == 0 && al16p(gu) && al16p(m)) {
    const int64_t n = R * (f / 8);
    launch(swiglu_fwd_vec_kernel, dim3(nblk(n, 256)), dim3(256), 0, st, R, f,
           static_cast<const __nv_bfloat16*>(gu), static_cast<__nv_bfloat16*>(m));
    return cudaGetLastError();
  }
  launch(swiglu_fwd_kernel, nblk(R * f, 256), 256, 0, st, R, f, dt, gu, m);
  return cudaGetLastError();
}

cudaError_t swiglu_bwd(int64_t R, int64_t f, int dt, const void* gu, const float* dm, void* dgu,
                       cudaStream_t st) {
  if (R * f <= 0) return cudaSuccess;
  launch(swiglu_bwd_kernel, nblk(R * f, 256), 256, 0, st, R, f, dt, gu, dm, dgu);
  return cudaGetLastError();
}

namespace {
// The 16-byte row path applies when rows are whole 16-byte units and both buffers aligned.
bool rows_vec_ok(int64_t cols, int dt, const void* a, const void* b) {
  const int64_t bytes = cols * (int64_t)dt_size(dt);
  return bytes % 16 == 0 && bytes / 16 <= (1 << 20) &&
         (reinterpret_cast<uintptr_t>(a) & 15u) == 0 && (reinterpret_cast<uintptr_t>(b) & 15u) == 0;
}
cudaError_t chunk_rows_vec(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols, int dt,
                           const void* src, void* dst, int to_seq, int accumulate_f32,
                           cudaStream_t st) {
  const int units = (int)(cols * (int64_t)dt_size(dt) / 16);
  const int threads = units >= 256 ? 256 : ((units + 31) / 32) * 32;
  launch(chunk_rows_vec_kernel, dim3((unsigned)(B * Tc)), dim3(threads), 0, st, Tc, s, T, units,
         static_cast<const uint4*>(src), static_cast<uint4*>(dst), to_seq, accumulate_f32);
  return cudaGetLastError();
}
}  // namespace

cudaError_t gather_chunk(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols, int dt,
                         const void* src, void* dst, cudaStream_t st) {
  const int64_t n = B * Tc * cols;
  if (n <= 0) return cudaSuccess;
  if (rows_vec_ok(cols, dt, src, dst)) return chunk_rows_vec(B, T, Tc, s, cols, dt, src, dst, 0, 0, st);
  launch(gather_chunk_kernel, nblk(n, 256), 256, 0, st, B, T, Tc, s, cols, dt, src, dst);
  return cudaGetLastError();
}

cudaError_t scatter_chunk_f32(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols,
                              const float* src, float* dst, int accumulate, cudaStream_t st) {
  const int64_t n = B * Tc * cols;
  if (n <= 0) return cudaSuccess;
  if (rows_vec_ok(cols, DT_F32, src, dst))
    return chunk_rows_vec(B, T, Tc, s, cols, DT_F32, src, dst, 1, accumulate, st);
  launch(scatter_chunk_kernel, nblk(n, 256), 256, 0, st, B, T, Tc, s, cols, DT_F32, src, dst,
                                                     accumulate);
  return cudaGetLastError();
}

cudaError_t scatter_chunk(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols, int dt,
                          const void* src, void* dst, cudaStream_t st) {
  const int64_t n = B * Tc * cols;
  if (n <= 0) return cudaSuccess;
  if (rows_vec_ok(cols, dt, src, dst)) return chunk_rows_vec(B, T, Tc, s, cols, dt, src, dst, 1, 0, st);
  launch(scatter_chunk_kernel, nblk(n, 256), 256, 0, st, B, T, Tc, s, cols, dt, src, dst, 0);
  return cudaGetLastError();
}

size_t colsum_partial_floats(int64_t cols) { return (size_t)kColsumParts * cols; }

cudaError_t colsum_acc(int64_t rows, int64_t cols, const float* src, float* dst, float* partial,
                       cudaStream_t st) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  dim3 g1(kColsumParts, nblk(cols, 256));
  launch(colsum_stage1_kernel, g1, 256, 0, st, rows, cols, src, partial);
  launch(colsum_partials_kernel, nblk(cols, kColsumCols), kColsumCols * kColsumGroups, 0, st,
         kColsumParts, cols, partial, dst);
  return cudaGetLastError();
}

cudaError_t add_residual(int64_t n, int xdt, const void* x, const float* z, int ydt, void* y,
                         cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  launch(add_residual_kernel, nblk(n, 256), 256, 0, st, n, xdt, x, z, ydt, y);
  return cudaGetLastError();
}

cudaError_t split_bf16(int64_t n, const float* x, void* hi, void* lo, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (n % 8 == 0 && al16p(x) && al16p(hi) && al16p(lo)) {
    launch(split_bf16_vec_kernel, dim3(nblk(n / 8, 256)), dim3(256), 0, st, n / 8, x,
           static_cast<__nv_bfloat16*>(hi), static_cast<__nv_bfloat16*>(lo));
    return cudaGetLastError();
  }
  launch(split_bf16_kernel, nblk(n, 256), 256, 0, st, n, x, static_cast<__nv_bfloat16*>(hi),
                                                  static_cast<__nv_bfloat16*>(lo));
  return cudaGetLastError();
}

cudaError_t copy_cast(int64_t n, int sdt, const void* src, int ddt, void* dst, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (n % 8 == 0 && al16p(src) && al16p(dst)) {
    const int64_t n8 = n / 8;
    const dim3 grid(nblk(n8, 256)), blk(256);
    if (sdt == DT_F32 && ddt == DT_BF16)
      launch(copy_cast_vec_kernel<float, __nv_bfloat16>, grid, blk, 0, st, n8,
             static_cast<const float*>(src), static_cast<__nv_bfloat16*>(dst));
    else if (sdt == DT_BF16 && ddt == DT_F32)
      launch(copy_cast_vec_kernel<__nv_bfloat16, float>, grid, blk, 0, st, n8,
             static_cast<const __nv_bfloat16*>(src), static_cast<float*>(dst));
    else if (sdt == DT_F32 && ddt == DT_F32)
      launch(copy_cast_vec_kernel<float, float>, grid, blk, 0, st, n8,
             static_cast<const float*>(src), static_cast<float*>(dst));
    else
      launch(copy_cast_vec_kernel<__nv_bfloat16, __nv_bfloat16>, grid, blk, 0, st, n8,
             static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst));
    return cudaGetLastError();
  }
  launch(copy_cast_kernel, nblk(n, 256), 256, 0, st, n, sdt, src, ddt, dst);
  return cudaGetLastError();
}

cudaError_t embed_fwd(int64_t rows, int64_t cols, int64_t vocab, int dt, const int* ids,
                      const void* table, void* y, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  launch(embed_fwd_kernel, (unsigned)rows, 256, 0, st, rows, cols, vocab, dt, ids, table, y);
  return cudaGetLastError();
}

size_t embed_bwd_ws_ints(int64_t rows, int64_t vocab) { return (size_t)(3 * vocab + rows); }

cudaError_t embed_bwd(int64_t rows, int64_t cols, int64_t vocab, const int* ids, const float* dy,
                      float* dtable, int* ws, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  int* cnt = ws;
  int* off = ws + vocab;
  int* pos = ws + 2 * vocab;
  int* order = ws + 3 * vocab;
  cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int) * vocab, st);
  if (e != cudaSuccess) return e;
  launch(embed_count_kernel, nblk(rows, 256), 256, 0, st, rows, vocab, ids, cnt);
  launch(scan_kernel, 1, 1024, 0, st, vocab, cnt, off);
  e = cudaMemcpyAsync(pos, off, sizeof(int) * vocab, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  launch(embed_place_kernel, nblk(rows, 256), 256, 0, st, rows, vocab, ids, pos, order);
  launch(embed_accum_kernel, (unsigned)vocab, 128, 0, st, rows, cols, ids, off, cnt, order, dy,
                                                       dtable);
  return cudaGetLastError();
}

}  // namespace sbp
