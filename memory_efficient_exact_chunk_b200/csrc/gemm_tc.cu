// Persistent bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
//   C[m, n] (op)= sum_k A(m, k) B(k, n),   A, B bf16 in either K-major or MN-major layout,
//   fp32 accumulation in TMEM, fused epilogues (store / accumulate fp32 or bf16, column bias,
//   row remap, cross-entropy log-sum-exp partials, cross-entropy logit gradient).
//
// CTA tile 128 x 256 x 64, 4-stage TMA -> shared-memory ring, warp-specialised:
//   warp 0      : TMA producer (one lane)
//   warp 1      : TMEM allocator + MMA issuer (one lane), M=128 N=256 K=16 instructions
//   warps 2..9  : epilogue, TMEM -> registers -> global (each warp owns 32 TMEM lanes and half
//                 of the tile's columns)
// The accumulator is double-buffered in TMEM (2 x 256 columns) so the epilogue of tile i
// overlaps the main loop of tile i+1.  One CTA per SM, grid = min(tiles, SMs).
// Every mbarrier wait is bounded; on timeout the CTA raises the device status word, drains its
// own TMA copies and MMAs (bounded), frees TMEM and exits.
#include <cuda.h>

#include <mutex>

#include "sbp_internal.cuh"
#include "tc_ptx.cuh"

// Cycle accounting of the pair kernel, compiled in only with -DSBP_GEMM_TIMING (the build's
// --timing library): per launch, CTAs 0/1 print the producer's time waiting for free ring
// stages, the MMA issuer's time waiting for operands and for a free accumulator, and the
// epilogue's time waiting for a full accumulator and working.  Off by default: no cost.
#ifdef SBP_GEMM_TIMING
#include <cstdio>
#define SBP_TIMED(...) __VA_ARGS__
#else
#define SBP_TIMED(...)
#endif

namespace sbp {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B_BYTES = BN * BK * 2;                 // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;  // + alignment slack
constexpr int TMEM_COLS = 2 * BN;                    // double-buffered accumulator
constexpr int kEpiWarps = 8;                        // 4 TMEM lane quarters x 2 column halves
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kGroupM = 8;                           // tile rasterisation group

struct TcArgs {
  GemmDesc g;
  int a_mn, b_mn;
  int nM, nN;
  int gm;               // row tiles per rasterisation group
  int* err;
};

// Tile t of a launch: groups of gm row tiles, row tiles fastest within a group, so the CTAs
// running at the same time share a few A row panels and B column panels in L2.
__device__ __forceinline__ void tile_coords(int t, int nM, int nN, int gm, int& mt, int& nt) {
  const int per_group = gm * nN;
  const int group = t / per_group;
  const int first_m = group * gm;
  const int gsz = min(nM - first_m, gm);
  const int r = t % per_group;
  mt = first_m + r % gsz;
  nt = r / gsz;
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// True when a launch has nothing to write: no live rows (every tile would be skipped), or
// C += A B over an empty K range (the weight gradient of a chunk without loss rows), which
// leaves C as it is.  The same for every CTA, so the grid (and a CTA pair) returns together,
// before any barrier or TMEM is set up.
__device__ __forceinline__ bool nothing_to_do(const GemmDesc& g) {
  const int64_t M = g.dynM ? (int64_t)*g.dynM : g.M;
  const int64_t K = g.dynK ? (int64_t)*g.dynK : g.K;
  return M <= 0 || (K <= 0 && g.epi == EPI_ACC && !g.bias);
}

__device__ __forceinline__ void store8_bf16(__nv_bfloat16* p, const float* v) {
  uint4 pk;
  __nv_bfloat162 t0 = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 t1 = __floats2bfloat162_rn(v[2], v[3]);
  __nv_bfloat162 t2 = __floats2bfloat162_rn(v[4], v[5]);
  __nv_bfloat162 t3 = __floats2bfloat162_rn(v[6], v[7]);
  pk.x = *reinterpret_cast<uint32_t*>(&t0);
  pk.y = *reinterpret_cast<uint32_t*>(&t1);
  pk.z = *reinterpret_cast<uint32_t*>(&t2);
  pk.w = *reinterpret_cast<uint32_t*>(&t3);
  *reinterpret_cast<uint4*>(p) = pk;
}

// Store / accumulate 32 consecutive values v[0..31] of row `row` starting at column n.  A
// later K block (blk > 0) always accumulates and does not add the bias again.
__device__ __forceinline__ void epi_store32(const GemmDesc& g, int64_t row, int64_t n, int64_t N,
                                            float (&v)[32], int blk) {
  const bool accum = g.epi == EPI_ACC || blk > 0;
  if (g.bias && blk == 0) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (n + j < N) v[j] += ld_dt(g.bias, g.bias_dt, n + j);
  }
  const int64_t off = row * g.ldc + n;
  if (n + 32 <= N) {
    if (g.cdt == DT_F32) {
      float* c = static_cast<float*>(g.C) + off;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 x = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        if (accum) {
          const float4 o = *reinterpret_cast<const float4*>(c + j);
          x.x += o.x; x.y += o.y; x.z += o.z; x.w += o.w;
        }
        *reinterpret_cast<float4*>(c + j) = x;
      }
    } else {
      __nv_bfloat16* c = static_cast<__nv_bfloat16*>(g.C) + off;
      if (accum) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += __bfloat162float(c[j]);
      }
#pragma unroll
      for (int j = 0; j < 32; j += 8) store8_bf16(c + j, v + j);
    }
  } else {
    for (int j = 0; j < 32 && n + j < N; ++j) {
      float x = v[j];
      if (accum) x += ld_dt(g.C, g.cdt, off + j);
      st_dt(g.C, g.cdt, off + j, x);
    }
  }
}

__device__ __forceinline__ float silu_grad_parts(float dm, float gv, float uv, float* du) {
  const float sg = 1.f / (1.f + __expf(-gv));
  *du = dm * gv * sg;
  return dm * uv * sg * (1.f + gv * (1.f - sg));
}

// SwiGLU backward for 32 consecutive columns: v = dM, g / u from aux (bf16), results to C (bf16).
__device__ __forceinline__ void epi_swiglu_bwd32(const GemmDesc& g, int64_t m, int64_t n,
                                                 int64_t N, const float (&v)[32]) {
  const __nv_bfloat16* gp = static_cast<const __nv_bfloat16*>(g.aux) + m * g.aux_ld + n;
  const __nv_bfloat16* up = gp + g.aux_off;
  __nv_bfloat16* dgp = static_cast<__nv_bfloat16*>(g.C) + m * g.ldc + n;
  __nv_bfloat16* dup = dgp + g.aux_off;
  if (n + 32 <= N) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 gq = *reinterpret_cast<const uint4*>(gp + 8 * q);
      const uint4 uq = *reinterpret_cast<const uint4*>(up + 8 * q);
      const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&gq);
      const __nv_bfloat16* ub = reinterpret_cast<const __nv_bfloat16*>(&uq);
      float dg[8], du[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dg[i] = silu_grad_parts(v[8 * q + i], __bfloat162float(gb[i]), __bfloat162float(ub[i]),
                                &du[i]);
      store8_bf16(dgp + 8 * q, dg);
      store8_bf16(dup + 8 * q, du);
    }
  } else {
    for (int i = 0; i < 32 && n + i < N; ++i) {
      float du;
      const float dg = silu_grad_parts(v[i], __bfloat162float(gp[i]), __bfloat162float(up[i]),
                                       &du);
      dgp[i] = __float2bfloat16_rn(dg);
      dup[i] = __float2bfloat16_rn(du);
    }
  }
}

// SwiGLU forward for 32 consecutive columns: v = u, g from aux (bf16); u (rounded to bf16) to
// C and m = silu(g) u of the rounded u to C2 (bf16) -- the values the separate SwiGLU kernel
// computes from the stored g and u, bit for bit, and the ones the backward differentiates.
__device__ __forceinline__ void epi_swiglu_fwd32(const GemmDesc& g, int64_t m, int64_t n,
                                                 int64_t N, const float (&v)[32]) {
  const __nv_bfloat16* gp = static_cast<const __nv_bfloat16*>(g.aux) + m * g.aux_ld + n;
  __nv_bfloat16* up = static_cast<__nv_bfloat16*>(g.C) + m * g.ldc + n;
  __nv_bfloat16* mp = static_cast<__nv_bfloat16*>(g.C2) + m * g.ldc2 + n;
  if (n + 32 <= N) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 gq = *reinterpret_cast<const uint4*>(gp + 8 * q);
      const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&gq);
      float mv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float gv = __bfloat162float(gb[i]);
        const float uv = __bfloat162float(__float2bfloat16_rn(v[8 * q + i]));
        mv[i] = gv / (1.f + expf(-gv)) * uv;
      }
      store8_bf16(up + 8 * q, v + 8 * q);
      store8_bf16(mp + 8 * q, mv);
    }
  } else {
    for (int i = 0; i < 32 && n + i < N; ++i) {
      const float gv = __bfloat162float(gp[i]);
      const __nv_bfloat16 ub = __float2bfloat16_rn(v[i]);
      up[i] = ub;
      mp[i] = __float2bfloat16_rn(gv / (1.f + expf(-gv)) * __bfloat162float(ub));
    }
  }
}

// Epilogue of one accumulator tile for the calling thread's row m: tile columns
// [c_lo, c_lo + BN / 2) (this warp's half) starting at global column n0, read from TMEM at
// tbase (this warp's lane quarter, accumulator base column).  nk = the k-steps summed into
// the accumulator (0: it holds nothing); blk = the index of its K block (see kblk).
__device__ __forceinline__ void epilogue_tile(const GemmDesc& g, uint32_t tbase, int64_t m,
                                              int64_t n0, int64_t M, int64_t N, int nk,
                                              int c_lo, int blk) {
  const int c_hi = c_lo + BN / 2;
  // the logit-gradient epilogue also writes the zero rows between the live row count and
  // the buffer's row count, so that a later product over those rows reads zeros
  const bool row_ok = m < (g.epi == EPI_CEGRAD ? g.M : M);
  if (g.epi == EPI_LSE) {
    for (int c = c_lo; c < c_hi; c += 64) {
      uint32_t r0[32], r1[32];
      tc::tmem_ld32(tbase + c, r0);
      tc::tmem_ld32(tbase + c + 32, r1);
      tc::tmem_ld_wait();
      const int64_t nc = n0 + c;
      if (!row_ok || nc >= N) continue;
      const int ncols = (int)imin(64, N - nc);
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float a = nk ? u2f(r0[j]) : 0.f, b = nk ? u2f(r1[j]) : 0.f;
        if (j < ncols) mx = fmaxf(mx, a);
        if (j + 32 < ncols) mx = fmaxf(mx, b);
      }
      const float mxl = mx * tc::kLog2e;
      float sm = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float a = nk ? u2f(r0[j]) : 0.f, b = nk ? u2f(r1[j]) : 0.f;
        if (j < ncols) sm += tc::ex2_approx(fmaf(a, tc::kLog2e, -mxl));
        if (j + 32 < ncols) sm += tc::ex2_approx(fmaf(b, tc::kLog2e, -mxl));
      }
      const int64_t tile = nc / 64;
      g.pmax[m * g.pld + tile] = mx;
      g.psum[m * g.pld + tile] = sm;
      const int64_t y = (int64_t)g.tgt[m] - g.col0 - nc;
      if (y >= 0 && y < ncols) {
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (y == j) z = u2f(r0[j]);
          if (y == j + 32) z = u2f(r1[j]);
        }
        g.zy[m] = nk ? z : 0.f;
      }
    }
  } else if (g.epi == EPI_ROPE) {
    // this warp's 128 columns are one head: rotate pairs (i, i + 64) with the row's position
    const int64_t rr = m % g.r_Tc;
    const int64_t pos = g.r_s + rr;
    const int64_t drow = g.r_T > 0 ? (m / g.r_Tc) * g.r_T + pos : m;
    const int64_t nh = n0 + c_lo;                 // the head's first column
#pragma unroll 1
    for (int c = 0; c < 64; c += 32) {
      uint32_t lo[32], hi[32];
      tc::tmem_ld32(tbase + c_lo + c, lo);
      tc::tmem_ld32(tbase + c_lo + 64 + c, hi);
      tc::tmem_ld_wait();
      if (!row_ok || nh >= N) continue;
      float a[32], bb[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        a[j] = nk ? u2f(lo[j]) : 0.f;
        bb[j] = nk ? u2f(hi[j]) : 0.f;
      }
      if (g.bias) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          a[j] += ld_dt(g.bias, g.bias_dt, nh + c + j);
          bb[j] += ld_dt(g.bias, g.bias_dt, nh + 64 + c + j);
        }
      }
      if (g.cosb) {
        const float* cr = g.cosb + pos * 64 + c;
        const float* sr = g.sinb + pos * 64 + c;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float cs = cr[j], sn = sr[j];
          const float y1 = a[j] * cs - bb[j] * sn;
          const float y2 = bb[j] * cs + a[j] * sn;
          a[j] = y1;
          bb[j] = y2;
        }
      }
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.C) + drow * g.ldc + nh + c;
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        store8_bf16(out + j, a + j);
        store8_bf16(out + 64 + j, bb + j);
      }
    }
  } else {
    float w = 0.f, l = 0.f;
    int64_t ycol = -1;
    int64_t crow = m;
    if (row_ok) {
      if (g.epi == EPI_CEGRAD) {
        w = g.wt[m];
        l = g.lse[m];
        ycol = (int64_t)g.tgt[m] - g.col0;
      } else if (g.crow) {
        crow = g.crow[m];
      }
    }
    for (int c = c_lo; c < c_hi; c += 32) {
      uint32_t r[32];
      tc::tmem_ld32(tbase + c, r);
      tc::tmem_ld_wait();
      const int64_t nc = n0 + c;
      if (!row_ok || nc >= N) continue;
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = nk ? u2f(r[j]) : 0.f;
      if (g.epi == EPI_SWIGLU_BWD) {
        epi_swiglu_bwd32(g, m, nc, N, v);
        continue;
      }
      if (g.epi == EPI_SWIGLU_FWD) {
        epi_swiglu_fwd32(g, m, nc, N, v);
        continue;
      }
      if (g.epi == EPI_CEGRAD) {
        const float ll = l * tc::kLog2e;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float p = tc::ex2_approx(fmaf(v[j], tc::kLog2e, -ll));
          if (nc + j == ycol) p -= 1.f;
          v[j] = w * p;
        }
      } else if (g.alpha != 1.f) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= g.alpha;
      }
      epi_store32(g, crow, nc, N, v, blk);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES], tfull_bar[2], tempty_bar[2];
  __shared__ uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GemmDesc& g = args.g;
  volatile int* abort_flag = &abort_sh;
  if (nothing_to_do(g)) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full_bar[s], 1);
      tc::mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull_bar[a], 1);
      tc::mbar_init(&tempty_bar[a], kEpiWarps);
    }
    tc::mbar_init(&drain_bar, 1);
    abort_sh = 0;
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tmA);
    tc::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tc::tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = tmem_base_sh;

  const int64_t M = g.dynM ? (int64_t)*g.dynM : g.M;
  const int64_t K = g.dynK ? (int64_t)*g.dynK : g.K;
  const int64_t N = g.N;
  const int nk = (int)((K + BK - 1) / BK);
  const int ntiles = args.nM * args.nN;
  // k-steps per K block and blocks per tile (one block, possibly empty, when kblk == 0)
  const int kpb = g.kblk > 0 ? (int)(g.kblk / BK) : (nk > 0 ? nk : 1);
  const int nblk = nk > 0 ? (nk + kpb - 1) / kpb : 1;
  const bool stall = g.stall_wait_ns > 0;
  const uint64_t wait_ns = stall ? (uint64_t)g.stall_wait_ns : tc::kWaitLimitNs;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok && !stall; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, args.nM, args.nN, args.gm, mt, nt);
        const int m0 = mt * BM, n0 = nt * BN;
        if (m0 >= M) continue;
        for (int kb = 0; kb < nk; ++kb) {
          if (!tc::mbar_wait(&empty_bar[s], ph ^ 1u, abort_flag, wait_ns)) { ok = false; break; }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          tc::mbar_expect_tx(&full_bar[s], STAGE_BYTES);
          const int k0 = kb * BK;
          if (!args.a_mn) {
            tc::tma_load_2d(sa, &tmA, &full_bar[s], k0, m0);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j)
              tc::tma_load_2d(sa + j * 8192, &tmA, &full_bar[s], m0 + 64 * j, k0);
          }
          if (!args.b_mn) {
            tc::tma_load_2d(sb, &tmB, &full_bar[s], k0, n0);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tc::tma_load_2d(sb + j * 8192, &tmB, &full_bar[s], n0 + 64 * j, k0);
          }
          issued_mask |= 1u << s;
          issued_phase = (issued_phase & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        // wind down: wait (bounded) for this CTA's own copies still in flight
        const uint64_t t0 = tc::globaltimer_ns();
        for (int q = 0; q < STAGES; ++q) {
          if (!(issued_mask & (1u << q))) continue;
          const uint32_t p = (issued_phase >> q) & 1u;
          while (!tc::mbar_try_wait(&full_bar[q], p) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(BM, BN, args.a_mn, args.b_mn);
      const uint32_t smem_base = tc::smem_u32(smem);
      // descriptors of stage 0 / k-step 0 and their increments (16-byte units): the loop
      // below only adds loop-invariant values, so the issuing thread keeps up with the
      // tensor pipe (computing each descriptor afresh costs it more than an N = 256 MMA)
      const uint64_t a_desc0 = args.a_mn ? tc::smem_desc_sw128(smem_base, 8192, 1024)
                                         : tc::smem_desc_sw128(smem_base, 16, 1024);
      const uint64_t b_desc0 = args.b_mn ? tc::smem_desc_sw128(smem_base + A_BYTES, 8192, 1024)
                                         : tc::smem_desc_sw128(smem_base + A_BYTES, 16, 1024);
      const uint64_t a_kstep = args.a_mn ? (2048 >> 4) : (32 >> 4);
      const uint64_t b_kstep = args.b_mn ? (2048 >> 4) : (32 >> 4);
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      bool issued = false;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, args.nM, args.nN, args.gm, mt, nt);
        if ((int64_t)mt * BM >= M) continue;
        for (int b = 0; b < nblk && ok; ++b) {
          if (!tc::mbar_wait(&tempty_bar[acc], aph ^ 1u, abort_flag, wait_ns)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          const int kb0 = b * kpb, kb1 = imin(nk, kb0 + kpb);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!tc::mbar_wait(&full_bar[s], ph, abort_flag, wait_ns)) { ok = false; break; }
            tc::fence_after_sync();
            const uint64_t soff = (uint64_t)(s * (STAGE_BYTES >> 4));
            const uint64_t ad = a_desc0 + soff, bd = b_desc0 + soff;
            tc::mma_f16_ss(d_tmem, ad, bd, idesc, kb != kb0 ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < BK / 16; ++kk)
              tc::mma_f16_ss(d_tmem, ad + kk * a_kstep, bd + kk * b_kstep, idesc, 1u);
            issued = true;
            tc::mma_commit(&empty_bar[s]);
            if (++s == STAGES) { s = 0; ph ^= 1u; }
          }
          if (!ok) break;
          tc::mma_commit(&tfull_bar[acc]);
          if (++acc == 2) { acc = 0; aph ^= 1u; }
        }
      }
      if (issued) {
        // make sure every MMA of this CTA has completed before TMEM is released
        tc::mma_commit(&drain_bar);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&drain_bar, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    const int c_lo = ((warp - 2) >> 2) * (BN / 2);
    int acc = 0;
    uint32_t aph = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(t, args.nM, args.nN, args.gm, mt, nt);
      const int64_t m0 = (int64_t)mt * BM, n0 = (int64_t)nt * BN;
      if (m0 >= M) continue;
      bool ok = true;
      for (int b = 0; b < nblk; ++b) {
        if (!tc::mbar_wait_warp(&tfull_bar[acc], aph, abort_flag, wait_ns)) { ok = false; break; }
        tc::fence_after_sync();
        const int64_t m = m0 + row_in_tile;
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
        epilogue_tile(g, tbase, m, n0, M, N, imin(nk - b * kpb, kpb), c_lo, b);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&tempty_bar[acc]);
        if (++acc == 2) { acc = 0; aph ^= 1u; }
      }
      if (!ok) break;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && abort_sh && args.err) atomicExch(args.err, DEV_TIMEOUT);
  if (warp == 1) tc::tmem_dealloc(tmem_base, TMEM_COLS);
}


// ============================================================================ CTA-pair kernel
// The same GEMM on 256 x 256 tiles computed by a pair of CTAs (a 2-CTA cluster) with
// tcgen05.mma.cta_group::2: each CTA stages 128 rows of A and 128 rows (N/2) of B per k-block,
// the even CTA issues M=256 N=256 MMAs that read both CTAs' shared memory, and each CTA keeps
// its 128 accumulator rows in its own TMEM.  Shared-memory traffic per MMA is half that of the
// single-CTA kernel, which is what lets the tensor cores run closer to their peak.
// Operands stream through six slots of 64 k-columns (per CTA: 128 rows of A and 128 rows of
// B, 16 KB each), consumed in pairs: one mbarrier completes when both slots of a pair hold
// data, so the MMA thread waits once per eight K = 16 MMAs (a wait costs the issuing thread
// about as long as an N = 256 MMA runs, and the tensor pipe idles meanwhile), while the
// producer refills each slot as soon as its own MMAs complete (up to five slots in flight
// ahead of the one being consumed).
constexpr int BM2 = 256, NSLOT2 = 6, NPAIR2 = NSLOT2 / 2, BK2 = 2 * BK;
constexpr int A2_BYTES = 128 * BK * 2;              // 16 KB per CTA per slot
constexpr int B2_BYTES = 128 * BK * 2;              // 16 KB per CTA per slot (half of N)
constexpr int SLOT2_BYTES = A2_BYTES + B2_BYTES;
constexpr int SMEM2_BYTES = NSLOT2 * SLOT2_BYTES + 1024;

__global__ void __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[NPAIR2], empty_bar[NSLOT2], tfull_bar[2], tempty_bar[2];
  __shared__ uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GemmDesc& g = args.g;
  volatile int* abort_flag = &abort_sh;
  if (nothing_to_do(g)) return;
  const uint32_t rank = tc::cluster_ctarank();      // 0 = leader (issues the MMAs)
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NPAIR2; ++s) tc::mbar_init(&full_bar[s], 1);
    for (int s = 0; s < NSLOT2; ++s) tc::mbar_init(&empty_bar[s], 1);
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull_bar[a], 1);
      tc::mbar_init(&tempty_bar[a], 2 * kEpiWarps);   // epilogue warps of both CTAs
    }
    tc::mbar_init(&drain_bar, 1);
    abort_sh = 0;
    tc::fence_barrier_init();
    tc::prefetch_tmap(&tmA);
    tc::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(&tmem_base_sh, TMEM_COLS);
    tc::tmem_relinquish_pair();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();                        // barriers of both CTAs initialised
  tc::fence_after_sync();
  const uint32_t tmem_base = tmem_base_sh;

  const int64_t M = g.dynM ? (int64_t)*g.dynM : g.M;
  const int64_t K = g.dynK ? (int64_t)*g.dynK : g.K;
  const int64_t N = g.N;
  const int nk = (int)((K + BK2 - 1) / BK2);
  const int ntiles = args.nM * args.nN;      // nM counts 256-row tiles here
  const int kpb = g.kblk > 0 ? (int)(g.kblk / BK2) : (nk > 0 ? nk : 1);
  const int nblk = nk > 0 ? (nk + kpb - 1) / kpb : 1;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      SBP_TIMED(long long w_empty = 0, tp0 = clock64(), c0; int ntl = 0;)
      for (int t = cluster; t < ntiles && ok; t += nclusters) {
        int mt, nt;
        tile_coords(t, args.nM, args.nN, args.gm, mt, nt);
        const int m0 = mt * BM2, n0 = nt * BN;
        if (m0 >= M) continue;
        SBP_TIMED(++ntl;)
        const int ma = m0 + 128 * (int)rank, nb = n0 + 128 * (int)rank;
        for (int kb = 0; kb < nk && ok; ++kb) {
          const uint32_t fb = tc::mapa(tc::smem_u32(&full_bar[s]), 0);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int q = 2 * s + h;
            SBP_TIMED(c0 = clock64();)
            if (!tc::mbar_wait(&empty_bar[q], ph ^ 1u, abort_flag)) { ok = false; break; }
            SBP_TIMED(w_empty += clock64() - c0;)
            uint8_t* sa = smem + q * SLOT2_BYTES;
            uint8_t* sb = sa + A2_BYTES;
            if (h == 0) {
              if (rank == 0) tc::mbar_expect_tx(&full_bar[s], 2 * 2 * SLOT2_BYTES);
              issued_mask |= 1u << s;
              issued_phase = (issued_phase & ~(1u << s)) | (ph << s);
            }
            const int k0 = kb * BK2 + h * BK;
            if (!args.a_mn) {
              tc::tma_load_2d_pair(sa, &tmA, fb, k0, ma);
            } else {
              tc::tma_load_2d_pair(sa, &tmA, fb, ma, k0);
              tc::tma_load_2d_pair(sa + 8192, &tmA, fb, ma + 64, k0);
            }
            if (!args.b_mn) {
              tc::tma_load_2d_pair(sb, &tmB, fb, k0, nb);
            } else {
              tc::tma_load_2d_pair(sb, &tmB, fb, nb, k0);
              tc::tma_load_2d_pair(sb + 8192, &tmB, fb, nb + 64, k0);
            }
          }
          if (++s == NPAIR2) { s = 0; ph ^= 1u; }
        }
      }
      SBP_TIMED(if (blockIdx.x < 2) printf(
          "SBPT PROD cta %d M %lld N %lld K %lld epi %d tiles %d total %lld w_empty %lld\n",
          (int)blockIdx.x, (long long)M, (long long)N, (long long)K, g.epi, ntl,
          clock64() - tp0, w_empty);)
      if (!ok && rank == 0) {
        // wind down: wait (bounded) for the pair's copies in flight on this CTA's barriers
        const uint64_t t0 = tc::globaltimer_ns();
        for (int q = 0; q < NPAIR2; ++q) {
          if (!(issued_mask & (1u << q))) continue;
          const uint32_t p = (issued_phase >> q) & 1u;
          while (!tc::mbar_try_wait(&full_bar[q], p) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(BM2, BN, args.a_mn, args.b_mn);
      const uint32_t smem_base = tc::smem_u32(smem);
      // slot-0 descriptors and the k-step increments (16-byte units), as in the single-CTA
      // kernel: the loop below only adds loop-invariant values
      const uint64_t a_desc0 = args.a_mn ? tc::smem_desc_sw128(smem_base, 8192, 1024)
                                         : tc::smem_desc_sw128(smem_base, 16, 1024);
      const uint64_t b_desc0 = args.b_mn ? tc::smem_desc_sw128(smem_base + A2_BYTES, 8192, 1024)
                                         : tc::smem_desc_sw128(smem_base + A2_BYTES, 16, 1024);
      const uint64_t a_kstep = args.a_mn ? (2048 >> 4) : (32 >> 4);
      const uint64_t b_kstep = args.b_mn ? (2048 >> 4) : (32 >> 4);
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      bool issued = false;
      SBP_TIMED(long long w_full = 0, w_temp = 0, ti0 = clock64(), c0; int nkbt = 0;)
      for (int t = cluster; t < ntiles && ok; t += nclusters) {
        int mt, nt;
        tile_coords(t, args.nM, args.nN, args.gm, mt, nt);
        if ((int64_t)mt * BM2 >= M) continue;
        for (int b = 0; b < nblk && ok; ++b) {
          SBP_TIMED(c0 = clock64();)
          if (!tc::mbar_wait(&tempty_bar[acc], aph ^ 1u, abort_flag)) { ok = false; break; }
          SBP_TIMED(w_temp += clock64() - c0;)
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          const int kb0 = b * kpb, kb1 = imin(nk, kb0 + kpb);
          for (int kb = kb0; kb < kb1; ++kb) {
            SBP_TIMED(c0 = clock64();)
            if (!tc::mbar_wait(&full_bar[s], ph, abort_flag)) { ok = false; break; }
            SBP_TIMED(w_full += clock64() - c0; ++nkbt;)
            tc::fence_after_sync();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t soff = (uint64_t)((2 * s + h) * (SLOT2_BYTES >> 4));
              const uint64_t ad = a_desc0 + soff, bd = b_desc0 + soff;
              tc::mma_f16_ss_pair(d_tmem, ad, bd, idesc, (kb != kb0 || h) ? 1u : 0u);
#pragma unroll
              for (int kk = 1; kk < BK / 16; ++kk)
                tc::mma_f16_ss_pair(d_tmem, ad + kk * a_kstep, bd + kk * b_kstep, idesc, 1u);
              tc::mma_commit_pair(&empty_bar[2 * s + h], 0x3);
            }
            issued = true;
            if (++s == NPAIR2) { s = 0; ph ^= 1u; }
          }
          if (!ok) break;
          tc::mma_commit_pair(&tfull_bar[acc], 0x3);
          if (++acc == 2) { acc = 0; aph ^= 1u; }
        }
      }
      if (issued) {
        tc::mma_commit_pair(&drain_bar, 0x1);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&drain_bar, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
        }
      }
      SBP_TIMED(if (blockIdx.x == 0) printf(
          "SBPT ISSUE M %lld N %lld K %lld epi %d kblocks %d total %lld w_full %lld w_tempty %lld\n",
          (long long)M, (long long)N, (long long)K, g.epi, nkbt, clock64() - ti0, w_full,
          w_temp);)
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const int c_lo = ((warp - 2) >> 2) * (BN / 2);
    const uint32_t te_leader = tc::mapa(tc::smem_u32(&tempty_bar[0]), 0);
    int acc = 0;
    uint32_t aph = 0;
    SBP_TIMED(long long w_tf = 0, t_ep = 0, te0 = clock64(), c0;)
    for (int t = cluster; t < ntiles; t += nclusters) {
      int mt, nt;
      tile_coords(t, args.nM, args.nN, args.gm, mt, nt);
      const int64_t m0 = (int64_t)mt * BM2, n0 = (int64_t)nt * BN;
      if (m0 >= M) continue;
      bool ok = true;
      for (int b = 0; b < nblk; ++b) {
        SBP_TIMED(c0 = clock64();)
        if (!tc::mbar_wait_warp(&tfull_bar[acc], aph, abort_flag)) { ok = false; break; }
        SBP_TIMED(w_tf += clock64() - c0;)
        tc::fence_after_sync();
        const int64_t m = m0 + 128 * rank + row_in_tile;
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
        SBP_TIMED(c0 = clock64();)
        epilogue_tile(g, tbase, m, n0, M, N, imin(nk - b * kpb, kpb), c_lo, b);
        SBP_TIMED(t_ep += clock64() - c0;)
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(te_leader + (uint32_t)(acc * sizeof(uint64_t)));
        if (++acc == 2) { acc = 0; aph ^= 1u; }
      }
      if (!ok) break;
    }
    SBP_TIMED(if (blockIdx.x == 0 && (warp == 2 || warp == 9) && lane == 0) printf(
        "SBPT EPI warp %d M %lld N %lld K %lld epi %d total %lld w_tfull %lld work %lld\n", warp,
        (long long)M, (long long)N, (long long)K, g.epi, clock64() - te0, w_tf, t_ep);)
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();                        // no CTA leaves while its peer may still signal it
  tc::fence_after_sync();
  if (threadIdx.x == 0 && abort_sh && args.err) atomicExch(args.err, DEV_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map: inner dimension `inner` (contiguous), outer dimension `outer` with a
// stride of `ld` elements; box {64, box_outer}, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld,
              int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Row tiles per rasterisation group.  When all of A fits well inside L2 (126 MB), one group
// spans every row tile: each B column panel is then read from DRAM once while A stays
// resident (with groups of kGroupM rows, B is read once per group).  Otherwise groups of
// kGroupM rows keep the panels the CTAs share at one time small.
int group_rows(const GemmDesc& g, int nM) {
  constexpr int64_t kResidentA = 48ll << 20;
  return g.M * g.K * 2 <= kResidentA ? nM : kGroupM;
}

}  // namespace

int sm_count() {
  static int n = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  });
  return n;
}

// Can the tensor-core kernel take this GEMM?
bool gemm_tc_supported(const GemmDesc& g) {
  if (g.adt != DT_BF16 || g.bdt != DT_BF16) return false;
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return false;
  const bool a_k = g.sak == 1 && g.sam % 8 == 0 && g.sam > 0;
  const bool a_m = g.sam == 1 && g.sak % 8 == 0 && g.sak > 0;
  const bool b_k = g.sbk == 1 && g.sbn % 8 == 0 && g.sbn > 0;
  const bool b_n = g.sbn == 1 && g.sbk % 8 == 0 && g.sbk > 0;
  if (!(a_k || a_m) || !(b_k || b_n)) return false;
  if (!al16(g.A) || !al16(g.B)) return false;
  if (g.epi == EPI_STORE || g.epi == EPI_ACC || g.epi == EPI_CEGRAD ||
      g.epi == EPI_SWIGLU_BWD) {
    if (!al16(g.C) || g.ldc % 8 != 0) return false;
  }
  if (g.epi == EPI_SWIGLU_BWD &&
      (g.cdt != DT_BF16 || !al16(g.aux) || g.aux_ld % 8 != 0 || g.aux_off % 8 != 0))
    return false;
  if (g.epi == EPI_SWIGLU_FWD &&
      (g.cdt != DT_BF16 || !al16(g.C) || g.ldc % 8 != 0 || !al16(g.aux) || g.aux_ld % 8 != 0 ||
       !al16(g.C2) || g.ldc2 % 8 != 0 || g.kblk != 0))
    return false;
  if (g.epi == EPI_ROPE &&
      (g.cdt != DT_BF16 || !al16(g.C) || g.ldc % 8 != 0 || g.N % 128 != 0 || g.kblk != 0 ||
       g.r_Tc <= 0))
    return false;
  if (g.M > (int64_t)INT32_MAX || g.N > (int64_t)INT32_MAX || g.K > (int64_t)INT32_MAX)
    return false;
  return encode_fn() != nullptr;
}

cudaError_t gemm_tc(const GemmDesc& g, int* err, cudaStream_t st) {
  TcArgs args;
  args.g = g;
  args.a_mn = (g.sak == 1) ? 0 : 1;
  args.b_mn = (g.sbk == 1) ? 0 : 1;
  args.nM = (int)((g.M + BM - 1) / BM);
  args.nN = (int)((g.N + BN - 1) / BN);
  args.gm = group_rows(g, args.nM);
  args.err = err;
  CUtensorMap ma, mb;
  bool ok;
  if (!args.a_mn) ok = make_map(&ma, g.A, g.K, g.M, g.sam, BM);     // rows of K
  else ok = make_map(&ma, g.A, g.M, g.K, g.sak, 64);               // k-rows of M
  if (!ok) return cudaErrorInvalidValue;
  if (!args.b_mn) ok = make_map(&mb, g.B, g.K, g.N, g.sbn, BN);
  else ok = make_map(&mb, g.B, g.N, g.K, g.sbk, 64);
  if (!ok) return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int tiles = args.nM * args.nN;
  const int grid = tiles < sm_count() ? tiles : sm_count();
  launch(gemm_tc_kernel, grid, kThreads, SMEM_BYTES, st, ma, mb, args);
  return cudaGetLastError();
}


// The CTA-pair kernel: 256 x 256 tiles; B boxes hold 128 rows (half of N) per CTA.
cudaError_t gemm_tc_pair(const GemmDesc& g, int* err, cudaStream_t st) {
  if (g.kblk % BK2 != 0) return cudaErrorNotSupported;   // K blocks are whole stages
  TcArgs args;
  args.g = g;
  args.a_mn = (g.sak == 1) ? 0 : 1;
  args.b_mn = (g.sbk == 1) ? 0 : 1;
  args.nM = (int)((g.M + BM2 - 1) / BM2);
  args.nN = (int)((g.N + BN - 1) / BN);
  args.gm = group_rows(g, args.nM);
  args.err = err;
  CUtensorMap ma, mb;
  bool ok;
  if (!args.a_mn) ok = make_map(&ma, g.A, g.K, g.M, g.sam, 128);
  else ok = make_map(&ma, g.A, g.M, g.K, g.sak, 64);
  if (!ok) return cudaErrorInvalidValue;
  if (!args.b_mn) ok = make_map(&mb, g.B, g.K, g.N, g.sbn, 128);
  else ok = make_map(&mb, g.B, g.N, g.K, g.sbk, 64);
  if (!ok) return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    SMEM2_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int tiles = args.nM * args.nN;
  const int pairs = sm_count() / 2;
  const int grid = 2 * (tiles < pairs ? tiles : pairs);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM2_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_count_launch();
  return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel, ma, mb, args);
}

}  // namespace sbp
