// Causal GQA attention backward of one query chunk over its key prefix on the tcgen05 tensor
// cores (head_dim 128, bf16 operands, fp32 accumulation).
//
// One CTA owns (sequence b, KV head g, 128-key tile kt) and loops over the query heads of g's
// group and the chunk's query tiles that can see those keys.  Per (query head, query tile):
//   S^T  = K Q^T            (TMEM cols [0,128))      dP^T = V dO^T   (TMEM cols [128,256))
//   P^T  = exp(S^T * scale - lse) -> bf16, written back into TMEM over the dP^T columns the
//          same warp has already read (the A operand of the next product, read from TMEM)
//   dS^T = P^T (dP^T - delta)     -> bf16 tile in shared memory
//   dV  += P^T dO           (TMEM cols [256,384))    dK  += dS^T Q   (TMEM cols [384,512))
//   dQ   = dS K             (TMEM cols [0,128) again) -> added to the fp32 dQ in global memory
// Q and dO go through a two-stage ring, so the next pair's tiles load during this pair.
// dK and dV stay in TMEM for the whole loop and are added once into the fp32 prefix
// accumulators (single owner: deterministic); dQ receives one vector atomic add per query tile
// and key tile.  Entries with key > query, queries outside the chunk and keys outside the
// prefix are masked by selection (not by multiplication), so stale values there never reach
// an accumulator.
//
// Warp roles: warp 0 TMA producer (K, V once; Q and dO per pair), warp 1 TMEM owner + MMA
// issuer, warps 2..9 element-wise + TMEM read-out (thread = key row, or query row for dQ; the
// warp's lane quarter is fixed by its index mod 4, the two warps of a quarter split the 128
// columns in halves).
#include <cuda.h>

#include <mutex>

#include "sbp_internal.cuh"
#include "tc_ptx.cuh"

namespace sbp {

namespace {

constexpr int HD = 128;
constexpr int BT = 128;                     // keys per key tile, queries per query tile
constexpr int TILE = 128 * HD * 2;          // 32 KB bf16 tile: two 64-column swizzled chunks
constexpr int CHUNK = TILE / 2;
constexpr int QD_STAGES = 2;
constexpr int SMEM_BYTES = (3 + 2 * QD_STAGES) * TILE + 1024;  // K, V, dS^T, 2 x (Q, dO)
constexpr int kEwWarps = 8;                 // element-wise warps: 4 lane quarters x 2 column halves
constexpr int kThreads = 64 + 32 * kEwWarps;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t C_S = 0, C_DP = 128, C_DV = 256, C_DK = 384;

struct BwdArgs {
  int64_t B, T, Tc, s, H, Hkv;
  int nq, nkt;
  const float* lse;     // [B*Tc, H] natural log
  const float* delta;   // [B*Tc, H]
  float* dq;            // [B*Tc, H, HD] fp32, accumulated
  float* dKp;           // [B, T, Hkv, HD] fp32, accumulated
  float* dVp;
  float scale;          // 1 / sqrt(hd)
  int* err;
};

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ void st_unit(uint8_t* tile, int r, int u, uint4 v) {
  const int chunk = u >> 3, uu = u & 7;
  *reinterpret_cast<uint4*>(tile + chunk * CHUNK + r * 128 + ((uu ^ (r & 7)) << 4)) = v;
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, f32 accumulate (A: 128 lanes x K/2 columns of
// packed bf16 pairs, K-major).
__device__ __forceinline__ void mma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Bounded barrier of the element-wise warps (an mbarrier with one arrival per warp that
// completes once per use), so that a warp that gave up on a wait cannot strand the others.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t parity, int lane,
                                           volatile int* abort_flag) {
  __syncwarp();
  if (lane == 0) tc::mbar_arrive(bar);
  return tc::mbar_wait_warp(bar, parity, abort_flag);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                   const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t kv_full, qd_full[QD_STAGES], qd_empty[QD_STAGES], sdp_full, ds_full,
      mma2_done, dq_free, drain;
  __shared__ uint64_t sync_a, sync_b;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  __shared__ __align__(16) float lse_s[BT];
  __shared__ __align__(16) float delta_s[BT];

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + TILE;
  uint8_t* sdSt = sV + TILE;
  uint8_t* sQ0 = sdSt + TILE;                    // stage st: Q at sQ0 + 2 st TILE, dO after it
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &abort_sh;

  // work decomposition: early key tiles (the most query tiles) first
  const int kt = (int)(blockIdx.x % a.nkt);
  const int64_t g = (blockIdx.x / a.nkt) % a.Hkv;
  const int64_t b = blockIdx.x / (a.nkt * a.Hkv);
  const int64_t grp = a.H / a.Hkv;
  const int64_t e = a.s + a.Tc;                  // prefix end
  const int64_t k_lo = (int64_t)kt * BT;
  // first query tile whose last row can see key k_lo
  int64_t i0 = (k_lo - a.s - (BT - 1) + (BT - 1)) / BT;
  if (k_lo - a.s - (BT - 1) <= 0) i0 = 0;
  const int nqt = (int)(a.nq - i0);              // query tiles per head
  const int npairs = nqt > 0 ? (int)(grp * nqt) : 0;

  if (threadIdx.x == 0) {
    tc::mbar_init(&kv_full, 1);
    for (int i = 0; i < QD_STAGES; ++i) {
      tc::mbar_init(&qd_full[i], 1);
      tc::mbar_init(&qd_empty[i], 1);
    }
    tc::mbar_init(&sdp_full, 1);
    tc::mbar_init(&ds_full, kEwWarps);
    tc::mbar_init(&mma2_done, 1);
    tc::mbar_init(&dq_free, kEwWarps);
    tc::mbar_init(&drain, 1);
    tc::mbar_init(&sync_a, kEwWarps);
    tc::mbar_init(&sync_b, kEwWarps);
    abort_sh = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&tmem_sh, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_sh;

  auto pair_coords = [&](int j, int64_t& hh, int64_t& qi) {
    hh = g * grp + j / nqt;
    qi = i0 + j % nqt;
  };

  if (warp == 0) {
    if (lane == 0 && npairs > 0) {
      // ---------------------------------------------------------------- producer
      const int32_t krow = (int32_t)(b * a.T + k_lo);
      tc::mbar_expect_tx(&kv_full, 2 * TILE);
      tc::tma_load_3d(sK, &tmK, &kv_full, 0, (int32_t)g, krow);
      tc::tma_load_3d(sK + CHUNK, &tmK, &kv_full, 64, (int32_t)g, krow);
      tc::tma_load_3d(sV, &tmV, &kv_full, 0, (int32_t)g, krow);
      tc::tma_load_3d(sV + CHUNK, &tmV, &kv_full, 64, (int32_t)g, krow);
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < npairs; ++j) {
        int64_t hh, qi;
        pair_coords(j, hh, qi);
        const int st = j % QD_STAGES;
        const uint32_t ph = (uint32_t)(j / QD_STAGES) & 1u;
        if (!tc::mbar_wait(&qd_empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* sQ = sQ0 + 2 * st * TILE;
        uint8_t* sdO = sQ + TILE;
        const int32_t qrow = (int32_t)(b * a.Tc + qi * BT);
        tc::mbar_expect_tx(&qd_full[st], 2 * TILE);
        tc::tma_load_3d(sQ, &tmQ, &qd_full[st], 0, (int32_t)hh, qrow);
        tc::tma_load_3d(sQ + CHUNK, &tmQ, &qd_full[st], 64, (int32_t)hh, qrow);
        tc::tma_load_3d(sdO, &tmdO, &qd_full[st], 0, (int32_t)hh, qrow);
        tc::tma_load_3d(sdO + CHUNK, &tmdO, &qd_full[st], 64, (int32_t)hh, qrow);
        issued = j + 1;
      }
      if (!ok) {
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&kv_full, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        for (int j = issued > QD_STAGES ? issued - QD_STAGES : 0; j < issued; ++j)
          while (!tc::mbar_try_wait(&qd_full[j % QD_STAGES], (uint32_t)(j / QD_STAGES) & 1u) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && npairs > 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t id_kk = tc::idesc_bf16_f32(128, 128, 0, 0);   // A K-major, B K-major
      const uint32_t id_km = tc::idesc_bf16_f32(128, 128, 0, 1);   // A K-major, B MN-major
      const uint32_t id_mm = tc::idesc_bf16_f32(128, 128, 1, 1);   // A MN-major, B MN-major
      const uint32_t aK = tc::smem_u32(sK), aV = tc::smem_u32(sV), adS = tc::smem_u32(sdSt),
                     aQ0 = tc::smem_u32(sQ0);
      bool ok = tc::mbar_wait(&kv_full, 0, abort_flag);
      bool issued = false;
      for (int j = 0; j < npairs && ok; ++j) {
        const uint32_t ph = (uint32_t)j & 1u;
        const int st = j % QD_STAGES;
        const uint32_t sph = (uint32_t)(j / QD_STAGES) & 1u;
        const uint32_t aQ = aQ0 + 2 * st * TILE, adO = aQ + TILE;
        if (!tc::mbar_wait(&qd_full[st], sph, abort_flag)) { ok = false; break; }
        if (j >= 1 && !tc::mbar_wait(&dq_free, ph ^ 1u, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // K = head dim
          const uint32_t off = (kk >> 2) * CHUNK + (kk & 3) * 32;
          tc::mma_f16_ss(tmem + C_S, tc::smem_desc_sw128(aK + off, 16, 1024),
                         tc::smem_desc_sw128(aQ + off, 16, 1024), id_kk, kk != 0);
          tc::mma_f16_ss(tmem + C_DP, tc::smem_desc_sw128(aV + off, 16, 1024),
                         tc::smem_desc_sw128(adO + off, 16, 1024), id_kk, kk != 0);
        }
        issued = true;
        tc::mma_commit(&sdp_full);
        if (!tc::mbar_wait(&ds_full, ph, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // K = queries for dV, dK; keys for dQ
          const uint32_t offk = (kk >> 2) * CHUNK + (kk & 3) * 32;   // K-major operand step
          const uint32_t offm = kk * 2048;                            // MN-major operand step
          const uint32_t acc = (j | kk) != 0;
          // P^T (packed bf16) sits in TMEM: queries 64h.. of half h at C_DP + 64 h
          const uint32_t pcol = C_DP + 64 * (kk >> 2) + 8 * (kk & 3);
          mma_f16_ts(tmem + C_DV, tmem + pcol, tc::smem_desc_sw128(adO + offm, CHUNK, 1024),
                     id_km, acc);
          tc::mma_f16_ss(tmem + C_DK, tc::smem_desc_sw128(adS + offk, 16, 1024),
                         tc::smem_desc_sw128(aQ + offm, CHUNK, 1024), id_km, acc);
          tc::mma_f16_ss(tmem + C_S, tc::smem_desc_sw128(adS + offm, CHUNK, 1024),
                         tc::smem_desc_sw128(aK + offm, CHUNK, 1024), id_mm, kk != 0);
        }
        tc::mma_commit(&mma2_done);
        tc::mma_commit(&qd_empty[st]);
      }
      if (issued) {
        tc::mma_commit(&drain);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&drain, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (npairs > 0) {
    // ------------------------------------------------------------------ element-wise warps
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;                // column half of this warp
    const int r = q4 * 32 + lane;                    // TMEM lane = key row (or query row)
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int kpos = (int)(k_lo + r);
    const float scale_log2 = a.scale * 1.4426950408889634f;
    const int tid = threadIdx.x - 64;                // 0..255
    const int e32 = (int)e;
    bool ok = true;
    for (int j = 0; j < npairs; ++j) {
      const uint32_t ph = (uint32_t)j & 1u;
      int64_t hh, qi;
      pair_coords(j, hh, qi);
      const int q0 = (int)(a.s + qi * BT);           // absolute position of query column 0
      // no masking needed when every key of the tile precedes every (valid) query of the tile
      const bool full = (k_lo + BT - 1 <= q0) && (qi * BT + BT <= a.Tc);
      // per-query statistics of this pair (thread tid < 128 loads query column tid)
      if (!group_sync(&sync_a, ph, lane, abort_flag)) { ok = false; break; }
      if (tid < BT) {
        const int64_t ql = qi * BT + tid;           // position within the chunk
        const bool qv = ql < a.Tc;
        const int64_t gi = (b * a.Tc + ql) * a.H + hh;
        lse_s[tid] = qv ? a.lse[gi] * 1.4426950408889634f : 0.f;
        delta_s[tid] = qv ? a.delta[gi] : 0.f;
      }
      if (!group_sync(&sync_b, ph, lane, abort_flag)) { ok = false; break; }
      if (!tc::mbar_wait_warp(&sdp_full, ph, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = half * 2 + cc;                 // 32-column slice
        uint32_t rs[32], rd[32];
        tc::tmem_ld32(tmem + lane_off + C_S + c * 32, rs);
        tc::tmem_ld32(tmem + lane_off + C_DP + c * 32, rd);
        tc::tmem_ld_wait();
        uint32_t pp[16], dd[16];
        const float4* l4 = reinterpret_cast<const float4*>(lse_s + c * 32);
        const float4* d4 = reinterpret_cast<const float4*>(delta_s + c * 32);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 lv = l4[i4], dv = d4[i4];
          const float la[4] = {lv.x, lv.y, lv.z, lv.w};
          const float da[4] = {dv.x, dv.y, dv.z, dv.w};
          float p[4], g[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int i = i4 * 4 + k;
            p[k] = ex2(fmaf(__uint_as_float(rs[i]), scale_log2, -la[k]));
            g[k] = p[k] * (__uint_as_float(rd[i]) - da[k]);
            if (!full) {
              const int qpos = q0 + c * 32 + i;
              const bool live = (kpos <= qpos) && (qpos < e32);
              p[k] = live ? p[k] : 0.f;
              g[k] = live ? g[k] : 0.f;
            }
          }
          pp[i4 * 2] = pack2(p[0], p[1]);
          pp[i4 * 2 + 1] = pack2(p[2], p[3]);
          dd[i4 * 2] = pack2(g[0], g[1]);
          dd[i4 * 2 + 1] = pack2(g[2], g[3]);
        }
        // packed P over dP^T columns this warp has already read (queries 32 cc .. of its half)
        tmem_st16(tmem + lane_off + C_DP + 64 * half + 16 * cc, pp);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_unit(sdSt, r, c * 4 + u, make_uint4(dd[4 * u], dd[4 * u + 1], dd[4 * u + 2], dd[4 * u + 3]));
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ds_full);
      // dQ of this query tile: TMEM lane r = query row r
      if (!tc::mbar_wait_warp(&mma2_done, ph, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      {
        const int64_t ql = qi * BT + r;
        const bool qv = ql < a.Tc;
        float* dqp = a.dq + ((b * a.Tc + ql) * a.H + hh) * HD;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const int c = half * 2 + cc;
          uint32_t rq[32];
          tc::tmem_ld32(tmem + lane_off + C_S + c * 32, rq);
          tc::tmem_ld_wait();
          if (qv) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 v = make_float4(__uint_as_float(rq[i]) * a.scale,
                                     __uint_as_float(rq[i + 1]) * a.scale,
                                     __uint_as_float(rq[i + 2]) * a.scale,
                                     __uint_as_float(rq[i + 3]) * a.scale);
              atomicAdd(reinterpret_cast<float4*>(dqp + c * 32 + i), v);
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&dq_free);
    }
    // dK, dV of this key tile: add into the fp32 prefix accumulators (single owner)
    if (ok) {
      const bool kv = kpos < e32;
      const int64_t ko = ((b * a.T + kpos) * a.Hkv + g) * HD;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = half * 2 + cc;
        uint32_t rk[32], rv[32];
        tc::tmem_ld32(tmem + lane_off + C_DK + c * 32, rk);
        tc::tmem_ld32(tmem + lane_off + C_DV + c * 32, rv);
        tc::tmem_ld_wait();
        if (kv) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4* pk = reinterpret_cast<float4*>(a.dKp + ko + c * 32 + i);
            float4* pv = reinterpret_cast<float4*>(a.dVp + ko + c * 32 + i);
            float4 x = *pk, y = *pv;
            x.x += __uint_as_float(rk[i]) * a.scale;
            x.y += __uint_as_float(rk[i + 1]) * a.scale;
            x.z += __uint_as_float(rk[i + 2]) * a.scale;
            x.w += __uint_as_float(rk[i + 3]) * a.scale;
            y.x += __uint_as_float(rv[i]);
            y.y += __uint_as_float(rv[i + 1]);
            y.z += __uint_as_float(rv[i + 2]);
            y.w += __uint_as_float(rv[i + 3]);
            *pk = x;
            *pv = y;
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && abort_sh && a.err) atomicExch(a.err, DEV_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// delta[r, h] = sum_d dO[r, h, d] * O[r, h, d]  (one warp per (row, head))
__global__ void attn_delta_kernel(int64_t rows_heads, const __nv_bfloat16* __restrict__ dO,
                                  const __nv_bfloat16* __restrict__ o, float* __restrict__ delta) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= rows_heads) return;
  const __nv_bfloat16* a = dO + w * HD;
  const __nv_bfloat16* c = o + w * HD;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < HD / 32; ++i)
    s = fmaf(__bfloat162float(a[lane + 32 * i]), __bfloat162float(c[lane + 32 * i]), s);
  s = warp_sum(s);
  if (lane == 0) delta[w] = s;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_bwd() {
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

bool map3(CUtensorMap* map, const void* base, int64_t heads, int64_t rows) {
  EncodeTiledFn fn = encode_fn_bwd();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)heads * HD * 2};
  cuuint32_t box[3] = {64u, 1u, 128u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_bwd_tc_supported(int64_t hd, int dt, const void* q, const void* Kp, const void* Vp,
                           const void* o, const void* dO, const float* dq) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return hd == HD && dt == DT_BF16 && al(q) && al(Kp) && al(Vp) && al(o) && al(dO) && al(dq) &&
         encode_fn_bwd() != nullptr;
}

// dq [B*Tc, H, HD] fp32 is overwritten; dKp/dVp [B, T, Hkv, HD] fp32 accumulate rows < s + Tc.
cudaError_t attn_bwd_tc(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                        const void* q, const void* Kp, const void* Vp, const void* o,
                        const void* dO, const float* lse, float* delta, float* dq, float* dKp,
                        float* dVp, int* err, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mdo;
  if (!map3(&mq, q, H, B * Tc) || !map3(&mk, Kp, Hkv, B * T) || !map3(&mv, Vp, Hkv, B * T) ||
      !map3(&mdo, dO, H, B * Tc))
    return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES);
  });
  if (attr != cudaSuccess) return attr;
  const int64_t rh = B * Tc * H;
  cudaError_t e = cudaMemsetAsync(dq, 0, sizeof(float) * (size_t)rh * HD, st);
  if (e != cudaSuccess) return e;
  launch(attn_delta_kernel, dim3((unsigned)((rh * 32 + 255) / 256)), dim3(256), 0, st, rh,
         static_cast<const __nv_bfloat16*>(dO), static_cast<const __nv_bfloat16*>(o), delta);
  BwdArgs a;
  a.B = B; a.T = T; a.Tc = Tc; a.s = s; a.H = H; a.Hkv = Hkv;
  a.nq = (int)((Tc + BT - 1) / BT);
  a.nkt = (int)((s + Tc + BT - 1) / BT);
  a.lse = lse;
  a.delta = delta;
  a.dq = dq;
  a.dKp = dKp;
  a.dVp = dVp;
  a.scale = 1.f / sqrtf((float)HD);
  a.err = err;
  const int64_t grid = B * Hkv * a.nkt;
  launch(attn_bwd_tc_kernel, dim3((unsigned)grid), dim3(kThreads), (size_t)SMEM_BYTES, st, mq, mk,
         mv, mdo, a);
  return cudaGetLastError();
}

}  // namespace sbp
