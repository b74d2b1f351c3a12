// Causal GQA attention forward of one query chunk over its key prefix on the tcgen05 tensor
// cores (head_dim 128, bf16 operands, fp32 softmax statistics and accumulation).
//
// One CTA per (sequence b, query head h, pair of adjacent 128-row query tiles).  The two tiles
// share every K / V tile the CTA loads and take turns on the tensor cores: while one tile's
// softmax warps turn its scores into probabilities, the tensor cores run the other tile's
// products, so neither the tensor pipe nor the exponential unit waits for the other.
//   warp 0      : TMA producer (both Q tiles once; K and V tiles of 128 keys through 2-stage
//                 rings, one load per key tile for both query tiles)
//   warp 1      : TMEM owner + MMA issuer, in the order
//                   S0_j S1_j | PV0_j S0_{j+1} PV1_j S1_{j+1} | PV0_{j+1} ...
//                 S_t = Q_t K_j^T into tile t's score columns; PV_t: O_t += P_t V_j with P_t
//                 read from TMEM (written by the softmax over the scores it replaces)
//   warps 2..5  : softmax of tile 0, warps 6..9: softmax of tile 1, one thread per query row:
//                 read S from TMEM, causal mask, online max / sum in the exp2 domain, P (bf16)
//                 back into TMEM, lazy rescale of O in TMEM, final O / l and log-sum-exp.
// The running maximum used as the exponent reference is only raised when the row maximum
// exceeds it by more than 2^8 (P <= 256), so O is rescaled rarely; the result is exact up to
// rounding because P, l and O share that reference.
// Key tiles are visited in order 0, 1, ... up to each query tile's diagonal; masked entries
// are exactly zero, so each query row's result does not depend on how the sequence was
// chunked (or on which tile of a pair it sits in).
// Ordering: S_t(j + 1) is issued after PV_t(j), whose P it overwrites; the tensor cores run a
// CTA's MMAs in issue order, and the commit that signals S_t(j + 1) also covers PV_t(j), so a
// softmax warp that has seen S_t(j + 1) may rescale O_t.
// Key-range split: a chunk of 4096 queries has 32 heads x 16 pairs = 512 CTAs of nearly equal
// work, 3.46 waves of the 148 SMs.  Pairs whose keys reach past a quarter of the sequence
// (key tile segt, fixed by the sequence length) therefore run as two CTAs, one per segment
// [0, segt) and [segt, end), the heavier segments launched first.  The CTA that finishes second combines both partials (maximum,
// sum, unnormalised O) in segment order, the other parks its partial in scratch; a row whose
// keys all precede the split gets exactly the unsplit result (its second partial is empty), and
// the split point does not depend on the chunking, so each row's result is still the same at
// every D.
#include <cuda.h>

#include <mutex>

#include "sbp_internal.cuh"
#include "tc_ptx.cuh"

namespace sbp {

namespace {

constexpr int HD = 128;                 // head dim handled by this kernel
constexpr int BQ = 128, BKV = 128;      // query rows / keys per tile
constexpr int TILE_BYTES = 128 * HD * 2;  // 32 KB: a 128 x 128 bf16 tile (two 64-wide chunks)
constexpr int CHUNK_BYTES = TILE_BYTES / 2;
constexpr int KV_STAGES = 2;
constexpr int SMEM_BYTES = 2 * TILE_BYTES                // Q0, Q1
                           + 2 * KV_STAGES * TILE_BYTES  // K, V rings
                           + 1024;                     // alignment slack
constexpr int kSoftmaxWarps = 8;        // two warpgroups, one per query tile
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;
constexpr uint32_t TMEM_COLS = 512;     // S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512)
constexpr uint32_t O_COL = 256;
constexpr float kRescaleThreshold = 8.f;  // log2 units

struct FwdArgs {
  int64_t B, T, Tc, s, H, Hkv;
  int nq;                 // query tiles per sequence
  int np;                 // query-tile pairs per sequence
  void* o;                // [B*Tc, H, HD] bf16
  float* lse;             // [B*Tc, H]  natural log
  float scale_log2;       // log2(e) / sqrt(hd)
  int* err;
  // Key-range split (segt > 0): a pair whose keys reach past key tile segt runs as two CTAs,
  // keys [0, 128 segt) and [128 segt, end); units = pairs of the launch (the grid is 2 units).
  int segt, units;
  int seg1_first;         // the grid's first half runs the second segments (the heavier ones)
  float* part;            // [B*Tc, H, HD] fp32: the first-finished segment's unnormalised O
  float* ml;              // [B*Tc, H, 2]: its running maximum (log2 units) and sum
  int* flags;             // [units, 2]: finish counter, partial-ready flag (zeroed per launch)
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
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

// max(a, b, c) in one instruction (the three-input form of max.f32; a NaN input is ignored,
// as fmaxf does)
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

// D[tmem] (+)= A[tmem] * B[smem], bf16 inputs, f32 accumulate (A: 128 lanes x K/2 columns of
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

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full, k_full[KV_STAGES], k_empty[KV_STAGES], v_full[KV_STAGES],
      v_empty[KV_STAGES], s_full[2], p_full[2], o_done[2], drain_bar, sm_sync;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh, role_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                  // tile t at sQ + t * TILE_BYTES
  uint8_t* sK = sQ + 2 * TILE_BYTES;
  uint8_t* sV = sK + KV_STAGES * TILE_BYTES;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &abort_sh;

  // heavy (late) query-tile pairs first, and the heavier segment of the split pairs first
  const int unit = (int)(blockIdx.x % (unsigned)a.units);
  const int seg = (int)(blockIdx.x / (unsigned)a.units) ^ a.seg1_first;
  const int qp = a.np - 1 - (unit % a.np);
  const int64_t h = (unit / a.np) % a.H;
  const int64_t b = unit / (a.np * a.H);
  const int64_t g = h / (a.H / a.Hkv);
  const bool has1 = 2 * qp + 1 < a.nq;
  int nkv_t[2];
  int64_t q_lo_t[2], q_hi_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = 2 * qp + t;
    q_lo_t[t] = a.s + (int64_t)qt * BQ;                            // position of row 0
    q_hi_t[t] = a.s + imin((int64_t)(qt + 1) * BQ, a.Tc);          // one past the last row
    nkv_t[t] = (t == 1 && !has1) ? 0 : (int)((q_hi_t[t] + BKV - 1) / BKV);
  }
  // The key range is split at the fixed key tile segt (a function of the sequence length
  // only), so each query row's two partial results do not depend on the chunking; a row that
  // sees no key past the split gets exactly its unsplit result.  From here on nkv_t counts the
  // key tiles of this CTA's segment, from key tile j0.
  const bool split = a.segt > 0 && (nkv_t[0] > a.segt || nkv_t[1] > a.segt);
  if (seg == 1 && !split) return;                  // whole CTA, before any set-up
  const int j0 = (split && seg == 1) ? a.segt : 0;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int end = (split && seg == 0) ? imin(nkv_t[t], a.segt) : nkv_t[t];
    nkv_t[t] = end > j0 ? end - j0 : 0;
  }
  const int nkv = nkv_t[0] > nkv_t[1] ? nkv_t[0] : nkv_t[1];     // key tiles j0 .. j0+nkv-1

  if (threadIdx.x == 0) {
    tc::mbar_init(&q_full, 1);
    for (int i = 0; i < KV_STAGES; ++i) {
      tc::mbar_init(&k_full[i], 1);
      tc::mbar_init(&k_empty[i], 1);
      tc::mbar_init(&v_full[i], 1);
      tc::mbar_init(&v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      tc::mbar_init(&s_full[t], 1);
      tc::mbar_init(&p_full[t], kSoftmaxWarps / 2);
      tc::mbar_init(&o_done[t], 1);
    }
    tc::mbar_init(&drain_bar, 1);
    tc::mbar_init(&sm_sync, kSoftmaxWarps);
    abort_sh = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      bool ok = true;
      const int32_t qrow = (int32_t)(b * a.Tc + (int64_t)(2 * qp) * BQ);
      tc::mbar_expect_tx(&q_full, (has1 ? 2 : 1) * TILE_BYTES);
      for (int t = 0; t < (has1 ? 2 : 1); ++t) {
        tc::tma_load_3d(sQ + t * TILE_BYTES, &tmQ, &q_full, 0, (int32_t)h, qrow + t * BQ);
        tc::tma_load_3d(sQ + t * TILE_BYTES + CHUNK_BYTES, &tmQ, &q_full, 64, (int32_t)h,
                        qrow + t * BQ);
      }
      uint32_t issued = 0;
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t ph = (uint32_t)(j / KV_STAGES) & 1u;
        const int32_t krow = (int32_t)(b * a.T + (int64_t)(j0 + j) * BKV);
        if (!tc::mbar_wait(&k_empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
        tc::mbar_expect_tx(&k_full[st], TILE_BYTES);
        tc::tma_load_3d(sK + st * TILE_BYTES, &tmK, &k_full[st], 0, (int32_t)g, krow);
        tc::tma_load_3d(sK + st * TILE_BYTES + CHUNK_BYTES, &tmK, &k_full[st], 64, (int32_t)g,
                        krow);
        if (!tc::mbar_wait(&v_empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
        tc::mbar_expect_tx(&v_full[st], TILE_BYTES);
        tc::tma_load_3d(sV + st * TILE_BYTES, &tmV, &v_full[st], 0, (int32_t)g, krow);
        tc::tma_load_3d(sV + st * TILE_BYTES + CHUNK_BYTES, &tmV, &v_full[st], 64, (int32_t)g,
                        krow);
        issued = (uint32_t)j + 1;
      }
      if (!ok) {
        // bounded drain of this CTA's own copies
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&q_full, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        for (uint32_t j = issued > KV_STAGES ? issued - KV_STAGES : 0; j < issued; ++j) {
          const int st = (int)(j % KV_STAGES);
          const uint32_t ph = (j / KV_STAGES) & 1u;
          while (!tc::mbar_try_wait(&k_full[st], ph) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
          while (!tc::mbar_try_wait(&v_full[st], ph) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1) {
    {
      // ---------------------------------------------------------------- MMA issuer
      // the whole warp runs the issue loop (waits, bookkeeping); one elected lane issues the
      // MMAs and commits: a lone lane in a divergent branch gets far fewer issue slots while
      // the softmax warps of its sub-partition issue back to back.  The lane is elected at each
      // use (the same lane every time, the warp being converged), which keeps a register free.
      const uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);   // Q K^T: both K-major
      const uint32_t id_o = tc::idesc_bf16_f32(128, 128, 0, 1);   // P V: V is MN-major
      const uint32_t aQ = tc::smem_u32(sQ), aK = tc::smem_u32(sK), aV = tc::smem_u32(sV);
      // shared-memory descriptors built once; a k-step, a query tile or a ring stage adds its
      // byte offset / 16 to the start address field (the tiles sit below 256 KB)
      static_assert(KV_STAGES == 2, "stage descriptors are selected between two stages");
      const uint64_t dQ0 = tc::smem_desc_sw128(aQ, 16, 1024);
      const uint64_t dK0 = tc::smem_desc_sw128(aK, 16, 1024);
      const uint64_t dV0 = tc::smem_desc_sw128(aV, CHUNK_BYTES, 1024);
      constexpr uint64_t kTile = (uint64_t)(TILE_BYTES >> 4);
      bool ok = tc::mbar_wait_warp(&q_full, 0, abort_flag);
      bool issued = false;
      int k_waited = -1;                 // last key tile whose K load this thread has seen
      auto wait_k = [&](int j) -> bool {
        if (k_waited >= j) return true;
        if (!tc::mbar_wait_warp(&k_full[j % KV_STAGES], (uint32_t)(j / KV_STAGES) & 1u,
                                abort_flag))
          return false;
        tc::fence_after_sync();
        k_waited = j;
        return true;
      };
      // S_t(j) = Q_t K_j^T
      auto scores = [&](int t, int j) {
        const uint64_t kb = dK0 + ((j % KV_STAGES) ? kTile : 0);
        const uint64_t qb = dQ0 + (t ? kTile : 0);
        if (tc::elect_one_sync()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * CHUNK_BYTES + (kk & 3) * 32) >> 4);
            tc::mma_f16_ss(tmem + (uint32_t)(t * 128), qb + off, kb + off, id_s,
                           kk != 0 ? 1u : 0u);
          }
          tc::mma_commit(&s_full[t]);
        }
        __syncwarp();
        issued = true;
      };
      // O_t += P_t(j) V_j; P_t packed two keys per column over S_t's first 64 columns
      auto pv = [&](int t, int j) -> bool {
        if (!tc::mbar_wait_warp(&p_full[t], (uint32_t)j & 1u, abort_flag)) return false;
        tc::fence_after_sync();
        const uint64_t vb = dV0 + ((j % KV_STAGES) ? kTile : 0);
        if (tc::elect_one_sync()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ts(tmem + O_COL + (uint32_t)(t * 128), tmem + (uint32_t)(t * 128 + 8 * kk),
                       vb + (uint64_t)((kk * 2048) >> 4), id_o, (j | kk) != 0 ? 1u : 0u);
          if (j == (t ? nkv_t[1] : nkv_t[0]) - 1) tc::mma_commit(&o_done[t]);
        }
        __syncwarp();
        return true;
      };
      if (ok && nkv > 0) {
        ok = wait_k(0);
        if (ok) {
          if (nkv_t[0] > 0) scores(0, 0);
          if (nkv_t[1] > 0) scores(1, 0);
          if (tc::elect_one_sync()) tc::mma_commit(&k_empty[0]);
        }
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % KV_STAGES;
        if (!tc::mbar_wait_warp(&v_full[st], (uint32_t)(j / KV_STAGES) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const bool more = j + 1 < nkv;
        if (j < nkv_t[0]) {
          if (!pv(0, j)) { ok = false; break; }
        }
        if (j + 1 < nkv_t[0]) {
          if (!wait_k(j + 1)) { ok = false; break; }
          scores(0, j + 1);
        }
        if (j < nkv_t[1]) {
          if (!pv(1, j)) { ok = false; break; }
        }
        if (tc::elect_one_sync()) tc::mma_commit(&v_empty[st]);
        if (j + 1 < nkv_t[1]) {
          if (!wait_k(j + 1)) { ok = false; break; }
          scores(1, j + 1);
        }
        if (more) {
          // every product that reads K_{j+1} is issued (a tile past its diagonal reads none)
          if (!wait_k(j + 1)) { ok = false; break; }
          if (tc::elect_one_sync()) tc::mma_commit(&k_empty[(j + 1) % KV_STAGES]);
        }
      }
      if (issued) {
        if (tc::elect_one_sync()) tc::mma_commit(&drain_bar);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&drain_bar, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int t = (warp - 2) >> 2;                // query tile of this warpgroup
    const int q4 = warp & 3;                      // TMEM lane quarter
    const int r = q4 * 32 + lane;                 // query row within the tile
    const int64_t q_lo = t ? q_lo_t[1] : q_lo_t[0], q_hi = t ? q_hi_t[1] : q_hi_t[0];
    const int64_t tq = q_lo + r;                  // absolute position
    const int n_kv = t ? nkv_t[1] : nkv_t[0];
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_col = (uint32_t)(t * 128), o_col = O_COL + (uint32_t)(t * 128);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!tc::mbar_wait_warp(&s_full[t], (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      float sv[128];
      {
        // the four 32-column loads in flight together, one wait
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tc::tmem_ld32(tmem + lane_off + s_col, r0);
        tc::tmem_ld32(tmem + lane_off + s_col + 32u, r1);
        tc::tmem_ld32(tmem + lane_off + s_col + 64u, r2);
        tc::tmem_ld32(tmem + lane_off + s_col + 96u, r3);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sv[i] = __uint_as_float(r0[i]);
          sv[32 + i] = __uint_as_float(r1[i]);
          sv[64 + i] = __uint_as_float(r2[i]);
          sv[96 + i] = __uint_as_float(r3[i]);
        }
      }
      // row maximum of the raw scores (the scale is positive and rounding is monotonic, so
      // the scaled maximum equals the maximum of the scaled scores); the scale is folded into
      // the exponent's FMA below.  Only tiles that reach past the first query need the causal
      // mask (masked scores become -inf).
      const int64_t k0 = (int64_t)(j0 + j) * BKV;
      const bool diag = k0 + BKV - 1 > q_lo;
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (diag) {
        const int lim = (int)(tq - k0);            // keys k0 + i with i > lim are masked
#pragma unroll
        for (int i = 0; i < 128; ++i) sv[i] = (i <= lim) ? sv[i] : -INFINITY;
      }
#pragma unroll
      for (int i = 0; i < 128; i += 2) m4[(i >> 1) & 3] = fmax3f(m4[(i >> 1) & 3], sv[i], sv[i + 1]);
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.scale_log2;
      float corr = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleThreshold) {
        corr = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mx);
        rescale = (j > 0);
        m_ref = mx;
        l *= corr;
      }
      // a row that has seen no key yet (only in a second segment: its keys all precede the
      // split) keeps P = 0 instead of exp2(-inf + inf)
      const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = fast_exp2(fmaf(sv[32 * c + 2 * i], a.scale_log2, nm));
          const float p1 = fast_exp2(fmaf(sv[32 * c + 2 * i + 1], a.scale_log2, nm));
          s4[i & 3] += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
        // P over the first 64 score columns (already read into registers)
        tmem_st16(tmem + lane_off + s_col + (uint32_t)(c * 16), pk);
      }
      // O_t += P(j - 1) V(j - 1) has completed (the commit that announced S(j) covers it), so
      // O may be rescaled before P(j) is announced; any lane that needs it makes the warp do it
      if (__any_sync(0xffffffffu, rescale)) {
        const float f = rescale ? corr : 1.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t rr[32];
          const uint32_t ta = tmem + lane_off + o_col + (uint32_t)(c * 32);
          tc::tmem_ld32(ta, rr);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
          tmem_st32(ta, rr);
        }
      }
      l += (s4[0] + s4[1]) + (s4[2] + s4[3]);
      tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[t]);
    }
    if (split) {
      // ---- a split pair: the CTA that finishes first parks its partial (unnormalised O, its
      // reference and sum); the other combines both in segment order and writes the result
      const bool have = n_kv >= 1;
      if (ok && have && tc::mbar_wait_warp(&o_done[t], 0, abort_flag)) tc::fence_after_sync();
      else if (have) ok = false;
      // the eight softmax warps meet on an mbarrier (bounded waits), phases 0, 1, 2 in turn
      int sync_phase = 0;
      auto softmax_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm_sync);
        return tc::mbar_wait_warp(&sm_sync, (uint32_t)(sync_phase++) & 1u, abort_flag);
      };
      bool synced = softmax_sync();
      if (warp == 2) {
        if (lane == 0) role_sh = (ok && synced) ? atomicAdd(&a.flags[2 * unit], 1) : -1;
        __syncwarp();
      }
      synced = softmax_sync() && synced;
      const int role = synced ? role_sh : -1;
      const bool row_ok = tq < q_hi;
      const int64_t grow = b * a.Tc + (tq - a.s);
      float* prow = a.part + (grow * a.H + h) * HD;
      float* mlrow = a.ml + (grow * a.H + h) * 2;
      const float m_own = have ? m_ref : -INFINITY, l_own = have ? l : 0.f;
      if (role == 0) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t rr[32];
          if (have) {
            tc::tmem_ld32(tmem + lane_off + o_col + (uint32_t)(c * 32), rr);
            tc::tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = 0u;
          }
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<uint4*>(prow + c * 32 + i) =
                  make_uint4(rr[i], rr[i + 1], rr[i + 2], rr[i + 3]);
          }
        }
        if (row_ok) *reinterpret_cast<float2*>(mlrow) = make_float2(m_own, l_own);
        __threadfence();
        if (softmax_sync() && warp == 2) {
          if (lane == 0) atomicExch(&a.flags[2 * unit + 1], 1);
          __syncwarp();
        }
      } else if (role == 1) {
        // the other CTA has taken its turn and is writing its partial: bounded wait for it, the
        // whole warp looping on lane 0's reading
        if (warp == 2) {
          const volatile int* ready = a.flags + 2 * unit + 1;
          const uint64_t t0 = tc::globaltimer_ns();
          for (;;) {
            int stop = 0;
            if (lane == 0) {
              if (*ready != 0) stop = 1;
              else if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) stop = 2;
            }
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop == 2 && lane == 0) *abort_flag = 1;
            if (stop != 0) break;
          }
          __syncwarp();
        }
        const bool got = softmax_sync();
        __threadfence();
        // warp-uniform from here: the TMEM loads are warp-collective; only the global accesses
        // of rows past the chunk's end are skipped
        if (__all_sync(0xffffffffu, got && *abort_flag == 0)) {
          const float2 mo = row_ok ? __ldcg(reinterpret_cast<const float2*>(mlrow))
                                   : make_float2(-INFINITY, 0.f);
          // segment 0 first: (m0, l0, O0) and (m1, l1, O1) in that order whichever is own
          const float m0 = seg == 0 ? m_own : mo.x, l0 = seg == 0 ? l_own : mo.y;
          const float m1 = seg == 0 ? mo.x : m_own, l1 = seg == 0 ? mo.y : l_own;
          const float m = fmaxf(m0, m1);
          const float a0 = m0 == m ? 1.f : (m0 == -INFINITY ? 0.f : fast_exp2(m0 - m));
          const float a1 = m1 == m ? 1.f : (m1 == -INFINITY ? 0.f : fast_exp2(m1 - m));
          const float ls = a0 * l0 + a1 * l1;
          const float inv = 1.f / ls;
          __nv_bfloat16* op = static_cast<__nv_bfloat16*>(a.o) + (grow * a.H + h) * HD;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t rr[32];
            if (have) {
              tc::tmem_ld32(tmem + lane_off + o_col + (uint32_t)(c * 32), rr);
              tc::tmem_ld_wait();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) rr[i] = 0u;
            }
            if (row_ok) {
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                float v[8];
#pragma unroll
                for (int k = 0; k < 8; k += 4) {
                  const float4 q =
                      __ldcg(reinterpret_cast<const float4*>(prow + c * 32 + i + k));
                  const float ot[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float ow = __uint_as_float(rr[i + k + e]);
                    const float o0 = seg == 0 ? ow : ot[e], o1 = seg == 0 ? ot[e] : ow;
                    v[k + e] = (a0 * o0 + a1 * o1) * inv;
                  }
                }
                uint4 w;
                w.x = pack_bf16(v[0], v[1]);
                w.y = pack_bf16(v[2], v[3]);
                w.z = pack_bf16(v[4], v[5]);
                w.w = pack_bf16(v[6], v[7]);
                *reinterpret_cast<uint4*>(op + c * 32 + i) = w;
              }
            }
          }
          if (row_ok) a.lse[grow * a.H + h] = (m + __log2f(ls)) * 0.69314718055994531f;
        }
      }
    } else
    // final: wait for the tile's last O += P V, normalise, store
    if (ok && n_kv >= 1 && tc::mbar_wait_warp(&o_done[t], 0, abort_flag)) {
      tc::fence_after_sync();
      const bool row_ok = tq < q_hi;
      const float inv = 1.f / l;
      const int64_t grow = b * a.Tc + (tq - a.s);
      __nv_bfloat16* op = static_cast<__nv_bfloat16*>(a.o) + (grow * a.H + h) * HD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tc::tmem_ld32(tmem + lane_off + o_col + (uint32_t)(c * 32), rr);
        tc::tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(rr[i]) * inv, __uint_as_float(rr[i + 1]) * inv);
            v.y = pack_bf16(__uint_as_float(rr[i + 2]) * inv, __uint_as_float(rr[i + 3]) * inv);
            v.z = pack_bf16(__uint_as_float(rr[i + 4]) * inv, __uint_as_float(rr[i + 5]) * inv);
            v.w = pack_bf16(__uint_as_float(rr[i + 6]) * inv, __uint_as_float(rr[i + 7]) * inv);
            *reinterpret_cast<uint4*>(op + c * 32 + i) = v;
          }
        }
      }
      if (row_ok) a.lse[grow * a.H + h] = (m_ref + __log2f(l)) * 0.69314718055994531f;
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_attn() {
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

// 3-D bf16 map over [rows, heads, HD] (HD innermost): box {64, 1, 128}, 128-byte swizzle.
bool make_map3(CUtensorMap* map, const void* base, int64_t heads, int64_t rows) {
  EncodeTiledFn fn = encode_fn_attn();
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

bool attn_tc_supported(int64_t hd, int dt, const void* q, const void* Kp, const void* Vp,
                       const void* o) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return hd == HD && dt == DT_BF16 && al(q) && al(Kp) && al(Vp) && al(o) &&
         encode_fn_attn() != nullptr;
}

size_t attn_fwd_split_flags(int64_t B, int64_t Tc, int64_t H) {
  const int64_t nq = (Tc + BQ - 1) / BQ, np = (nq + 1) / 2;
  return (size_t)2 * B * H * np;
}

cudaError_t attn_fwd_tc(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                        const void* q, const void* Kp, const void* Vp, void* o, float* lse,
                        const AttnFwdSplit& sc, int* err, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map3(&mq, q, H, B * Tc) || !make_map3(&mk, Kp, Hkv, B * T) ||
      !make_map3(&mv, Vp, Hkv, B * T))
    return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES);
  });
  if (attr != cudaSuccess) return attr;
  FwdArgs a;
  a.B = B; a.T = T; a.Tc = Tc; a.s = s; a.H = H; a.Hkv = Hkv;
  a.nq = (int)((Tc + BQ - 1) / BQ);
  a.np = (a.nq + 1) / 2;
  a.o = o;
  a.lse = lse;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  a.err = err;
  // Pairs whose keys reach past a quarter of the sequence (key tile segt, a function of T only)
  // run as two CTAs, so that a chunk's 32 heads x 16 pairs fill whole waves of the SMs; the
  // heavier segment's CTAs are launched first and the lighter ones fill the last wave.
  const int64_t units = B * H * a.np;
  const int64_t nkv_max = (s + Tc + BKV - 1) / BKV;
  a.segt = (int)(((T + BKV - 1) / BKV + 3) / 4);
  a.seg1_first = nkv_max - a.segt > a.segt ? 1 : 0;
  a.units = (int)units;
  a.part = nullptr;
  a.ml = nullptr;
  a.flags = nullptr;
  const bool split = sc.part && sc.ml && sc.flags && nkv_max > a.segt;
  if (split) {
    a.part = sc.part;
    a.ml = sc.ml;
    a.flags = sc.flags;
    cudaError_t e = cudaMemsetAsync(a.flags, 0, sizeof(int) * 2 * (size_t)units, st);
    if (e != cudaSuccess) return e;
  } else {
    a.segt = 0;
    a.seg1_first = 0;
  }
  const int64_t grid = units * (split ? 2 : 1);
  launch(attn_fwd_tc_kernel, dim3((unsigned)grid), dim3(kThreads), (size_t)SMEM_BYTES, st, mq, mk,
         mv, a);
  return cudaGetLastError();
}

}  // namespace sbp
