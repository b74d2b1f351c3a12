// Causal GQA attention backward of one query chunk over its key prefix on the tcgen05 tensor
// cores (head_dim 128, bf16 operands, fp32 accumulation), as two kernels that each keep their
// accumulator in TMEM and write it once (no atomics; both results are deterministic and do not
// depend on how the sequence was chunked):
//
// dK/dV kernel: one CTA owns (sequence b, KV head g, 128-key tile) and loops over the query
// heads of g's group and the chunk's query tiles that can see those keys.  Each (head, query
// tile) pair is taken as two halves of 64 queries; per half h:
//   S^T_h  = K Q_h^T   (TMEM c_s(h), 64 columns)     dP^T_h = V dO_h^T  (TMEM c_dp(h))
//   P^T_h  = exp(S^T_h * scale - lse) -> bf16, written back into TMEM over the dP^T_h columns
//            the same warp has already read (the A operand of the dV product)
//   dS^T_h = P^T_h (dP^T_h - delta)    -> bf16, shared-memory buffer h
//   dV    += P^T_h dO_h (TMEM [256,384))            dK += dS^T_h Q_h (TMEM [384,512))
// The two halves have their own TMEM columns and dS^T buffers, so the tensor cores compute the
// scores of one half (and the dV / dK products of the other) while the element-wise warps
// turn the scores of a half into P^T and dS^T.
// The query tiles are taken in blocks of a fixed number of tiles counted from the chunk start
// (all heads of the group within a block); after each block dK, dV are added into the fp32
// prefix accumulators (single owner, no atomics).  A chunk whose length is a multiple of the
// block therefore adds exactly the partial sums the same queries give inside a longer chunk.
//
// dQ kernel: one CTA owns (sequence b, query head h, 128-query tile) and loops over the key
// tiles of its causal prefix, each as two halves of 64 keys:  S_h = Q K_h^T, dP_h = dO V_h^T,
// dS_h = P_h (dP_h - delta) -> shared-memory buffer h, dQ += dS_h K_h (TMEM), stored once at
// the end; the halves are pipelined the same way.
//
// Entries with key > query, queries outside the chunk and keys outside the prefix are masked
// by selection (not by multiplication), so stale values never reach an accumulator.
// Warp roles (both kernels): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2..9
// element-wise (the warp's TMEM lane quarter is its index mod 4; the two warps of a quarter
// split the 64 columns of a half).
#include <cuda.h>

#include <mutex>

#include "sbp_internal.cuh"

// Cycle accounting of the dK/dV kernel, compiled in only with -DSBP_ATTN_TIMING (the build's
// --timing library): CTA 0 prints, per launch, the producer's cycles waiting for a free Q/dO
// stage, the MMA issuer's cycles waiting for dS / Q,dO / the accumulator flush and issuing,
// and two element-wise warps' cycles waiting for Q,dO and for the scores, working, and
// flushing.  Off by default: no cost.
#ifdef SBP_ATTN_TIMING
#include <cstdio>
#define SBP_ATTN_TIMED(...) __VA_ARGS__
#else
#define SBP_ATTN_TIMED(...)
#endif
#include "tc_ptx.cuh"

namespace sbp {

namespace {

constexpr int HD = 128;
constexpr int BT = 128;                     // keys per key tile, queries per query tile
constexpr int TILE = 128 * HD * 2;          // 32 KB bf16 tile: two 64-column swizzled chunks
constexpr int CHUNK = TILE / 2;
constexpr int QD_STAGES = 2;
// All shared state lives in the dynamic allocation (no static shared memory), whose start is
// 1024-byte aligned as the 128-byte swizzle needs: the tiles first, then the statistics and
// the barriers.
struct KvShared {
  float stat[2 /*QD_STAGES*/][2][BT];   // per stage: lse (log2 units), delta
  uint64_t kv_full, qd_full[2], qd_empty[2], sdp_full[2], ds_full[2], kv_free, drain;
  uint32_t tmem;
  int abort;
};
constexpr int KV_TILES_BYTES = (3 + 2 * QD_STAGES) * TILE;        // K, V, dS^T, 2 x (Q, dO)
constexpr int KV_SMEM_BYTES = KV_TILES_BYTES + (int)sizeof(KvShared);
constexpr int KV_RING = 2;                                         // K/V stages of the dQ kernel
struct QShared {
  uint64_t qd_full, kv_full[KV_RING], kv_empty[KV_RING], sdp_full[2], ds_full[2], dq_done, drain;
  uint32_t tmem;
  int abort;
};
constexpr int Q_TILES_BYTES = (3 + 2 * KV_RING) * TILE;           // Q, dO, dS, 2 x (K, V)
constexpr int Q_SMEM_BYTES = Q_TILES_BYTES + (int)sizeof(QShared);
constexpr int kEwWarps = 8;                 // element-wise warps: 4 lane quarters x 2 column halves
constexpr int kThreads = 64 + 32 * kEwWarps;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns: half h of a tile keeps its scores at c_s(h) and their gradient at c_dp(h)
// (64 columns each); the fp32 accumulators dV, dK (key-tile kernel) or dQ (query-tile kernel)
// take the upper columns.
constexpr uint32_t C_DV = 256, C_DK = 384, C_DQ = 256;
__device__ __forceinline__ uint32_t c_s(int h) { return 128u * (uint32_t)h; }
__device__ __forceinline__ uint32_t c_dp(int h) { return 128u * (uint32_t)h + 64u; }
constexpr int HALF = TILE / 4;              // 64 rows x 128 bytes: a 64-row slice of a chunk

struct BwdArgs {
  int64_t B, T, Tc, s, H, Hkv;
  int nq, nkt;
  int qb;               // query tiles per dK/dV accumulation block
  int64_t Tcp;          // Tc rounded up to the query tile
  const float* lse_t;   // [H, B, Tcp] log2 units, zero padded
  const float* delta_t; // [H, B, Tcp], zero padded
  float* dq;            // [B*Tc, H, HD] fp32, overwritten (dQ kernel)
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
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// ================================================================== dK / dV kernel
// The work of a key tile, pair by pair: (query head hh of the group, query tile qi) for the
// query tiles i0 .. nq - 1, ordered block by block (qb tiles, counted from the chunk start)
// and head-major inside a block; first / last: the pair opens / closes its block.  Every role
// of the CTA walks the same sequence with its own iterator (no divisions per pair).
struct PairPos {
  int64_t hh, qi;
  bool first, last;
};
struct PairIter {
  int qs, nbt, hi, t;       // block start tile, tiles in the block, head in group, tile in block
  int grp, qb, nq;
  __device__ __forceinline__ void init(int i0, int nq_, int grp_, int qb_) {
    grp = grp_;
    qb = qb_;
    nq = nq_;
    qs = i0;
    nbt = min((i0 / qb + 1) * qb, nq) - i0;
    hi = 0;
    t = 0;
  }
  __device__ __forceinline__ PairPos pos(int64_t g) const {
    PairPos p;
    p.hh = g * grp + hi;
    p.qi = qs + t;
    p.first = hi == 0 && t == 0;
    p.last = hi == grp - 1 && t == nbt - 1;
    return p;
  }
  __device__ __forceinline__ void next() {
    if (++t == nbt) {
      t = 0;
      if (++hi == grp) {
        hi = 0;
        qs += nbt;
        nbt = min(qb, nq - qs);
      }
    }
  }
};

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                   const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  KvShared& sh = *reinterpret_cast<KvShared*>(smem_raw + KV_TILES_BYTES);
  uint8_t* sK = smem_raw;
  uint8_t* sV = sK + TILE;
  uint8_t* sdSt = sV + TILE;                     // half h: dS^T [128 keys x 64 queries] at h*CHUNK
  uint8_t* sQ0 = sdSt + TILE;                    // stage st: Q at sQ0 + 2 st TILE, dO after it
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sh.abort;

  // work decomposition: early key tiles (the most query tiles) first
  const int kt = (int)(blockIdx.x % a.nkt);
  const int64_t g = (blockIdx.x / a.nkt) % a.Hkv;
  const int64_t b = blockIdx.x / (a.nkt * a.Hkv);
  const int64_t grp = a.H / a.Hkv;
  const int64_t e = a.s + a.Tc;                  // prefix end
  const int64_t k_lo = (int64_t)kt * BT;
  // first query tile whose last row can see key k_lo
  const int64_t i0 = (k_lo - a.s - (BT - 1) <= 0) ? 0 : (k_lo - a.s) / BT;
  const int nqt = (int)(a.nq - i0);              // query tiles per head
  // the swizzled tiles need a 1024-byte aligned base: refuse to run (status raised) otherwise
  const bool misaligned = (tc::smem_u32(smem_raw) & 1023u) != 0;
  const int npairs = (nqt > 0 && !misaligned) ? (int)(grp * nqt) : 0;

  if (threadIdx.x == 0) {
    tc::mbar_init(&sh.kv_full, 1);
    for (int i = 0; i < QD_STAGES; ++i) {
      tc::mbar_init(&sh.qd_full[i], 1);
      tc::mbar_init(&sh.qd_empty[i], 1);
    }
    for (int h = 0; h < 2; ++h) {
      tc::mbar_init(&sh.sdp_full[h], 1);
      tc::mbar_init(&sh.ds_full[h], kEwWarps);
    }
    tc::mbar_init(&sh.kv_free, kEwWarps);
    tc::mbar_init(&sh.drain, 1);
    sh.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&sh.tmem, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sh.tmem;

  if (warp == 0) {
    if (lane == 0 && npairs > 0) {
      // ---------------------------------------------------------------- producer
      const int32_t krow = (int32_t)(b * a.T + k_lo);
      tc::mbar_expect_tx(&sh.kv_full, 2 * TILE);
      tc::tma_load_3d(sK, &tmK, &sh.kv_full, 0, (int32_t)g, krow);
      tc::tma_load_3d(sK + CHUNK, &tmK, &sh.kv_full, 64, (int32_t)g, krow);
      tc::tma_load_3d(sV, &tmV, &sh.kv_full, 0, (int32_t)g, krow);
      tc::tma_load_3d(sV + CHUNK, &tmV, &sh.kv_full, 64, (int32_t)g, krow);
      bool ok = true;
      int issued = 0;
      SBP_ATTN_TIMED(long long w_empty = 0, tp0 = clock64(), c0;)
      PairIter it;
      it.init((int)i0, a.nq, (int)grp, a.qb);
      for (int j = 0; j < npairs; ++j, it.next()) {
        const PairPos pos = it.pos(g);
        const int st = j % QD_STAGES;
        const uint32_t ph = (uint32_t)(j / QD_STAGES) & 1u;
        SBP_ATTN_TIMED(c0 = clock64();)
        if (!tc::mbar_wait(&sh.qd_empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
        SBP_ATTN_TIMED(w_empty += clock64() - c0;)
        uint8_t* sQ = sQ0 + 2 * st * TILE;
        uint8_t* sdO = sQ + TILE;
        const int32_t qrow = (int32_t)(b * a.Tc + pos.qi * BT);
        tc::mbar_expect_tx(&sh.qd_full[st], 2 * TILE + 2 * BT * 4);
        const int64_t srow = (pos.hh * a.B + b) * a.Tcp + pos.qi * BT;
        tc::bulk_load(&sh.stat[st][0][0], a.lse_t + srow, BT * 4, &sh.qd_full[st]);
        tc::bulk_load(&sh.stat[st][1][0], a.delta_t + srow, BT * 4, &sh.qd_full[st]);
        tc::tma_load_3d(sQ, &tmQ, &sh.qd_full[st], 0, (int32_t)pos.hh, qrow);
        tc::tma_load_3d(sQ + CHUNK, &tmQ, &sh.qd_full[st], 64, (int32_t)pos.hh, qrow);
        tc::tma_load_3d(sdO, &tmdO, &sh.qd_full[st], 0, (int32_t)pos.hh, qrow);
        tc::tma_load_3d(sdO + CHUNK, &tmdO, &sh.qd_full[st], 64, (int32_t)pos.hh, qrow);
        issued = j + 1;
      }
      SBP_ATTN_TIMED(if (blockIdx.x == 0) printf(
          "SBPT KVPROD s %lld Tc %lld pairs %d total %lld w_empty %lld\n", (long long)a.s,
          (long long)a.Tc, npairs, clock64() - tp0, w_empty);)
      if (!ok) {
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&sh.kv_full, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        for (int j = issued > QD_STAGES ? issued - QD_STAGES : 0; j < issued; ++j)
          while (!tc::mbar_try_wait(&sh.qd_full[j % QD_STAGES], (uint32_t)(j / QD_STAGES) & 1u) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && npairs > 0) {
      // ---------------------------------------------------------------- MMA issuer
      // Two 64-query halves per pair, each with its own S^T / dP^T columns and dS^T buffer,
      // so the scores of one half are computed while the element-wise warps work on the other.
      const uint32_t id_s = tc::idesc_bf16_f32(128, 64, 0, 0);     // S^T, dP^T: N = 64 queries
      const uint32_t id_g = tc::idesc_bf16_f32(128, 128, 0, 1);    // dV, dK: B MN-major
      const uint32_t aK = tc::smem_u32(sK), aV = tc::smem_u32(sV), adS = tc::smem_u32(sdSt),
                     aQ0 = tc::smem_u32(sQ0);
      bool ok = tc::mbar_wait(&sh.kv_full, 0, abort_flag);
      bool issued = false;
      // Shared-memory descriptors built once; a k-step adds its byte offset / 16 to the start
      // address field (the tiles sit below 256 KB, so the field cannot carry over).  This keeps
      // the single issuing thread fast enough for the 128 x 64 x 16 products.
      const uint64_t dK = tc::smem_desc_sw128(aK, 16, 1024), dV = tc::smem_desc_sw128(aV, 16, 1024);
      const uint64_t dS = tc::smem_desc_sw128(adS, 16, 1024);
      // the two Q/dO stages differ by a constant: stage 1's start address field is stage 0's
      // plus 2 TILE / 16 (selected, not indexed, so the descriptors stay in registers)
      static_assert(QD_STAGES == 2, "stage descriptors are selected between two stages");
      const uint64_t dQk0 = tc::smem_desc_sw128(aQ0, 16, 1024);
      const uint64_t dOk0 = tc::smem_desc_sw128(aQ0 + TILE, 16, 1024);
      const uint64_t dQm0 = tc::smem_desc_sw128(aQ0, CHUNK, 1024);
      const uint64_t dOm0 = tc::smem_desc_sw128(aQ0 + TILE, CHUNK, 1024);
      constexpr uint64_t kStage = (uint64_t)((2 * TILE) >> 4);
      // S^T_h = K Q_h^T and dP^T_h = V dO_h^T of pair j's half h
      auto scores = [&](int j, int h) {
        const uint64_t so = (j & 1) ? kStage : 0;
        const uint64_t bq = dQk0 + so + (uint64_t)((h * HALF) >> 4);
        const uint64_t bo = dOk0 + so + (uint64_t)((h * HALF) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // K = head dim
          const uint64_t off = (uint64_t)(((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4);
          tc::mma_f16_ss(tmem + c_s(h), dK + off, bq + off, id_s, kk != 0);
          tc::mma_f16_ss(tmem + c_dp(h), dV + off, bo + off, id_s, kk != 0);
        }
        tc::mma_commit(&sh.sdp_full[h]);
      };
      // dV += P^T_h dO_h (P^T from TMEM), dK += dS^T_h Q_h; `first`: the block's first product
      auto grads = [&](int j, int h, bool first) {
        const uint64_t so = (j & 1) ? kStage : 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {   // K = 64 queries of the half
          const uint64_t offm = so + (uint64_t)(((4 * h + kk) * 2048) >> 4);  // MN-major k-step
          const uint32_t acc = (!first || kk != 0) ? 1u : 0u;
          // packed P^T of queries 32 w.. of half h sits at c_dp(h) + 32 w (w = column half)
          const uint32_t pcol = c_dp(h) + 32 * (kk >> 1) + 8 * (kk & 1);
          mma_f16_ts(tmem + C_DV, tmem + pcol, dOm0 + offm, id_g, acc);
          tc::mma_f16_ss(tmem + C_DK, dS + (uint64_t)((h * CHUNK + kk * 32) >> 4), dQm0 + offm,
                         id_g, acc);
        }
      };
      int nflush = 0;
      SBP_ATTN_TIMED(long long w_ds = 0, w_qd = 0, w_free = 0, t_iss = 0, ti0 = clock64(), c0;)
      if (ok && tc::mbar_wait(&sh.qd_full[0], 0, abort_flag)) {
        tc::fence_after_sync();
        scores(0, 0);
        scores(0, 1);
        issued = true;
      } else {
        ok = false;
      }
      PairIter it;
      it.init((int)i0, a.nq, (int)grp, a.qb);
      for (int j = 0; j < npairs && ok; ++j, it.next()) {
        const PairPos pos = it.pos(g);
        const uint32_t ph = (uint32_t)j & 1u;
        SBP_ATTN_TIMED(c0 = clock64();)
        if (!tc::mbar_wait(&sh.ds_full[0], ph, abort_flag)) { ok = false; break; }
        SBP_ATTN_TIMED(w_ds += clock64() - c0;)
        // a new block overwrites dK / dV: the element-wise warps must have added the last one
        if (pos.first && j > 0) {
          SBP_ATTN_TIMED(c0 = clock64();)
          if (!tc::mbar_wait(&sh.kv_free, (uint32_t)nflush & 1u, abort_flag)) { ok = false; break; }
          SBP_ATTN_TIMED(w_free += clock64() - c0;)
          ++nflush;
        }
        tc::fence_after_sync();
        SBP_ATTN_TIMED(c0 = clock64();)
        grads(j, 0, pos.first);
        SBP_ATTN_TIMED(t_iss += clock64() - c0;)
        const bool more = j + 1 < npairs;
        if (more) {
          const int st1 = (j + 1) % QD_STAGES;
          SBP_ATTN_TIMED(c0 = clock64();)
          if (!tc::mbar_wait(&sh.qd_full[st1], (uint32_t)((j + 1) / QD_STAGES) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          SBP_ATTN_TIMED(w_qd += clock64() - c0;)
          tc::fence_after_sync();
          SBP_ATTN_TIMED(c0 = clock64();)
          scores(j + 1, 0);
          SBP_ATTN_TIMED(t_iss += clock64() - c0;)
        }
        SBP_ATTN_TIMED(c0 = clock64();)
        if (!tc::mbar_wait(&sh.ds_full[1], ph, abort_flag)) { ok = false; break; }
        SBP_ATTN_TIMED(w_ds += clock64() - c0;)
        tc::fence_after_sync();
        SBP_ATTN_TIMED(c0 = clock64();)
        grads(j, 1, false);
        tc::mma_commit(&sh.qd_empty[j % QD_STAGES]);
        if (more) scores(j + 1, 1);
        SBP_ATTN_TIMED(t_iss += clock64() - c0;)
      }
      SBP_ATTN_TIMED(if (blockIdx.x == 0) printf(
          "SBPT KVISSUE s %lld Tc %lld pairs %d total %lld w_ds %lld w_qd %lld w_free %lld "
          "issue %lld\n", (long long)a.s, (long long)a.Tc, npairs, clock64() - ti0, w_ds, w_qd,
          w_free, t_iss);)
      if (issued) {
        tc::mma_commit(&sh.drain);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&sh.drain, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (npairs > 0) {
    // ------------------------------------------------------------------ element-wise warps
    const int q4 = warp & 3;
    const int wh = (warp - 2) >> 2;                  // column half: queries 32 wh .. of a half
    const int r = q4 * 32 + lane;                    // TMEM lane = key row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int kpos = (int)(k_lo + r);
    const float scale_log2 = a.scale * 1.4426950408889634f;
    const int e32 = (int)e;
    const bool kv = kpos < e32;
    const int64_t ko = ((b * a.T + kpos) * a.Hkv + g) * HD;
    bool ok = true;
    SBP_ATTN_TIMED(long long w_q = 0, w_sdp = 0, t_work = 0, t_flush = 0, te0 = clock64(), c0;)
    PairIter it;
    it.init((int)i0, a.nq, (int)grp, a.qb);
    for (int j = 0; j < npairs && ok; ++j, it.next()) {
      const uint32_t ph = (uint32_t)j & 1u;
      const PairPos pos = it.pos(g);
      if (pos.first && kv) {
        // bring this row's dK / dV accumulator lines into L2 ahead of the block's flush
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          prefetch_l2(a.dKp + ko + wh * 64 + u * 32);
          prefetch_l2(a.dVp + ko + wh * 64 + u * 32);
        }
      }
      const int st = j % QD_STAGES;     // this pair's Q/dO stage also holds lse and delta
      // acquire the bulk copies of this stage (already complete once the scores are ready)
      SBP_ATTN_TIMED(c0 = clock64();)
      if (!tc::mbar_wait_warp(&sh.qd_full[st], (uint32_t)(j / QD_STAGES) & 1u, abort_flag)) {
        ok = false;
        break;
      }
      SBP_ATTN_TIMED(w_q += clock64() - c0;)
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int qoff = 64 * h + 32 * wh;             // this warp's queries within the tile
        const int q0 = (int)(a.s + pos.qi * BT) + qoff;  // absolute position of its first query
        // no masking needed when every key of the tile precedes every (valid) query here
        const bool full = (k_lo + BT - 1 <= q0) && (pos.qi * BT + qoff + 32 <= a.Tc);
        const float* lse_s = sh.stat[st][0] + qoff;
        const float* delta_s = sh.stat[st][1] + qoff;
        SBP_ATTN_TIMED(c0 = clock64();)
        if (!tc::mbar_wait_warp(&sh.sdp_full[h], ph, abort_flag)) { ok = false; break; }
        SBP_ATTN_TIMED(w_sdp += clock64() - c0; c0 = clock64();)
        tc::fence_after_sync();
        uint32_t rs[32], rd[32];
        tc::tmem_ld32(tmem + lane_off + c_s(h) + 32 * wh, rs);
        tc::tmem_ld32(tmem + lane_off + c_dp(h) + 32 * wh, rd);
        tc::tmem_ld_wait();
        uint32_t pp[16], dd[16];
        const float4* l4 = reinterpret_cast<const float4*>(lse_s);
        const float4* d4 = reinterpret_cast<const float4*>(delta_s);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 lv = l4[i4], dv = d4[i4];
          const float la[4] = {lv.x, lv.y, lv.z, lv.w};
          const float da[4] = {dv.x, dv.y, dv.z, dv.w};
          float p[4], gg[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int i = i4 * 4 + k;
            p[k] = ex2(fmaf(__uint_as_float(rs[i]), scale_log2, -la[k]));
            gg[k] = p[k] * (__uint_as_float(rd[i]) - da[k]);
            if (!full) {
              const int qpos = q0 + i;
              const bool live = (kpos <= qpos) && (qpos < e32);
              p[k] = live ? p[k] : 0.f;
              gg[k] = live ? gg[k] : 0.f;
            }
          }
          pp[i4 * 2] = pack2(p[0], p[1]);
          pp[i4 * 2 + 1] = pack2(p[2], p[3]);
          dd[i4 * 2] = pack2(gg[0], gg[1]);
          dd[i4 * 2 + 1] = pack2(gg[2], gg[3]);
        }
        // packed P^T over the dP^T columns this warp has just read
        tmem_st16(tmem + lane_off + c_dp(h) + 32 * wh, pp);
        // dS^T of this half (the previous pair's dK product of this half has read the buffer:
        // its completion precedes the scores this warp has waited for)
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_unit(sdSt + h * CHUNK, r, 4 * wh + u,
                  make_uint4(dd[4 * u], dd[4 * u + 1], dd[4 * u + 2], dd[4 * u + 3]));
        tmem_st_wait();
        fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sh.ds_full[h]);
        SBP_ATTN_TIMED(t_work += clock64() - c0;)
      }
      if (!ok || !pos.last) continue;
      SBP_ATTN_TIMED(c0 = clock64();)
      // end of a block: add its dK, dV into the fp32 prefix accumulators (single owner)
      // the release of this pair's Q/dO stage is committed after its last dK / dV product
      if (!tc::mbar_wait_warp(&sh.qd_empty[j % QD_STAGES], (uint32_t)(j / QD_STAGES) & 1u,
                              abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = wh * 2 + cc;
        uint32_t rk[32], rv[32];
        tc::tmem_ld32(tmem + lane_off + C_DK + c * 32, rk);
        tc::tmem_ld32(tmem + lane_off + C_DV + c * 32, rv);
        tc::tmem_ld_wait();
        if (kv) {
          // all loads first (one memory latency), then the adds and the stores
          float4* pk = reinterpret_cast<float4*>(a.dKp + ko + c * 32);
          float4* pv = reinterpret_cast<float4*>(a.dVp + ko + c * 32);
          float4 x[8], y[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            x[i] = pk[i];
            y[i] = pv[i];
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            x[i].x += __uint_as_float(rk[4 * i]) * a.scale;
            x[i].y += __uint_as_float(rk[4 * i + 1]) * a.scale;
            x[i].z += __uint_as_float(rk[4 * i + 2]) * a.scale;
            x[i].w += __uint_as_float(rk[4 * i + 3]) * a.scale;
            y[i].x += __uint_as_float(rv[4 * i]);
            y[i].y += __uint_as_float(rv[4 * i + 1]);
            y[i].z += __uint_as_float(rv[4 * i + 2]);
            y[i].w += __uint_as_float(rv[4 * i + 3]);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            pk[i] = x[i];
            pv[i] = y[i];
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0 && j + 1 < npairs) tc::mbar_arrive(&sh.kv_free);
      SBP_ATTN_TIMED(t_flush += clock64() - c0;)
    }
    SBP_ATTN_TIMED(if (blockIdx.x == 0 && (warp == 2 || warp == 9) && lane == 0) printf(
        "SBPT KVEW warp %d s %lld Tc %lld pairs %d total %lld w_qd %lld w_sdp %lld work %lld "
        "flush %lld\n", warp, (long long)a.s, (long long)a.Tc, npairs, clock64() - te0, w_q,
        w_sdp, t_work, t_flush);)
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && (sh.abort || misaligned) && a.err) atomicExch(a.err, DEV_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ================================================================== dQ kernel
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  QShared& sh = *reinterpret_cast<QShared*>(smem_raw + Q_TILES_BYTES);
  uint8_t* sQ = smem_raw;
  uint8_t* sdO = sQ + TILE;
  uint8_t* sdS = sdO + TILE;                     // half h: dS [128 queries x 64 keys] at h*CHUNK
  uint8_t* sKV0 = sdS + TILE;                    // ring stage st: K at sKV0 + 2 st TILE, V after
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sh.abort;

  // heavy (late) query tiles first
  const int qt = a.nq - 1 - (int)(blockIdx.x % a.nq);
  const int64_t h = (blockIdx.x / a.nq) % a.H;
  const int64_t b = blockIdx.x / (a.nq * a.H);
  const int64_t g = h / (a.H / a.Hkv);
  const int64_t q_lo = a.s + (int64_t)qt * BT;                  // absolute position of row 0
  const int64_t q_hi = a.s + imin((int64_t)(qt + 1) * BT, a.Tc);  // one past the last valid row
  const bool misaligned = (tc::smem_u32(smem_raw) & 1023u) != 0;
  const int nkv = misaligned ? 0 : (int)((q_hi + BT - 1) / BT);  // key tiles 0 .. nkv-1

  if (threadIdx.x == 0) {
    tc::mbar_init(&sh.qd_full, 1);
    for (int i = 0; i < KV_RING; ++i) {
      tc::mbar_init(&sh.kv_full[i], 1);
      tc::mbar_init(&sh.kv_empty[i], 1);
    }
    for (int hh = 0; hh < 2; ++hh) {
      tc::mbar_init(&sh.sdp_full[hh], 1);
      tc::mbar_init(&sh.ds_full[hh], kEwWarps);
    }
    tc::mbar_init(&sh.dq_done, 1);
    tc::mbar_init(&sh.drain, 1);
    sh.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&sh.tmem, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sh.tmem;

  if (warp == 0) {
    if (lane == 0 && nkv > 0) {
      // ---------------------------------------------------------------- producer
      const int32_t qrow = (int32_t)(b * a.Tc + (int64_t)qt * BT);
      tc::mbar_expect_tx(&sh.qd_full, 2 * TILE);
      tc::tma_load_3d(sQ, &tmQ, &sh.qd_full, 0, (int32_t)h, qrow);
      tc::tma_load_3d(sQ + CHUNK, &tmQ, &sh.qd_full, 64, (int32_t)h, qrow);
      tc::tma_load_3d(sdO, &tmdO, &sh.qd_full, 0, (int32_t)h, qrow);
      tc::tma_load_3d(sdO + CHUNK, &tmdO, &sh.qd_full, 64, (int32_t)h, qrow);
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % KV_RING;
        const uint32_t ph = (uint32_t)(j / KV_RING) & 1u;
        if (!tc::mbar_wait(&sh.kv_empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* sK = sKV0 + 2 * st * TILE;
        uint8_t* sV = sK + TILE;
        const int32_t krow = (int32_t)(b * a.T + (int64_t)j * BT);
        tc::mbar_expect_tx(&sh.kv_full[st], 2 * TILE);
        tc::tma_load_3d(sK, &tmK, &sh.kv_full[st], 0, (int32_t)g, krow);
        tc::tma_load_3d(sK + CHUNK, &tmK, &sh.kv_full[st], 64, (int32_t)g, krow);
        tc::tma_load_3d(sV, &tmV, &sh.kv_full[st], 0, (int32_t)g, krow);
        tc::tma_load_3d(sV + CHUNK, &tmV, &sh.kv_full[st], 64, (int32_t)g, krow);
        issued = j + 1;
      }
      if (!ok) {
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&sh.qd_full, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        for (int j = issued > KV_RING ? issued - KV_RING : 0; j < issued; ++j)
          while (!tc::mbar_try_wait(&sh.kv_full[j % KV_RING], (uint32_t)(j / KV_RING) & 1u) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nkv > 0) {
      // ---------------------------------------------------------------- MMA issuer
      // Two 64-key halves per key tile, each with its own S / dP columns and dS buffer.
      const uint32_t id_s = tc::idesc_bf16_f32(128, 64, 0, 0);     // S, dP: N = 64 keys
      const uint32_t id_g = tc::idesc_bf16_f32(128, 128, 0, 1);    // dQ: B MN-major
      const uint32_t aQ = tc::smem_u32(sQ), adO = tc::smem_u32(sdO), adS = tc::smem_u32(sdS),
                     aKV0 = tc::smem_u32(sKV0);
      // descriptors built once; k-steps add their offset / 16 (see the key-tile kernel)
      const uint64_t dQ = tc::smem_desc_sw128(aQ, 16, 1024), dO = tc::smem_desc_sw128(adO, 16, 1024);
      const uint64_t dS = tc::smem_desc_sw128(adS, 16, 1024);
      static_assert(KV_RING == 2, "stage descriptors are selected between two stages");
      const uint64_t dKk0 = tc::smem_desc_sw128(aKV0, 16, 1024);
      const uint64_t dVk0 = tc::smem_desc_sw128(aKV0 + TILE, 16, 1024);
      const uint64_t dKm0 = tc::smem_desc_sw128(aKV0, CHUNK, 1024);
      constexpr uint64_t kStage = (uint64_t)((2 * TILE) >> 4);
      // S_h = Q K_h^T and dP_h = dO V_h^T of key tile j's half hh
      auto scores = [&](int j, int hh) {
        const uint64_t so = (j & 1) ? kStage : 0;
        const uint64_t bk = dKk0 + so + (uint64_t)((hh * HALF) >> 4);
        const uint64_t bv = dVk0 + so + (uint64_t)((hh * HALF) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // K = head dim
          const uint64_t off = (uint64_t)(((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4);
          tc::mma_f16_ss(tmem + c_s(hh), dQ + off, bk + off, id_s, kk != 0);
          tc::mma_f16_ss(tmem + c_dp(hh), dO + off, bv + off, id_s, kk != 0);
        }
        tc::mma_commit(&sh.sdp_full[hh]);
      };
      // dQ += dS_h K_h
      auto dq_prod = [&](int j, int hh) {
        const uint64_t so = (j & 1) ? kStage : 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {   // K = 64 keys of the half
          tc::mma_f16_ss(tmem + C_DQ, dS + (uint64_t)((hh * CHUNK + kk * 32) >> 4),
                         dKm0 + so + (uint64_t)(((4 * hh + kk) * 2048) >> 4), id_g,
                         (j | hh | kk) != 0 ? 1u : 0u);
        }
      };
      bool ok = tc::mbar_wait(&sh.qd_full, 0, abort_flag) &&
                tc::mbar_wait(&sh.kv_full[0], 0, abort_flag);
      bool issued = false;
      if (ok) {
        tc::fence_after_sync();
        scores(0, 0);
        scores(0, 1);
        issued = true;
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const uint32_t ph = (uint32_t)j & 1u;
        if (!tc::mbar_wait(&sh.ds_full[0], ph, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        dq_prod(j, 0);
        const bool more = j + 1 < nkv;
        if (more) {
          const int st1 = (j + 1) % KV_RING;
          if (!tc::mbar_wait(&sh.kv_full[st1], (uint32_t)((j + 1) / KV_RING) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          scores(j + 1, 0);
        }
        if (!tc::mbar_wait(&sh.ds_full[1], ph, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        dq_prod(j, 1);
        tc::mma_commit(&sh.kv_empty[j % KV_RING]);
        if (more) scores(j + 1, 1);
      }
      if (ok) tc::mma_commit(&sh.dq_done);
      if (issued) {
        tc::mma_commit(&sh.drain);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&sh.drain, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (nkv > 0) {
    // ------------------------------------------------------------------ element-wise warps
    const int q4 = warp & 3;
    const int wh = (warp - 2) >> 2;                  // column half: keys 32 wh .. of a half
    const int r = q4 * 32 + lane;                    // TMEM lane = query row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int t = (int)(q_lo + r);                   // absolute query position
    const bool qv = t < q_hi;
    const int64_t srow = (h * a.B + b) * a.Tcp + (int64_t)qt * BT + r;
    const float lse_r = a.lse_t[srow];               // log2 units (0 in the padding)
    const float dl_r = a.delta_t[srow];
    const float scale_log2 = a.scale * 1.4426950408889634f;
    bool ok = true;
    for (int j = 0; j < nkv && ok; ++j) {
      const uint32_t ph = (uint32_t)j & 1u;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        const int k0 = j * BT + 64 * hh + 32 * wh;   // this warp's first key
        const bool diag = k0 + 31 > (int)q_lo;       // some key may follow some query
        if (!tc::mbar_wait_warp(&sh.sdp_full[hh], ph, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        uint32_t rs[32], rd[32];
        tc::tmem_ld32(tmem + lane_off + c_s(hh) + 32 * wh, rs);
        tc::tmem_ld32(tmem + lane_off + c_dp(hh) + 32 * wh, rd);
        tc::tmem_ld_wait();
        uint32_t dd[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float gg[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float p = ex2(fmaf(__uint_as_float(rs[i + k]), scale_log2, -lse_r));
            float v = p * (__uint_as_float(rd[i + k]) - dl_r);
            if (diag) v = (k0 + i + k <= t && qv) ? v : 0.f;
            else v = qv ? v : 0.f;
            gg[k] = v;
          }
          dd[i >> 1] = pack2(gg[0], gg[1]);
        }
        // dS of this half (the previous tile's dQ product of this half has read the buffer:
        // its completion precedes the scores this warp has waited for)
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_unit(sdS + hh * CHUNK, r, 4 * wh + u,
                  make_uint4(dd[4 * u], dd[4 * u + 1], dd[4 * u + 2], dd[4 * u + 3]));
        fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sh.ds_full[hh]);
      }
    }
    // dQ of this query tile, written once
    if (ok && tc::mbar_wait_warp(&sh.dq_done, 0, abort_flag)) {
      tc::fence_after_sync();
      float* dqp = a.dq + ((b * a.Tc + (t - a.s)) * a.H + h) * HD;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = wh * 2 + cc;
        uint32_t rq[32];
        tc::tmem_ld32(tmem + lane_off + C_DQ + c * 32, rq);
        tc::tmem_ld_wait();
        if (qv) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dqp + c * 32 + i) =
                make_float4(__uint_as_float(rq[i]) * a.scale, __uint_as_float(rq[i + 1]) * a.scale,
                            __uint_as_float(rq[i + 2]) * a.scale,
                            __uint_as_float(rq[i + 3]) * a.scale);
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (threadIdx.x == 0 && (sh.abort || misaligned) && a.err) atomicExch(a.err, DEV_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Per (row, head): delta = sum_d dO * O and lse in log2 units, written head-major into
// [H, B, Tcp] rows padded to whole query tiles (padding = 0), so that the backward kernel can
// bulk-copy the 128 values of a query tile.  One warp per (row, head) of the chunk.
__global__ void attn_stats_kernel(int64_t B, int64_t Tc, int64_t Tcp, int64_t H,
                                  const __nv_bfloat16* __restrict__ dO,
                                  const __nv_bfloat16* __restrict__ o,
                                  const float* __restrict__ lse, float* __restrict__ lse_t,
                                  float* __restrict__ delta_t) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= H * B * Tcp) return;
  const int64_t t = w % Tcp, b = (w / Tcp) % B, h = w / (Tcp * B);
  float s = 0.f, l = 0.f;
  if (t < Tc) {
    const int64_t rh = (b * Tc + t) * H + h;
    const __nv_bfloat16* pa = dO + rh * HD;
    const __nv_bfloat16* pc = o + rh * HD;
#pragma unroll
    for (int i = 0; i < HD / 32; ++i)
      s = fmaf(__bfloat162float(pa[lane + 32 * i]), __bfloat162float(pc[lane + 32 * i]), s);
    s = warp_sum(s);
    l = lse[rh] * 1.4426950408889634f;
  }
  if (lane == 0) {
    delta_t[w] = s;
    lse_t[w] = l;
  }
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

size_t attn_bwd_tc_stats_floats(int64_t B, int64_t Tc, int64_t H) {
  return (size_t)2 * H * B * ((Tc + BT - 1) / BT) * BT;
}

// stats: scratch of attn_bwd_tc_stats_floats() floats (16-byte aligned).
// dq [B*Tc, H, HD] fp32 is overwritten; dKp/dVp [B, T, Hkv, HD] fp32 accumulate rows < s + Tc.
cudaError_t attn_bwd_tc(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                        const void* q, const void* Kp, const void* Vp, const void* o,
                        const void* dO, const float* lse, float* stats, float* dq, float* dKp,
                        float* dVp, int* err, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mdo;
  if (!map3(&mq, q, H, B * Tc) || !map3(&mk, Kp, Hkv, B * T) || !map3(&mv, Vp, Hkv, B * T) ||
      !map3(&mdo, dO, H, B * Tc))
    return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(attn_bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                KV_SMEM_BYTES);
    if (attr == cudaSuccess)
      attr = cudaFuncSetAttribute(attn_bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  Q_SMEM_BYTES);
  });
  if (attr != cudaSuccess) return attr;
  const int64_t Tcp = ((Tc + BT - 1) / BT) * BT;
  float* lse_t = stats;
  float* delta_t = stats + H * B * Tcp;
  const int64_t nw = H * B * Tcp;
  launch(attn_stats_kernel, dim3((unsigned)((nw * 32 + 255) / 256)), dim3(256), 0, st, B, Tc,
         Tcp, H, static_cast<const __nv_bfloat16*>(dO), static_cast<const __nv_bfloat16*>(o),
         lse, lse_t, delta_t);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BwdArgs a;
  a.B = B; a.T = T; a.Tc = Tc; a.s = s; a.H = H; a.Hkv = Hkv;
  a.nq = (int)((Tc + BT - 1) / BT);
  a.nkt = (int)((s + Tc + BT - 1) / BT);
  a.qb = (int)(kKvTokenBlock / BT);
  a.Tcp = Tcp;
  a.lse_t = lse_t;
  a.delta_t = delta_t;
  a.dq = dq;
  a.dKp = dKp;
  a.dVp = dVp;
  a.scale = 1.f / sqrtf((float)HD);
  a.err = err;
  // the two kernels are independent: the key-tile kernel (whose CTAs carry very unequal
  // amounts of work) runs on a side stream so that the query-tile kernel fills its tail
  SidePool* sp = side_pool();
  cudaStream_t kv_st = st;
  std::unique_lock<std::recursive_mutex> lk;
  if (sp) {
    lk = std::unique_lock<std::recursive_mutex>(sp->mu);
    e = cudaEventRecord(sp->ev[14], st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sp->s[2], sp->ev[14], 0);
    if (e != cudaSuccess) return e;
    kv_st = sp->s[2];
  }
  launch(attn_bwd_kv_kernel, dim3((unsigned)(B * Hkv * a.nkt)), dim3(kThreads),
         (size_t)KV_SMEM_BYTES, kv_st, mq, mk, mv, mdo, a);
  launch(attn_bwd_q_kernel, dim3((unsigned)(B * H * a.nq)), dim3(kThreads),
         (size_t)Q_SMEM_BYTES, st, mq, mk, mv, mdo, a);
  e = cudaGetLastError();
  if (e == cudaSuccess && sp) {
    e = cudaEventRecord(sp->ev[15], kv_st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, sp->ev[15], 0);
  }
  return e;
}

}  // namespace sbp
