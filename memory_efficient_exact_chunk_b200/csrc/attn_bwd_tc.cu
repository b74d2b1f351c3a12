// Causal GQA attention backward of one query chunk over its key prefix on the tcgen05 tensor
// cores (head_dim 128, bf16 operands, fp32 accumulation), as two kernels that each keep their
// accumulator in TMEM and write it once (no atomics; both results are deterministic and do not
// depend on how the sequence was chunked).
//
// Every product reads its A operand from TMEM (the tcgen05.mma form with A in tensor memory)
// and only its B operand from shared memory: measured on B200, an M = 128, N = 128, K = 16
// instruction then takes about 74 cycles against about 126 with both operands in shared
// memory (64 at the nominal rate), and N = 64 instructions are no faster than N = 128 ones.
// So the tile a CTA owns is copied into TMEM once (packed bf16 pairs), scores are computed
// 128 x 128 at a time, and P^T / dS^T (or dS) are written back into TMEM as packed bf16 over
// the scores they are computed from.
//
// dK/dV kernel: one CTA owns (sequence b, KV head g, 128-key tile).  It loops over the query
// heads of g's group and the chunk's query tiles that can see those keys; per (head, query
// tile) pair, in one of two 128-column score regions SP used alternately:
//   S^T  = K Q^T                  -> SP   (the element-wise warps read it out)
//   dP^T = V dO^T                 -> SP   (while the warps compute P^T = exp(S^T - lse))
//   P^T, dS^T = P^T (dP^T - delta) -> SP as packed bf16 (each warp over columns it has read)
//   dV += P^T dO,  dK += dS^T Q   (A = P^T, dS^T from TMEM; B = dO, Q from shared memory)
// K and V stay in shared memory as the A operands of the score products: the two score
// regions, not a TMEM copy of K and V, take the TMEM beside the dK / dV accumulators, so the
// tensor cores compute the next pair's scores while the element-wise warps work on this one.
// The query tiles are taken in blocks of a fixed number of tiles counted from the chunk start
// (all heads of the group within a block); after each block dK, dV are added into the fp32
// prefix accumulators (single owner; bulk asynchronous reduce-adds from shared memory, in
// block order).  A chunk whose length is a multiple of the block therefore adds exactly the
// partial sums the same queries give inside a longer chunk.  Q tiles flow through a 3-slot
// ring and dO tiles (with the pair's lse and delta) through a 2-slot ring: the scores of the
// next pair read Q first, so its copy starts a pair earlier than dO's.
//
// dQ kernel: one CTA owns (sequence b, query head h, 128-query tile); Q and dO live in TMEM.
// It loops over the key tiles of its causal prefix with two score regions used alternately,
// so the tensor cores compute the scores of key tile j + 1 while the element-wise warps work
// on tile j:  S = Q K^T, dP = dO V^T, dS = P (dP - delta) -> packed bf16 over S / dP,
// dQ += dS K (TMEM), stored once at the end.
//
// Entries with key > query, queries outside the chunk and keys outside the prefix are masked
// by selection (not by multiplication), so stale values never reach an accumulator.
// Warp roles (both kernels): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2..9
// element-wise (the warp's TMEM lane quarter is its index mod 4; the two warps of a quarter
// split the 128 columns of a score tile into halves of 64).
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
constexpr int Q_SLOTS = 3;                  // Q ring of the dK/dV kernel (S^T reads Q first:
                                            // a third slot lets its copy start a pair earlier)
constexpr int DO_SLOTS = 2;                 // dO ring of the dK/dV kernel (with the statistics)
constexpr int KV_RING = 3;                  // K/V stages of the dQ kernel (the Q/dO staging
                                            // copy lands in the last one before K/V do)
// All shared state lives in the dynamic allocation (no static shared memory), whose start is
// 1024-byte aligned as the 128-byte swizzle needs: the tiles first, then the statistics and
// the barriers.
struct KvShared {
  float stat[DO_SLOTS][2][BT];    // per dO slot: lse (log2 units), delta of the pair's queries
  // per Q slot: q_full, q_empty (the MMAs reading it have completed), q_free (the element-wise
  // warps are done with it); per dO slot: do_full (dO and the statistics), do_empty, st_free.
  // The element-wise warps use a slot only for the statistics and, at the end of a block, to
  // stage the dK / dV rows for the bulk reduce-adds (rows 0-63 in the Q slot, 64-127 in the dO
  // slot of the block's last pair).
  uint64_t kv_full, q_full[Q_SLOTS], q_empty[Q_SLOTS], q_free[Q_SLOTS], do_full[DO_SLOTS],
      do_empty[DO_SLOTS], st_free[DO_SLOTS], s_full[2], s_read[2], dp_full[2], ds_full[2],
      kv_free, drain;
  uint32_t tmem;
  int abort;
};
constexpr int KV_TILES_BYTES = (2 + Q_SLOTS + DO_SLOTS) * TILE;   // K, V, Q ring, dO ring
constexpr int KV_SMEM_BYTES = KV_TILES_BYTES + (int)sizeof(KvShared);
struct QShared {
  // per ring stage: kv_full (K and V; one wait per key tile in the MMA thread) and kv_empty
  // (the stage may be refilled)
  uint64_t qd_full, q_tmem, kv_full[KV_RING], kv_empty[KV_RING], s_full[2], s_read[2],
      dp_full[2], ds_full[2], dq_done, drain;
  uint32_t tmem;
  int abort;
};
constexpr int Q_TILES_BYTES = 2 * KV_RING * TILE;                 // KV_RING x (K, V)
constexpr int Q_SMEM_BYTES = Q_TILES_BYTES + (int)sizeof(QShared);
constexpr int kEwWarps = 8;                 // element-wise warps: 4 lane quarters x 2 column halves
constexpr int kThreads = 64 + 32 * kEwWarps;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns.  dK/dV kernel: two score regions, the fp32 accumulators dV and dK.  dQ
// kernel: Q and dO (packed bf16, 64 columns each), two score regions, dQ.
constexpr uint32_t KV_SP0 = 0, KV_DV = 256, KV_DK = 384;
constexpr uint32_t Q_QT = 0, Q_OT = 64, Q_SP0 = 128, Q_DQ = 384;
__device__ __forceinline__ uint32_t kv_sp(int x) { return KV_SP0 + 128u * (uint32_t)x; }
__device__ __forceinline__ uint32_t q_sp(int x) { return Q_SP0 + 128u * (uint32_t)x; }
// Packed-bf16 A operands written back over a score region: the warps of column half wh own
// score columns [64 wh, 64 wh + 64).  dQ kernel: dS of those 64 keys at the start of the range,
// so the k-step kk of a K = 128 product (16 keys) starts at column 64 (kk / 4) + 8 (kk % 4).
// dK/dV kernel: per 32 queries (columns [32 c, 32 c + 32) of the range), P^T at +0 and dS^T at
// +16, so the k-step kk (16 queries) of P^T starts at 64 (kk / 4) + 32 ((kk / 2) % 2) +
// 8 (kk % 2) and that of dS^T 16 columns later.
__device__ __forceinline__ uint32_t packed_col(int kk) {
  return 64u * (uint32_t)(kk >> 2) + 8u * (uint32_t)(kk & 3);
}
__device__ __forceinline__ uint32_t kv_packed_col(int kk) {
  return 64u * (uint32_t)(kk >> 2) + 32u * (uint32_t)((kk >> 1) & 1) + 8u * (uint32_t)(kk & 1);
}

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
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
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
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
// Bulk asynchronous reduce-add of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// fp32 values from shared memory into global memory, tracked in the calling thread's bulk
// groups; the shared-memory writes it reads must precede it behind fence.proxy.async.
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, const float* ssrc,
                                                    uint32_t bytes) {
  asm volatile("fence.proxy.async.shared::cta;\n\t"
               "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;\n\t"
               "cp.async.bulk.commit_group;" ::"l"(reinterpret_cast<uint64_t>(gdst)),
               "r"(tc::smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
// the calling thread's bulk operations have read their shared-memory sources
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// the calling thread's bulk operations have completed (global writes done)
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Copy this thread's row r of a 128 x 128 bf16 tile staged by TMA (two 64-column chunks, each
// 128 rows of 128 bytes with the 128-byte swizzle) into TMEM as packed bf16 pairs: chunk c
// (columns 64 c ..) goes to TMEM columns col0 + 32 c ..; the caller's warp owns the lane.
__device__ __forceinline__ void tile_row_to_tmem(const uint8_t* tile, int r, int c,
                                                 uint32_t taddr) {
  uint32_t w[32];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + c * CHUNK + r * 128 +
                                                    ((u ^ (r & 7)) << 4));
    w[4 * u] = v.x;
    w[4 * u + 1] = v.y;
    w[4 * u + 2] = v.z;
    w[4 * u + 3] = v.w;
  }
  tmem_st32(taddr, w);
}

// ================================================================== dK / dV kernel
// The work of a key tile, pair by pair: (query head hh of the group, query tile qi) for the
// query tiles i0 .. nq - 1, ordered block by block (qb tiles, counted from the chunk start)
// and head-major inside a block; first / last: the pair opens / closes its block, left: pairs
// after it in its block.  Every role of the CTA walks the same sequence with its own iterator
// (no divisions per pair).
struct PairPos {
  int64_t hh, qi;
  bool first, last;
  int left;
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
    p.left = (grp - 1 - hi) * nbt + (nbt - 1 - t);
    p.last = p.left == 0;
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
  uint8_t* sQ0 = sV + TILE;                      // Q slot i at sQ0 + i TILE
  uint8_t* sdO0 = sQ0 + Q_SLOTS * TILE;          // dO slot i at sdO0 + i TILE
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
    for (int i = 0; i < Q_SLOTS; ++i) {
      tc::mbar_init(&sh.q_full[i], 1);
      tc::mbar_init(&sh.q_empty[i], 1);
      tc::mbar_init(&sh.q_free[i], kEwWarps);
    }
    for (int i = 0; i < DO_SLOTS; ++i) {
      tc::mbar_init(&sh.do_full[i], 1);
      tc::mbar_init(&sh.do_empty[i], 1);
      tc::mbar_init(&sh.st_free[i], kEwWarps);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(&sh.s_full[x], 1);
      tc::mbar_init(&sh.s_read[x], kEwWarps);
      tc::mbar_init(&sh.dp_full[x], 1);
      tc::mbar_init(&sh.ds_full[x], kEwWarps);
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
      int issued_q = 0, issued_do = 0;
      PairIter it;
      it.init((int)i0, a.nq, (int)grp, a.qb);
      for (int j = 0; j < npairs; ++j, it.next()) {
        const PairPos pos = it.pos(g);
        const int qs = j % Q_SLOTS, ds = j % DO_SLOTS;
        const uint32_t qph = (uint32_t)(j / Q_SLOTS) & 1u, dph = (uint32_t)(j / DO_SLOTS) & 1u;
        const int32_t qrow = (int32_t)(b * a.Tc + pos.qi * BT);
        if (!tc::mbar_wait(&sh.q_empty[qs], qph ^ 1u, abort_flag) ||
            !tc::mbar_wait(&sh.q_free[qs], qph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sQ = sQ0 + qs * TILE;
        tc::mbar_expect_tx(&sh.q_full[qs], TILE);
        tc::tma_load_3d(sQ, &tmQ, &sh.q_full[qs], 0, (int32_t)pos.hh, qrow);
        tc::tma_load_3d(sQ + CHUNK, &tmQ, &sh.q_full[qs], 64, (int32_t)pos.hh, qrow);
        issued_q = j + 1;
        if (!tc::mbar_wait(&sh.do_empty[ds], dph ^ 1u, abort_flag) ||
            !tc::mbar_wait(&sh.st_free[ds], dph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sdO = sdO0 + ds * TILE;
        const int64_t srow = (pos.hh * a.B + b) * a.Tcp + pos.qi * BT;
        tc::mbar_expect_tx(&sh.do_full[ds], TILE + 2 * BT * 4);
        tc::tma_load_3d(sdO, &tmdO, &sh.do_full[ds], 0, (int32_t)pos.hh, qrow);
        tc::tma_load_3d(sdO + CHUNK, &tmdO, &sh.do_full[ds], 64, (int32_t)pos.hh, qrow);
        tc::bulk_load(&sh.stat[ds][0][0], a.lse_t + srow, BT * 4, &sh.do_full[ds]);
        tc::bulk_load(&sh.stat[ds][1][0], a.delta_t + srow, BT * 4, &sh.do_full[ds]);
        issued_do = j + 1;
      }
      if (!ok) {
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&sh.kv_full, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        for (int j = issued_q > Q_SLOTS ? issued_q - Q_SLOTS : 0; j < issued_q; ++j) {
          const uint32_t pj = (uint32_t)(j / Q_SLOTS) & 1u;
          while (!tc::mbar_try_wait(&sh.q_full[j % Q_SLOTS], pj) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        }
        for (int j = issued_do > DO_SLOTS ? issued_do - DO_SLOTS : 0; j < issued_do; ++j) {
          const uint32_t pj = (uint32_t)(j / DO_SLOTS) & 1u;
          while (!tc::mbar_try_wait(&sh.do_full[j % DO_SLOTS], pj) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1) {
    if (npairs > 0) {
      // ---------------------------------------------------------------- MMA issuer
      // the whole warp runs the issue loop; one elected lane issues the MMAs and commits (as in
      // the dQ kernel)
      const bool leader = tc::elect_one_sync();
      // order: S^T_0 | dP^T_j S^T_{j+1} grads_j | ...  (S^T_{j+1} goes into the other score
      // region, whose P^T / dS^T the grads of pair j - 1, issued before it, have read)
      const uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);    // S^T, dP^T: B K-major
      const uint32_t id_g = tc::idesc_bf16_f32(128, 128, 0, 1);    // dV, dK: B MN-major
      const uint32_t aQ0 = tc::smem_u32(sQ0), adO0 = tc::smem_u32(sdO0);
      // shared-memory descriptors built once; a k-step or a slot adds its byte offset / 16 to
      // the start address field (the tiles sit below 256 KB, so the field cannot carry over)
      const uint64_t dK = tc::smem_desc_sw128(tc::smem_u32(sK), 16, 1024);
      const uint64_t dV = tc::smem_desc_sw128(tc::smem_u32(sV), 16, 1024);
      const uint64_t dQk0 = tc::smem_desc_sw128(aQ0, 16, 1024);
      const uint64_t dOk0 = tc::smem_desc_sw128(adO0, 16, 1024);
      const uint64_t dQm0 = tc::smem_desc_sw128(aQ0, CHUNK, 1024);
      const uint64_t dOm0 = tc::smem_desc_sw128(adO0, CHUNK, 1024);
      constexpr uint64_t kSlot = (uint64_t)(TILE >> 4);
      // S^T_j = K Q_j^T into score region j & 1
      auto scores = [&](int j) {
        const uint64_t so = (uint64_t)(j % Q_SLOTS) * kSlot;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // K = head dim
            const uint64_t off = (uint64_t)(((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4);
            tc::mma_f16_ss(tmem + kv_sp(j & 1), dK + off, dQk0 + so + off, id_s, kk != 0);
          }
          tc::mma_commit(&sh.s_full[j & 1]);
        }
        __syncwarp();
      };
      bool ok = tc::mbar_wait_warp(&sh.kv_full, 0, abort_flag) &&
                tc::mbar_wait_warp(&sh.q_full[0], 0, abort_flag);
      bool issued = false;
      if (ok) {
        tc::fence_after_sync();
        scores(0);
        issued = true;
      }
      int nflush = 0;
      PairIter it;
      it.init((int)i0, a.nq, (int)grp, a.qb);
      for (int j = 0; j < npairs && ok; ++j, it.next()) {
        const PairPos pos = it.pos(g);
        const int x = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        const int qs = j % Q_SLOTS, ds = j % DO_SLOTS;
        const uint64_t sq = (uint64_t)qs * kSlot, sd = (uint64_t)ds * kSlot;
        // dP^T_j = V dO_j^T over S^T_j once the element-wise warps have read S^T_j
        if (!tc::mbar_wait_warp(&sh.s_read[x], ph, abort_flag) ||
            !tc::mbar_wait_warp(&sh.do_full[ds], (uint32_t)(j / DO_SLOTS) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4);
            tc::mma_f16_ss(tmem + kv_sp(x), dV + off, dOk0 + sd + off, id_s, kk != 0);
          }
          tc::mma_commit(&sh.dp_full[x]);
        }
        __syncwarp();
        if (j + 1 < npairs) {
          if (!tc::mbar_wait_warp(&sh.q_full[(j + 1) % Q_SLOTS],
                                  (uint32_t)((j + 1) / Q_SLOTS) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          scores(j + 1);
        }
        // dV += P^T dO, dK += dS^T Q once P^T, dS^T are in TMEM; a new block overwrites dK / dV,
        // so the element-wise warps must have added the last one
        if (!tc::mbar_wait_warp(&sh.ds_full[x], ph, abort_flag)) { ok = false; break; }
        if (pos.first && j > 0) {
          if (!tc::mbar_wait_warp(&sh.kv_free, (uint32_t)nflush & 1u, abort_flag)) {
            ok = false;
            break;
          }
          ++nflush;
        }
        tc::fence_after_sync();
        if (leader) {
          // dK first: its completion releases the Q slot, whose next copy is two pairs ahead
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // K = 128 queries
            const uint64_t offm = (uint64_t)((kk * 2048) >> 4);          // MN-major k-step
            mma_f16_ts(tmem + KV_DK, tmem + kv_sp(x) + kv_packed_col(kk) + 16,
                       dQm0 + sq + offm, id_g, (!pos.first || kk != 0) ? 1u : 0u);
          }
          tc::mma_commit(&sh.q_empty[qs]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t offm = (uint64_t)((kk * 2048) >> 4);
            mma_f16_ts(tmem + KV_DV, tmem + kv_sp(x) + kv_packed_col(kk), dOm0 + sd + offm, id_g,
                       (!pos.first || kk != 0) ? 1u : 0u);
          }
          tc::mma_commit(&sh.do_empty[ds]);
        }
        __syncwarp();
      }
      if (issued) {
        if (leader) tc::mma_commit(&sh.drain);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&sh.drain, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (npairs > 0) {
    // ------------------------------------------------------------------ element-wise warps
    const int q4 = warp & 3;
    const int wh = (warp - 2) >> 2;                  // column half: queries 64 wh .. 64 wh + 63
    const int r = q4 * 32 + lane;                    // TMEM lane = key row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int kpos = (int)(k_lo + r);
    const float scale_log2 = a.scale * 1.4426950408889634f;
    const int e32 = (int)e;
    const bool kv = kpos < e32;
    const int64_t ko = ((b * a.T + kpos) * a.Hkv + g) * HD;
    bool ok = true;
    PairIter it;
    it.init((int)i0, a.nq, (int)grp, a.qb);
    for (int j = 0; j < npairs && ok; ++j, it.next()) {
      const int x = j & 1;
      const uint32_t ph = (uint32_t)(j >> 1) & 1u;
      const PairPos pos = it.pos(g);
      const uint32_t sp = tmem + lane_off + kv_sp(x) + 64u * (uint32_t)wh;  // this warp's columns
      const int qs = j % Q_SLOTS, ds = j % DO_SLOTS;   // the dO slot holds lse and delta
      if (!tc::mbar_wait_warp(&sh.do_full[ds], (uint32_t)(j / DO_SLOTS) & 1u, abort_flag)) {
        ok = false;
        break;
      }
      const int qoff = 64 * wh;                        // this warp's queries within the tile
      const int q0 = (int)(a.s + pos.qi * BT) + qoff;  // absolute position of its first query
      // no masking needed when every key of the tile precedes every (valid) query here
      const bool full = (k_lo + BT - 1 <= q0) && (pos.qi * BT + qoff + 64 <= a.Tc);
      const float* lse_s = sh.stat[ds][0] + qoff;
      const float* delta_s = sh.stat[ds][1] + qoff;
      // S^T of this warp's 64 queries, one TMEM load
      if (!tc::mbar_wait_warp(&sh.s_full[x], ph, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      uint32_t p[64];
      tc::tmem_ld64(sp, p);
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sh.s_read[x]);     // SP may take dP^T now
      // P^T = exp(S^T * scale - lse) while the tensor cores compute dP^T
#pragma unroll
      for (int i4 = 0; i4 < 16; ++i4) {
        const float4 lv = reinterpret_cast<const float4*>(lse_s)[i4];
        const float la[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = i4 * 4 + k;
          float v = ex2(fmaf(__uint_as_float(p[i]), scale_log2, -la[k]));
          if (!full) {
            const int qpos = q0 + i;
            v = ((kpos <= qpos) && (qpos < e32)) ? v : 0.f;
          }
          p[i] = __float_as_uint(v);
        }
      }
      if (!tc::mbar_wait_warp(&sh.dp_full[x], ph, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      // dS^T = P^T (dP^T - delta), per 32 queries: P^T and dS^T of those queries go back as
      // packed bf16 over the 32 dP^T columns just read (P^T at +0, dS^T at +16)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t rd[32];
        tc::tmem_ld32(sp + 32u * (uint32_t)c, rd);
        tc::tmem_ld_wait();
        uint32_t pw[16], dsw[16];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 dv = reinterpret_cast<const float4*>(delta_s)[8 * c + i4];
          const float da[4] = {dv.x, dv.y, dv.z, dv.w};
          float pp[4], gg[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            pp[k] = __uint_as_float(p[32 * c + 4 * i4 + k]);
            gg[k] = pp[k] * (__uint_as_float(rd[4 * i4 + k]) - da[k]);
          }
          pw[2 * i4] = pack2(pp[0], pp[1]);
          pw[2 * i4 + 1] = pack2(pp[2], pp[3]);
          dsw[2 * i4] = pack2(gg[0], gg[1]);
          dsw[2 * i4 + 1] = pack2(gg[2], gg[3]);
        }
        tmem_st16(sp + 32u * (uint32_t)c, pw);
        tmem_st16(sp + 32u * (uint32_t)c + 16u, dsw);
      }
      tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sh.ds_full[x]);
      if (!pos.last) {
        if (lane == 0) {
          tc::mbar_arrive(&sh.st_free[ds]);                // statistics read
          tc::mbar_arrive(&sh.q_free[qs]);                 // the Q slot is not staged
        }
        continue;
      }
      // end of a block: add its dK, dV into the fp32 prefix accumulators (single owner); the
      // release of this pair's Q/dO stage is committed after its last dK / dV product
      if (!tc::mbar_wait_warp(&sh.do_empty[ds], (uint32_t)(j / DO_SLOTS) & 1u, abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      // The Q and dO slots of the block's last pair (32 KB each) are free: dK, then dV, of the
      // block are staged there as fp32 rows (512 B per key row, rows 0-63 in the Q slot and
      // 64-127 in the dO slot; this lane's row, this warp's 64 columns) and added
      // into the prefix accumulators by bulk asynchronous reduce-adds, one per (row, column
      // half), so the flush does not wait for global memory.  This CTA is the only writer of
      // these rows; the previous block's reduce-adds into them have completed before these
      // are issued, so every element receives its block sums in block order.
      float* srow = reinterpret_cast<float*>(r < 64 ? sQ0 + qs * TILE : sdO0 + ds * TILE) +
                    (r & 63) * HD + wh * 64;
      bulk_wait_all();
#pragma unroll 1
      for (int acc = 0; acc < 2; ++acc) {
        const bool isk = acc == 0;
        const float f = isk ? a.scale : 1.f;
        if (!isk) bulk_wait_read();                    // the dK rows have been read
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t rv[32];
          tc::tmem_ld32(tmem + lane_off + (isk ? KV_DK : KV_DV) + (wh * 2 + c2) * 32, rv);
          tc::tmem_ld_wait();
          // rows past the prefix end are not staged (nothing reads them; a stray generic
          // write could also land after the next TMA write of the stage)
          if (kv) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<float4*>(srow + c2 * 32)[i] =
                  make_float4(__uint_as_float(rv[4 * i]) * f, __uint_as_float(rv[4 * i + 1]) * f,
                              __uint_as_float(rv[4 * i + 2]) * f,
                              __uint_as_float(rv[4 * i + 3]) * f);
          }
        }
        if (kv) bulk_reduce_add_f32((isk ? a.dKp : a.dVp) + ko + wh * 64, srow, 64 * 4);
      }
      // dK / dV are out of TMEM: the next block's products may overwrite them
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0 && j + 1 < npairs) tc::mbar_arrive(&sh.kv_free);
      bulk_wait_read();                                // the staged rows have been read
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&sh.st_free[ds]);
        tc::mbar_arrive(&sh.q_free[qs]);
      }
    }
    bulk_wait_all();                                   // the last block's adds have landed
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
  uint8_t* sKV0 = smem_raw;                      // ring stage st: K at sKV0 + 2 st TILE, V after
  // Q and dO are staged in the last ring stage; the producer refills that stage with K/V only
  // once the element-wise warps have copied them into TMEM
  uint8_t* sQ = sKV0 + 2 * (KV_RING - 1) * TILE;
  uint8_t* sdO = sQ + TILE;
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
    tc::mbar_init(&sh.q_tmem, kEwWarps);
    for (int i = 0; i < KV_RING; ++i) {
      tc::mbar_init(&sh.kv_full[i], 1);
      tc::mbar_init(&sh.kv_empty[i], 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(&sh.s_full[x], 1);
      tc::mbar_init(&sh.s_read[x], kEwWarps);
      tc::mbar_init(&sh.dp_full[x], 1);
      tc::mbar_init(&sh.ds_full[x], kEwWarps);
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
        // the last stage holds the Q / dO staging copy until it is in TMEM
        if (j == KV_RING - 1 && !tc::mbar_wait(&sh.q_tmem, 0, abort_flag)) { ok = false; break; }
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
        for (int j = issued > KV_RING ? issued - KV_RING : 0; j < issued; ++j) {
          const uint32_t pj = (uint32_t)(j / KV_RING) & 1u;
          while (!tc::mbar_try_wait(&sh.kv_full[j % KV_RING], pj) &&
                 tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1) {
    if (nkv > 0) {
      // the whole warp runs the issue loop (waits, bookkeeping); one elected lane issues the
      // MMAs and their commits: a lone lane in a divergent branch gets far fewer issue slots
      // while the element-wise warps of its sub-partition issue back to back
      const bool leader = tc::elect_one_sync();
      // ---------------------------------------------------------------- MMA issuer
      // order: S_0 | dP_j S_{j+1} dQ_j | ...  (S_{j+1} goes into the other score region, whose
      // previous dS has been read by dQ_{j-1}, issued before it)
      const uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);    // S, dP: B K-major
      const uint32_t id_g = tc::idesc_bf16_f32(128, 128, 0, 1);    // dQ: B MN-major
      const uint32_t aKV0 = tc::smem_u32(sKV0);
      const uint64_t dKk0 = tc::smem_desc_sw128(aKV0, 16, 1024);
      const uint64_t dVk0 = tc::smem_desc_sw128(aKV0 + TILE, 16, 1024);
      const uint64_t dKm0 = tc::smem_desc_sw128(aKV0, CHUNK, 1024);
      constexpr uint64_t kStage = (uint64_t)((2 * TILE) >> 4);   // 192 KB of stages < 256 KB
      // S_j = Q K_j^T into score region j & 1
      auto scores = [&](int j) {
        const uint64_t so = (uint64_t)(j % KV_RING) * kStage;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // K = head dim
            const uint64_t off = so + (uint64_t)(((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4);
            mma_f16_ts(tmem + q_sp(j & 1), tmem + Q_QT + 8 * kk, dKk0 + off, id_s, kk != 0);
          }
          tc::mma_commit(&sh.s_full[j & 1]);
        }
        __syncwarp();
      };
      bool ok = tc::mbar_wait_warp(&sh.q_tmem, 0, abort_flag) &&   // Q, dO copied into TMEM
                tc::mbar_wait_warp(&sh.kv_full[0], 0, abort_flag);
      bool issued = false;
      if (ok) {
        tc::fence_after_sync();
        scores(0);
        issued = true;
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int x = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        const uint64_t so = (uint64_t)(j % KV_RING) * kStage;
        // dP_j = dO V_j^T over S_j once the element-wise warps have read S_j (V_j arrived with
        // K_j, whose barrier was waited for before S_j)
        if (!tc::mbar_wait_warp(&sh.s_read[x], ph, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t off = so + (uint64_t)(((kk >> 2) * CHUNK + (kk & 3) * 32) >> 4);
            mma_f16_ts(tmem + q_sp(x), tmem + Q_OT + 8 * kk, dVk0 + off, id_s, kk != 0);
          }
          tc::mma_commit(&sh.dp_full[x]);
        }
        __syncwarp();
        if (j + 1 < nkv) {
          const int st1 = (j + 1) % KV_RING;
          if (!tc::mbar_wait_warp(&sh.kv_full[st1], (uint32_t)((j + 1) / KV_RING) & 1u,
                                  abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          scores(j + 1);
        }
        // dQ += dS_j K_j
        if (!tc::mbar_wait_warp(&sh.ds_full[x], ph, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // K = 128 keys
            mma_f16_ts(tmem + Q_DQ, tmem + q_sp(x) + packed_col(kk),
                       dKm0 + so + (uint64_t)((kk * 2048) >> 4), id_g, (j | kk) != 0 ? 1u : 0u);
          }
          tc::mma_commit(&sh.kv_empty[j % KV_RING]);
        }
        __syncwarp();
      }
      if (ok && leader) tc::mma_commit(&sh.dq_done);
      if (issued) {
        if (leader) tc::mma_commit(&sh.drain);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&sh.drain, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else if (nkv > 0) {
    // ------------------------------------------------------------------ element-wise warps
    const int q4 = warp & 3;
    const int wh = (warp - 2) >> 2;                  // column half: keys 64 wh .. of a tile
    const int r = q4 * 32 + lane;                    // TMEM lane = query row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int t = (int)(q_lo + r);                   // absolute query position
    const bool qv = t < q_hi;
    const int64_t srow = (h * a.B + b) * a.Tcp + (int64_t)qt * BT + r;
    const float lse_r = a.lse_t[srow];               // log2 units (0 in the padding)
    const float dl_r = a.delta_t[srow];
    const float scale_log2 = a.scale * 1.4426950408889634f;
    bool ok = tc::mbar_wait_warp(&sh.qd_full, 0, abort_flag);
    if (ok) {
      // Q and dO rows of this lane into TMEM (packed), this warp's 64-column half of each
      tile_row_to_tmem(sQ, r, wh, tmem + lane_off + Q_QT + 32u * (uint32_t)wh);
      tile_row_to_tmem(sdO, r, wh, tmem + lane_off + Q_OT + 32u * (uint32_t)wh);
      tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sh.q_tmem);
    }
    for (int j = 0; j < nkv && ok; ++j) {
      const int x = j & 1;
      const uint32_t ph = (uint32_t)(j >> 1) & 1u;
      const uint32_t sp = tmem + lane_off + q_sp(x) + 64u * (uint32_t)wh;
      const int k0 = j * BT + 64 * wh;               // this warp's first key
      const bool diag = k0 + 63 > (int)q_lo;         // some key may follow some query
      if (!tc::mbar_wait_warp(&sh.s_full[x], ph, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      uint32_t p[64];
      tc::tmem_ld64(sp, p);                            // this warp's 64 scores, one load
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sh.s_read[x]);   // the region may take dP_j now
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        float v = ex2(fmaf(__uint_as_float(p[i]), scale_log2, -lse_r));
        if (diag) v = (k0 + i <= t && qv) ? v : 0.f;
        else v = qv ? v : 0.f;
        p[i] = __float_as_uint(v);
      }
      if (!tc::mbar_wait_warp(&sh.dp_full[x], ph, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      // dS = P (dP - delta), packed over this warp's first 32 columns (all 64 read above)
      uint32_t rd[64];
      tc::tmem_ld64(sp, rd);
      tc::tmem_ld_wait();
      uint32_t dw[32];
#pragma unroll
      for (int i = 0; i < 32; ++i)
        dw[i] = pack2(__uint_as_float(p[2 * i]) * (__uint_as_float(rd[2 * i]) - dl_r),
                      __uint_as_float(p[2 * i + 1]) * (__uint_as_float(rd[2 * i + 1]) - dl_r));
      tmem_st32(sp, dw);
      tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sh.ds_full[x]);
    }
    // dQ of this query tile, written once
    if (ok && tc::mbar_wait_warp(&sh.dq_done, 0, abort_flag)) {
      tc::fence_after_sync();
      float* dqp = a.dq + ((b * a.Tc + (t - a.s)) * a.H + h) * HD;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = wh * 2 + cc;
        uint32_t rq[32];
        tc::tmem_ld32(tmem + lane_off + Q_DQ + c * 32, rq);
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
