// Causal GQA attention forward of one query chunk over its key prefix on the tcgen05 tensor
// cores (head_dim 128, bf16 operands, fp32 softmax statistics and accumulation).
//
// One CTA per (sequence b, query head h, 128-row query tile).  Warp roles:
//   warp 0      : TMA producer (Q once; K and V tiles of 128 keys through 2-stage rings)
//   warp 1      : TMEM owner + MMA issuer: S_j = Q K_j^T into one of two TMEM score buffers,
//                 O += P_j V_j into the TMEM output accumulator
//   warps 2..5  : softmax, one thread per query row: read S_j from TMEM, causal mask, online
//                 max / sum in the exp2 domain, P_j (bf16) into shared memory in the layout the
//                 next MMA reads, lazy rescale of O in TMEM, final O / l and log-sum-exp.
// The running maximum used as the exponent reference is only raised when the row maximum
// exceeds it by more than 2^8 (P <= 256), so O is rescaled rarely; the result is exact up to
// rounding because P, l and O share that reference.
// Key tiles are visited in order 0, 1, ... up to the query tile's diagonal; masked entries are
// exactly zero, so each query row's result does not depend on how the sequence was chunked.
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
constexpr int SMEM_BYTES = TILE_BYTES                 // Q
                           + 2 * KV_STAGES * TILE_BYTES  // K, V rings
                           + TILE_BYTES                // P
                           + 1024;                     // alignment slack
constexpr int kThreads = 192;
constexpr uint32_t TMEM_COLS = 512;     // S0 [0,128) S1 [128,256) O [256,384)
constexpr uint32_t O_COL = 256;
constexpr float kRescaleThreshold = 8.f;  // log2 units

struct FwdArgs {
  int64_t B, T, Tc, s, H, Hkv;
  int nq;                 // query tiles per sequence
  void* o;                // [B*Tc, H, HD] bf16
  float* lse;             // [B*Tc, H]  natural log
  float scale_log2;       // log2(e) / sqrt(hd)
  int* err;
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
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// generic-proxy shared-memory writes -> visible to the tensor cores (async proxy)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

// Store 8 bf16 (16 bytes) of row r, 16-byte unit u (0..15 over 128 columns) of a 128 x 128
// K-major tile with 128-byte swizzle (two 64-column chunks).
__device__ __forceinline__ void st_tile_unit(uint8_t* tile, int r, int u, uint4 v) {
  const int chunk = u >> 3, uu = u & 7;
  uint8_t* p = tile + chunk * CHUNK_BYTES + r * 128 + ((uu ^ (r & 7)) << 4);
  *reinterpret_cast<uint4*>(p) = v;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full, k_full[KV_STAGES], k_empty[KV_STAGES], v_full[KV_STAGES],
      v_empty[KV_STAGES], s_full[2], s_empty[2], p_full, pv_done, drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TILE_BYTES;
  uint8_t* sV = sK + KV_STAGES * TILE_BYTES;
  uint8_t* sP = sV + KV_STAGES * TILE_BYTES;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &abort_sh;

  // heavy (late) query tiles first
  const int qt = a.nq - 1 - (int)(blockIdx.x % a.nq);
  const int64_t h = (blockIdx.x / a.nq) % a.H;
  const int64_t b = blockIdx.x / (a.nq * a.H);
  const int64_t g = h / (a.H / a.Hkv);
  const int64_t q_lo = a.s + (int64_t)qt * BQ;                 // absolute position of row 0
  const int64_t q_hi = a.s + imin((int64_t)(qt + 1) * BQ, a.Tc);  // one past the last valid row
  const int nkv = (int)((q_hi + BKV - 1) / BKV);              // key tiles 0 .. nkv-1

  if (threadIdx.x == 0) {
    tc::mbar_init(&q_full, 1);
    for (int i = 0; i < KV_STAGES; ++i) {
      tc::mbar_init(&k_full[i], 1);
      tc::mbar_init(&k_empty[i], 1);
      tc::mbar_init(&v_full[i], 1);
      tc::mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&s_full[i], 1);
      tc::mbar_init(&s_empty[i], 4);
    }
    tc::mbar_init(&p_full, 4);
    tc::mbar_init(&pv_done, 1);
    tc::mbar_init(&drain_bar, 1);
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
      const int32_t qrow = (int32_t)(b * a.Tc + (int64_t)qt * BQ);
      tc::mbar_expect_tx(&q_full, TILE_BYTES);
      tc::tma_load_3d(sQ, &tmQ, &q_full, 0, (int32_t)h, qrow);
      tc::tma_load_3d(sQ + CHUNK_BYTES, &tmQ, &q_full, 64, (int32_t)h, qrow);
      uint32_t issued = 0;
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t ph = (uint32_t)(j / KV_STAGES) & 1u;
        const int32_t krow = (int32_t)(b * a.T + (int64_t)j * BKV);
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
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);   // Q K^T: both K-major
      const uint32_t id_o = tc::idesc_bf16_f32(128, 128, 0, 1);   // P V: V is MN-major
      const uint32_t aQ = tc::smem_u32(sQ), aK = tc::smem_u32(sK), aV = tc::smem_u32(sV),
                     aP = tc::smem_u32(sP);
      bool ok = tc::mbar_wait(&q_full, 0, abort_flag);
      bool issued = false;
      // shared-memory descriptors built once; a k-step or a ring stage adds its byte offset / 16
      // to the start address field (the tiles sit below 256 KB, so the field cannot carry over)
      static_assert(KV_STAGES == 2, "stage descriptors are selected between two stages");
      const uint64_t dQ = tc::smem_desc_sw128(aQ, 16, 1024);
      const uint64_t dK0 = tc::smem_desc_sw128(aK, 16, 1024);
      const uint64_t dP = tc::smem_desc_sw128(aP, 16, 1024);
      const uint64_t dV0 = tc::smem_desc_sw128(aV, CHUNK_BYTES, 1024);
      constexpr uint64_t kStage = (uint64_t)(TILE_BYTES >> 4);
      auto do_pv = [&](int jj) -> bool {
        const int st = jj % KV_STAGES;
        const uint32_t ph = (uint32_t)(jj / KV_STAGES) & 1u;
        if (!tc::mbar_wait(&p_full, (uint32_t)jj & 1u, abort_flag)) return false;
        if (!tc::mbar_wait(&v_full[st], ph, abort_flag)) return false;
        tc::fence_after_sync();
        const uint64_t vb = dV0 + (st ? kStage : 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = dP + (uint64_t)(((kk >> 2) * CHUNK_BYTES + (kk & 3) * 32) >> 4);
          const uint64_t bd = vb + (uint64_t)((kk * 2048) >> 4);
          tc::mma_f16_ss(tmem + O_COL, ad, bd, id_o, (jj | kk) != 0 ? 1u : 0u);
        }
        tc::mma_commit(&pv_done);
        tc::mma_commit(&v_empty[st]);
        return true;
      };
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t ph = (uint32_t)(j / KV_STAGES) & 1u;
        const int sb = j & 1;
        const uint32_t sph = (uint32_t)(j >> 1) & 1u;
        if (!tc::mbar_wait(&k_full[st], ph, abort_flag)) { ok = false; break; }
        if (!tc::mbar_wait(&s_empty[sb], sph ^ 1u, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        const uint64_t kb = dK0 + (st ? kStage : 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * CHUNK_BYTES + (kk & 3) * 32) >> 4);
          tc::mma_f16_ss(tmem + (uint32_t)(sb * 128), dQ + off, kb + off, id_s, kk != 0 ? 1u : 0u);
        }
        issued = true;
        tc::mma_commit(&s_full[sb]);
        tc::mma_commit(&k_empty[st]);
        if (j >= 1 && !do_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nkv >= 1) ok = do_pv(nkv - 1);
      if (issued) {
        tc::mma_commit(&drain_bar);
        const uint64_t t0 = tc::globaltimer_ns();
        while (!tc::mbar_try_wait(&drain_bar, 0) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {}
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // query row within the tile
    const int64_t t = q_lo + r;                   // absolute position
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      if (!tc::mbar_wait_warp(&s_full[sb], (uint32_t)(j >> 1) & 1u, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tc::tmem_ld32(tmem + lane_off + (uint32_t)(sb * 128 + c * 32), rr);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(rr[i]);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s_empty[sb]);
      // scale into the exp2 domain; only tiles that reach past the first query need the
      // causal mask
      const int64_t k0 = (int64_t)j * BKV;
      const bool diag = k0 + BKV - 1 > q_lo;
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (diag) {
        const int lim = (int)(t - k0);             // keys k0 + i with i > lim are masked
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float x = (i <= lim) ? sv[i] * a.scale_log2 : -INFINITY;
          sv[i] = x;
          m4[i & 3] = fmaxf(m4[i & 3], x);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float x = sv[i] * a.scale_log2;
          sv[i] = x;
          m4[i & 3] = fmaxf(m4[i & 3], x);
        }
      }
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      float corr = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleThreshold) {
        const float mn = mx;
        corr = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mn);
        rescale = (j > 0);
        m_ref = mn;
        l *= corr;
      }
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float p0 = fast_exp2(sv[2 * i] - m_ref);
        const float p1 = fast_exp2(sv[2 * i + 1] - m_ref);
        s4[i & 3] += p0 + p1;
        pk[i] = pack_bf16(p0, p1);
      }
      const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      l += sum;
      // P_j may overwrite P_{j-1} (and O may be rescaled) once O += P_{j-1} V_{j-1} is done
      if (j >= 1) {
        if (!tc::mbar_wait_warp(&pv_done, (uint32_t)(j - 1) & 1u, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
      }
      // warp-uniform decision: any lane that needs a rescale makes the warp do it
      if (__any_sync(0xffffffffu, rescale)) {
        const float f = rescale ? corr : 1.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t rr[32];
          const uint32_t ta = tmem + lane_off + O_COL + (uint32_t)(c * 32);
          tc::tmem_ld32(ta, rr);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
          tmem_st32(ta, rr);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int u = 0; u < 16; ++u)
        st_tile_unit(sP, r, u, make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]));
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full);
    }
    // final: wait for the last O += P V, normalise, store
    if (ok && nkv >= 1 &&
        tc::mbar_wait_warp(&pv_done, (uint32_t)(nkv - 1) & 1u, abort_flag)) {
      tc::fence_after_sync();
      const bool row_ok = t < q_hi;
      const float inv = 1.f / l;
      const int64_t grow = b * a.Tc + (t - a.s);
      __nv_bfloat16* op = static_cast<__nv_bfloat16*>(a.o) + (grow * a.H + h) * HD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        tc::tmem_ld32(tmem + lane_off + O_COL + (uint32_t)(c * 32), rr);
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

cudaError_t attn_fwd_tc(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                        const void* q, const void* Kp, const void* Vp, void* o, float* lse,
                        int* err, cudaStream_t st) {
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
  a.o = o;
  a.lse = lse;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  a.err = err;
  const int64_t grid = B * H * a.nq;
  launch(attn_fwd_tc_kernel, dim3((unsigned)grid), dim3(kThreads), (size_t)SMEM_BYTES, st, mq, mk,
         mv, a);
  return cudaGetLastError();
}

}  // namespace sbp
