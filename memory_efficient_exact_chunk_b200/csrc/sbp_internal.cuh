// Internal declarations shared by the libsbp translation units (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include <mutex>
#include <utility>

namespace sbp {

// ---------------------------------------------------------------------------------------------
// side streams (streams.cu): kSideStreams streams and kSideEvents events per device; `mu` is
// held while one call queues work on them (keeps the event record / wait order of a call).
// Events 0..7: LM head, 8..13: decoder layer, 14..15: attention backward, 16..19: LM-head
// input staging from host memory.  Streams 0, 1: products next to the caller's stream,
// 2: the attention backward's key-tile kernel and the LM head's host-to-device staging.
// ---------------------------------------------------------------------------------------------
constexpr int kSideStreams = 3, kSideEvents = 20;
struct SidePool {
  std::recursive_mutex mu;
  cudaStream_t s[kSideStreams] = {};
  cudaEvent_t ev[kSideEvents] = {};
  bool ok = false;
};
SidePool* side_pool();

// ---------------------------------------------------------------------------------------------
// launch accounting (profile.cu): every kernel of the library goes through launch(), which
// counts it; the profiler (sbp_profile.h) reads the count and times GEMM launches with events.
// ---------------------------------------------------------------------------------------------
void prof_count_launch();
bool prof_enabled();
enum ProfKind : int { PROF_GEMM_TC = 0, PROF_GEMM_SIMT = 1, PROF_ATTN_FWD = 2, PROF_ATTN_BWD = 3,
                       PROF_KINDS = 4 };
// events bracketing one launch of `kind` on `st` (no-ops unless profiling)
void prof_mark_begin(int kind, cudaStream_t st);
void prof_mark_end(int kind, cudaStream_t st);

template <typename... KArgs, typename... Args>
inline void launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args&&... args) {
  prof_count_launch();
  kernel<<<grid, block, smem, st>>>(std::forward<Args>(args)...);
}

enum Dt : int { DT_F32 = 0, DT_BF16 = 1 };

// Message returned by sbp_last_error() on this thread (sbp_api.cu).
void set_last_error(const char* msg);
// Device status word of the workspace of the entry point running on this thread (sbp_api.cu);
// kernels with bounded waits raise their timeouts there.
int* status_word();

inline size_t dt_size(int dt) { return dt == DT_BF16 ? 2 : 4; }
__host__ __device__ __forceinline__ int64_t imin(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t imax(int64_t a, int64_t b) { return a > b ? a : b; }

// Device status word kept in the first bytes of every workspace.
enum : int { DEV_OK = 0, DEV_BAD_TARGET = 6, DEV_TIMEOUT = 5 };
constexpr size_t kStatusBytes = 256;

// ---------------------------------------------------------------------------------------------
// scalar load/store helpers
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float ld_f(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_f(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}
__device__ __forceinline__ float ld_dt(const void* p, int dt, int64_t i) {
  return dt == DT_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i])
                       : static_cast<const float*>(p)[i];
}
__device__ __forceinline__ void st_dt(void* p, int dt, int64_t i, float v) {
  if (dt == DT_BF16)
    static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    static_cast<float*>(p)[i] = v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------------------------------------------
// GEMM:  C[m, n] (op)= alpha * sum_k A(m, k) * B(k, n)  with element strides
//   A(m, k) = A[m * sam + k * sak],  B(k, n) = B[k * sbk + n * sbn],  C row-major (ldc).
// Epilogues:
//   EPI_STORE  : C = alpha * acc (+ bias[n])
//   EPI_ACC    : C += alpha * acc (+ bias[n])
//   EPI_LSE    : per row and column tile, partial max / sum-exp of acc over the tile's columns
//                (pmax/psum[m * pld + tile]); zy[m] = acc at column tgt[m] - col0 if in tile.
//   EPI_CEGRAD : C = wt[m] * (exp(acc - lse[m]) - [col0 + n == tgt[m]])  (cross-entropy
//                gradient of the logits), stored in the C dtype.
//   EPI_SWIGLU_BWD : acc = dM (gradient of m = silu(g) u); with g = aux[m, n] and
//                u = aux[m, aux_off + n] (aux row stride aux_ld, C dtype):
//                C[m, n] = dM u silu'(g),  C[m, aux_off + n] = dM silu(g).
//   EPI_SWIGLU_FWD : acc = u (the up projection); with g = aux[m, n] (bf16, row stride aux_ld):
//                C[m, n] = u (bf16) and C2[m, n] = silu(g) u (bf16, row stride ldc2).
//   EPI_ROPE   : the Q / K / V projection of a chunk (head_dim 128, bf16 C): y = acc (+ bias),
//                rotated per 128-column head by the rotate-half RoPE at position
//                r_s + m % r_Tc when cosb is set (cos / sin tables [T, 64]), written to row
//                (m / r_Tc) r_T + r_s + m % r_Tc of C when r_T > 0 (the K/V prefix of the
//                sequence), else to row m.
// dynM / dynK (nullable) give the true M / K on the device (<= the static M / K).
// crow (nullable) maps row m of the result to row crow[m] of C.
// ---------------------------------------------------------------------------------------------
enum Epi : int { EPI_STORE = 0, EPI_ACC = 1, EPI_LSE = 2, EPI_CEGRAD = 3, EPI_SWIGLU_BWD = 4,
                 EPI_ROPE = 5, EPI_SWIGLU_FWD = 6 };

struct GemmDesc {
  int64_t M = 0, N = 0, K = 0;
  const int* dynM = nullptr;
  const int* dynK = nullptr;
  int adt = DT_F32, bdt = DT_F32, cdt = DT_F32;
  const void* A = nullptr;
  int64_t sam = 0, sak = 0;
  const void* B = nullptr;
  int64_t sbk = 0, sbn = 0;
  void* C = nullptr;
  int64_t ldc = 0;
  const int* crow = nullptr;
  const void* bias = nullptr;
  int bias_dt = DT_F32;
  int epi = EPI_STORE;
  float alpha = 1.f;
  // cross-entropy epilogue parameters
  const float* lse = nullptr;
  const int* tgt = nullptr;
  const float* wt = nullptr;
  int64_t col0 = 0;
  float* pmax = nullptr;
  float* psum = nullptr;
  int64_t pld = 0;
  float* zy = nullptr;
  // SwiGLU-backward / -forward epilogue operand, and the forward's second output
  const void* aux = nullptr;
  int64_t aux_ld = 0, aux_off = 0;
  void* C2 = nullptr;
  int64_t ldc2 = 0;
  // RoPE epilogue: cos / sin tables (nullable: no rotation) and the row map
  const float* cosb = nullptr;
  const float* sinb = nullptr;
  int64_t r_Tc = 0, r_s = 0, r_T = 0;
  // > 0: the accumulator is flushed into C after every kblk elements of K (a multiple of 64),
  // so C is a left-to-right fp32 sum of partial products over consecutive K blocks that
  // start at the GEMM's first K row.  Used on the reductions over tokens (weight gradients):
  // no accumulator sums more than kblk tokens, and a chunk whose length is a multiple of kblk
  // rounds exactly as the same tokens do inside a longer chunk.  Only with EPI_STORE / EPI_ACC.
  int64_t kblk = 0;
  // device status word raised on a bounded-wait timeout (nullable)
  int* err = nullptr;
  // 0 = pick automatically, 1 = CUDA cores only, 2 = tensor cores (either kernel),
  // 3 = tensor cores, single-CTA kernel, 4 = tensor cores, CTA-pair kernel
  int path = 0;
  // Test hook of the bounded waits (set only by sbp_debug_gemm_stall_bf16): > 0 makes the
  // single-CTA kernel's producer issue no copy at all and bounds every wait by this many ns,
  // so the MMA issuer's first operand wait runs out with no copy or MMA in flight and the
  // kernel takes its timeout exit (status word raised, TMEM freed).
  int64_t stall_wait_ns = 0;
};

// Number of column tiles the EPI_LSE epilogue writes per row (its partial buffers' width).
int64_t gemm_lse_tiles(int64_t N);

// Longest run of tokens one tensor-core accumulator sums before its partial sum is added
// into the fp32 result in a plain fp32 add: kTokenBlock for the weight-gradient products
// (GemmDesc::kblk), kKvTokenBlock for the attention dK/dV sums over queries (which add all
// query heads of a KV group, so their accumulators see four to eight times more terms per
// token).  The accumulator's own rounding error grows with the number of terms it has added;
// these blocks bound it, and a chunk whose length is a multiple of the block adds the same
// partial sums as a longer chunk.
constexpr int64_t kTokenBlock = 4096;
constexpr int64_t kKvTokenBlock = 2048;

cudaError_t gemm(const GemmDesc& g, cudaStream_t st);
bool gemm_tc_supported(const GemmDesc& g);
// SMs of the device current at the first call (cached)
int sm_count();

// ---------------------------------------------------------------------------------------------
// element-wise / row kernels (elementwise.cu)
// ---------------------------------------------------------------------------------------------
// y = rmsnorm(x) * g ; rstd (nullable).  x dtype xdt, g/y dtype ydt.
cudaError_t rmsnorm_fwd(int64_t rows, int64_t cols, int xdt, const void* x, int gdt,
                        const void* g, int ydt, void* y, float* rstd, float eps,
                        cudaStream_t st);
// out = (base ? base : 0) + (accumulate ? out : 0) + rmsnorm_bwd(dy); dg += (deterministic).
// partial: workspace of rmsnorm_bwd_partial_floats(cols) floats.
size_t rmsnorm_bwd_partial_floats(int64_t cols);
cudaError_t rmsnorm_bwd(int64_t rows, int64_t cols, int xdt, const void* x, int gdt,
                        const void* g, const float* rstd, const float* dy, const float* base,
                        float* out, int accumulate, float* dg, float* partial, cudaStream_t st);
// cos/sin tables [T, hd/2] fp32 from fp64 angles pos * theta^(-2j/hd).
cudaError_t rope_table(int64_t T, int64_t hd, double theta, float* cosb, float* sinb,
                       cudaStream_t st);
// QKV post-processing of one chunk: qkv [R, dq + 2 dkv] fp32 (R = B * Tc rows, row r is token
// s + r % Tc of sequence r / Tc) -> q [R, dq] (RoPE'd, dt), K/V prefix [B, T, dkv] (dt).
// `part` restricts it to the query heads (QKV_Q) or to the key/value heads (QKV_KV); columns of
// qkv outside that part are not read.
enum { QKV_ALL = 0, QKV_Q = 1, QKV_KV = 2 };
cudaError_t qkv_post(int64_t R, int64_t Tc, int64_t s, int64_t T, int64_t H, int64_t Hkv,
                     int64_t hd, const float* qkv, int dt, void* q, void* Kp, void* Vp,
                     const float* cosb, const float* sinb, cudaStream_t st,
                     int part = QKV_ALL);
// In-place inverse RoPE on x [R, heads, hd] fp32 with position(r) = s + r % Tc.
cudaError_t rope_inv_f32(int64_t R, int64_t Tc, int64_t s, int64_t heads, int64_t hd, float* x,
                         const float* cosb, const float* sinb, cudaStream_t st);
// dK prefix rows of chunk [s, s + Tc) for all sequences -> dst [B * Tc, dkv] fp32 with RoPE^-1.
cudaError_t gather_rope_inv(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t heads,
                            int64_t hd, const float* src, float* dst, const float* cosb,
                            const float* sinb, cudaStream_t st);
// m = silu(g) * u from gu [R, 2f] (g = cols [0, f), u = [f, 2f)), dtype dt.
cudaError_t swiglu_fwd(int64_t R, int64_t f, int dt, const void* gu, void* m, cudaStream_t st);
// dgu [R, 2f] (dt) from dm [R, f] fp32 and gu.
cudaError_t swiglu_bwd(int64_t R, int64_t f, int dt, const void* gu, const float* dm, void* dgu,
                       cudaStream_t st);
// Row gather/scatter between [B, T, cols] and a chunk buffer [B * Tc, cols].
cudaError_t gather_chunk(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols, int dt,
                         const void* src, void* dst, cudaStream_t st);
cudaError_t scatter_chunk_f32(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols,
                              const float* src, float* dst, int accumulate, cudaStream_t st);
cudaError_t scatter_chunk(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols, int dt,
                          const void* src, void* dst, cudaStream_t st);
// dst[c] += sum_r src[r, c] (deterministic; partial of colsum_partial_floats(cols) floats).
size_t colsum_partial_floats(int64_t cols);
cudaError_t colsum_acc(int64_t rows, int64_t cols, const float* src, float* dst, float* partial,
                       cudaStream_t st);
// y = x + z (dt out) with x dt, z fp32: used for residual outputs.
cudaError_t add_residual(int64_t n, int xdt, const void* x, const float* z, int ydt, void* y,
                         cudaStream_t st);
cudaError_t copy_cast(int64_t n, int sdt, const void* src, int ddt, void* dst, cudaStream_t st);
// hi = bf16(x), lo = bf16(x - hi)
cudaError_t split_bf16(int64_t n, const float* x, void* hi, void* lo, cudaStream_t st);
// The two steps above fused for the chunk's rows of a [B, T, ...] fp32 prefix: hi / lo rows r
// of the inverse-rotated (gather_rope_inv_split) or plain (gather_split_bf16) row
// (r / Tc) T + s + r % Tc; both need gather_split_ok (head_dim and cols multiples of 8,
// 16-byte aligned buffers).
bool gather_split_ok(int64_t hd, int64_t cols, const void* src, const void* hi, const void* lo,
                     const float* cosb, const float* sinb);
cudaError_t gather_rope_inv_split(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t heads,
                                  int64_t hd, const float* src, void* hi, void* lo,
                                  const float* cosb, const float* sinb, cudaStream_t st);
cudaError_t gather_split_bf16(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t cols,
                              const float* src, void* hi, void* lo, cudaStream_t st);

// LM head helpers (lmhead.cu)
// Stable compaction of chunk rows [s, e) with w != 0 (and a valid target) into idx[0..n),
// count[0] = n; bad targets with w != 0 raise the device status.
cudaError_t ce_compact(int64_t s, int64_t e, int64_t V, const int* tgt, const float* w,
                       int* idx, int* count, int* status, cudaStream_t st);
// hc[r] = h[idx[r]] (r < n), rows [n, Rmax) = 0; wc, yc likewise (0 / -1); zy = 0, lse = 0.
cudaError_t ce_gather(int64_t Rmax, int64_t d, int dt, const void* h, const int* idx,
                      const int* count, const int* tgt, const float* w, void* hc, int* yc,
                      float* wc, float* zy, float* lse, cudaStream_t st);
// lse[r] from partials; loss (= if first else +=) sum_r wc[r] (lse[r] - zy[r]).
cudaError_t ce_finish(int64_t Rmax, int64_t tiles, const float* pmax, const float* psum,
                      int64_t pld, const int* count, const float* wc, const float* zy,
                      float* lse, float* row_loss, float* loss, int first, cudaStream_t st);
// out rows idx[r] (r < n) of d_hidden chunk: zero rows [s, e) of dh first.
cudaError_t zero_rows(int64_t s, int64_t e, int64_t d, float* dh, cudaStream_t st);
// token_ce[s, e) = 0, then token_ce[idx[r]] = lse[r] - zy[r] for the chunk's r < *count
cudaError_t ce_token_scatter(int64_t s, int64_t e, int64_t Rmax, const int* idx, const int* count,
                             const float* lse, const float* zy, float* token_ce, cudaStream_t st);
// DPO: sequence log-probabilities, per-pair loss terms, the loss and the per-token weights
cudaError_t dpo_weights(int64_t P, int64_t T, const float* token_ce, const float* mask,
                        const float* ref_logp, float beta, float* seq_logp, float* terms,
                        float* loss, float* weights, cudaStream_t st);

// attention: tensor-core forward (attn_tc.cu, head_dim 128, bf16) and CUDA-core kernels
// (attention_simt.cu, any even head_dim <= 256, fp32 or bf16).  attn_fwd/attn_bwd dispatch;
// path: 0 = automatic, 1 = CUDA cores, 2 = tensor cores.
bool attn_tc_supported(int64_t hd, int dt, const void* q, const void* Kp, const void* Vp,
                       const void* o);
// Scratch of the tensor-core forward's key-range split: part [B*Tc, H, 128] fp32, ml
// [B*Tc, H, 2] fp32, flags attn_fwd_split_flags() ints (zeroed by the launch).  Null pointers:
// no split (then results differ in rounding from calls that split, so every caller of a
// sequence passes them).
struct AttnFwdSplit {
  float* part = nullptr;
  float* ml = nullptr;
  int* flags = nullptr;
};
size_t attn_fwd_split_flags(int64_t B, int64_t Tc, int64_t H);
cudaError_t attn_fwd_tc(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                        const void* q, const void* Kp, const void* Vp, void* o, float* lse,
                        const AttnFwdSplit& sc, int* err, cudaStream_t st);
// Forward for chunk queries q [B*Tc, H, hd] at positions s.. over prefix keys [0, s + Tc).
cudaError_t attn_fwd(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                     int64_t hd, int dt, const void* q, const void* Kp, const void* Vp, void* o,
                     float* lse, const AttnFwdSplit& sc, cudaStream_t st, int path = 0);
// Backward: dq [B*Tc, H, hd] fp32 (overwritten); dKp/dVp [B, T, Hkv, hd] fp32 (+= rows < s+Tc);
// delta: scratch of attn_bwd_scratch_floats() floats.
cudaError_t attn_bwd(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                     int64_t hd, int dt, const void* q, const void* Kp, const void* Vp,
                     const void* o, const void* dO, const float* lse, float* delta, float* dq,
                     float* dKp, float* dVp, cudaStream_t st, int path = 0);
bool attn_bwd_tc_supported(int64_t hd, int dt, const void* q, const void* Kp, const void* Vp,
                           const void* o, const void* dO, const float* dq);
cudaError_t attn_bwd_tc(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H, int64_t Hkv,
                        const void* q, const void* Kp, const void* Vp, const void* o,
                        const void* dO, const float* lse, float* stats, float* dq, float* dKp,
                        float* dVp, int* err, cudaStream_t st);
// scratch floats of the tensor-core backward's per-query statistics
size_t attn_bwd_tc_stats_floats(int64_t B, int64_t Tc, int64_t H);
// scratch floats attn_bwd needs in its `delta` argument (either path)
inline size_t attn_bwd_scratch_floats(int64_t B, int64_t Tc, int64_t H) {
  const size_t a = (size_t)B * Tc * H, b = attn_bwd_tc_stats_floats(B, Tc, H);
  return a > b ? a : b;
}

// embedding (elementwise.cu)
cudaError_t embed_fwd(int64_t rows, int64_t cols, int64_t vocab, int dt, const int* ids,
                      const void* table, void* y, cudaStream_t st);
cudaError_t embed_bwd(int64_t rows, int64_t cols, int64_t vocab, const int* ids, const float* dy,
                      float* dtable, int* ws, cudaStream_t st);
size_t embed_bwd_ws_ints(int64_t rows, int64_t vocab);

}  // namespace sbp
