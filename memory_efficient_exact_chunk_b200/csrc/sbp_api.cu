// C ABI of libsbp (declared in include/sbp.h): argument checks, workspace carving and the
// host-side chunk loops that queue the kernels on the caller's stream.
//
// Sources: "StreamBP: Memory-Efficient Backpropagation" (skill page), sections Core Concept,
// Architecture Overview and Implementation; "StreamBP: Memory-Efficient Exact Backpropagation
// for Long Sequence Training of LLMs" (paper page), Abstract.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <string>

#include "sbp.h"
#include "sbp_debug.h"
#include "sbp_dpo.h"
#include "sbp_internal.cuh"

using namespace sbp;

namespace {

thread_local std::string g_err;
// status word of the workspace of the entry point running on this thread (GEMMs raise their
// bounded-wait timeouts there)
thread_local int* tl_status = nullptr;

sbp_status fail(sbp_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

#define SBP_CK(expr)                                                                 \
  do {                                                                               \
    cudaError_t e_ = (expr);                                                         \
    if (e_ != cudaSuccess)                                                           \
      return fail(SBP_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));     \
  } while (0)

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Bump allocator over the caller's workspace (dry run when base == nullptr).
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
  void* take_bytes(size_t n) { return take<char>(n); }
};

// ------------------------------------------------------------------------ chunk bounds
inline int64_t chunk_size(int64_t T, int D) { return T / D; }
inline void chunk_range(int64_t T, int D, int i, int64_t& s, int64_t& e) {
  const int64_t c = chunk_size(T, D);
  s = (int64_t)i * c;
  e = (i < D - 1) ? (int64_t)(i + 1) * c : T;
}
inline int64_t chunk_max(int64_t T, int D) { return T - (int64_t)(D - 1) * chunk_size(T, D); }

// ------------------------------------------------------------------------ LM head plan
constexpr int64_t kVocabBlock = 16384;

struct CePlan {
  int* status;
  int* idx;
  int* count;
  void* hc;
  int* yc;
  float *wc, *zy, *lse, *row_loss, *pmax, *psum;
  float* loss_tmp;   // loss accumulator when the caller passes none (forward entry)
  void* G[2];   // double-buffered logit-gradient block
  int64_t Rmax, tiles, Vb;
};

void ce_carve(Carver& c, int64_t N, int64_t d, int64_t V, int D, int dt, CePlan& p) {
  p.status = static_cast<int*>(c.take_bytes(kStatusBytes));
  p.Rmax = chunk_max(N, D);
  p.tiles = gemm_lse_tiles(V);
  p.Vb = V < kVocabBlock ? V : kVocabBlock;
  p.idx = c.take<int>(p.Rmax);
  p.count = c.take<int>(64);
  p.hc = c.take_bytes((size_t)p.Rmax * d * dt_size(dt));
  p.yc = c.take<int>(p.Rmax);
  p.wc = c.take<float>(p.Rmax);
  p.zy = c.take<float>(p.Rmax);
  p.lse = c.take<float>(p.Rmax);
  p.row_loss = c.take<float>(p.Rmax);
  p.pmax = c.take<float>((size_t)p.Rmax * p.tiles);
  p.psum = c.take<float>((size_t)p.Rmax * p.tiles);
  p.loss_tmp = c.take<float>(64);
  p.G[0] = c.take_bytes((size_t)p.Rmax * p.Vb * dt_size(dt));
  p.G[1] = c.take_bytes((size_t)p.Rmax * p.Vb * dt_size(dt));
}

// ------------------------------------------------------------------------ layer plan
struct LayerPlan {
  int* status;
  float *cosb, *sinb;
  void *Kp, *Vp;
  float *dKp, *dVp;
  void *xg, *n1, *q, *o, *n2, *gu, *m, *dgu, *dO;
  float *dyg, *rstd1, *qkv, *alse, *hbuf, *rstd2, *dn2, *dh, *delta, *dq, *dn1, *dxg;
  float *dkpre, *dvg, *rpart, *cpart;
  int* aflags;   // the attention forward's split flags (its partials use dq and delta)
  // bf16 operand copies of fp32 gradients (bf16 path only)
  void *dyg16, *dh16, *dq16, *khi, *klo, *vhi, *vlo;
  int64_t R;
};

// The Q / K / V projections get their bias, the rotate-half RoPE, the cast to bf16 and the
// append to the K/V prefix in the tensor-core GEMM's epilogue (no fp32 staging of the
// projections) on the bf16 path with head_dim 128.
bool qkv_fused(const sbp_layer_cfg& L) {
  return L.dtype == SBP_BF16 && L.head_dim == 128 && L.d_model % 8 == 0;
}

void layer_carve(Carver& c, const sbp_layer_cfg& L, LayerPlan& p) {
  const int dt = L.dtype;
  const size_t es = dt_size(dt);
  const int64_t B = L.batch, T = L.seq_len, d = L.d_model, f = L.ffn;
  const int64_t dq = L.n_heads * L.head_dim, dkv = L.n_kv_heads * L.head_dim;
  const int64_t R = B * chunk_max(T, L.num_chunks);
  p.R = R;
  p.status = static_cast<int*>(c.take_bytes(kStatusBytes));
  p.cosb = c.take<float>((size_t)T * (L.head_dim / 2));
  p.sinb = c.take<float>((size_t)T * (L.head_dim / 2));
  p.Kp = c.take_bytes((size_t)B * T * dkv * es);
  p.Vp = c.take_bytes((size_t)B * T * dkv * es);
  p.dKp = c.take<float>((size_t)B * T * dkv);
  p.dVp = c.take<float>((size_t)B * T * dkv);
  p.xg = c.take_bytes((size_t)R * d * es);
  p.dyg = c.take<float>((size_t)R * d);
  p.n1 = c.take_bytes((size_t)R * d * es);
  p.rstd1 = c.take<float>(R);
  // fp32 staging of the Q/K/V projections: only where RoPE is not done in the GEMM epilogue
  p.qkv = c.take<float>(qkv_fused(L) ? 0 : (size_t)R * (dq + 2 * dkv));
  p.q = c.take_bytes((size_t)R * dq * es);
  p.o = c.take_bytes((size_t)R * dq * es);
  p.alse = c.take<float>((size_t)R * L.n_heads);
  p.hbuf = c.take<float>((size_t)R * d);
  p.n2 = c.take_bytes((size_t)R * d * es);
  p.rstd2 = c.take<float>(R);
  p.gu = c.take_bytes((size_t)R * 2 * f * es);
  p.m = c.take_bytes((size_t)R * f * es);
  p.dgu = c.take_bytes((size_t)R * 2 * f * es);
  p.dn2 = c.take<float>((size_t)R * d);
  p.dh = c.take<float>((size_t)R * d);
  p.dO = c.take_bytes((size_t)R * dq * es);
  p.delta = c.take<float>(attn_bwd_scratch_floats(B, chunk_max(T, L.num_chunks), L.n_heads));
  p.dq = c.take<float>((size_t)R * dq);
  p.dn1 = c.take<float>((size_t)R * d);
  p.dxg = c.take<float>((size_t)R * d);
  p.dkpre = c.take<float>((size_t)R * dkv);
  p.dvg = c.take<float>((size_t)R * dkv);
  p.rpart = c.take<float>(rmsnorm_bwd_partial_floats(d));
  p.aflags = c.take<int>(attn_fwd_split_flags(B, chunk_max(T, L.num_chunks), L.n_heads));
  int64_t wmax = dq > dkv ? dq : dkv;
  p.cpart = c.take<float>(colsum_partial_floats(wmax));
  p.dyg16 = p.dh16 = p.dq16 = p.khi = p.klo = p.vhi = p.vlo = nullptr;
  if (dt == DT_BF16) {
    p.dyg16 = c.take_bytes((size_t)R * d * 2);
    p.dh16 = c.take_bytes((size_t)R * d * 2);
    p.dq16 = c.take_bytes((size_t)R * dq * 2);
    p.khi = c.take_bytes((size_t)R * dkv * 2);
    p.klo = c.take_bytes((size_t)R * dkv * 2);
    p.vhi = c.take_bytes((size_t)R * dkv * 2);
    p.vlo = c.take_bytes((size_t)R * dkv * 2);
  }
}

// GEMM descriptor helpers.  Matrices are row-major with the given leading dimension.
//   "N" operand (no transpose): A(m,k) = A[m*ld + k]   /  B(k,n) = B[k*ld + n]
//   "T" operand (transposed)  : A(m,k) = A[k*ld + m]   /  B(k,n) = B[n*ld + k]
GemmDesc mk_gemm(int64_t M, int64_t N, int64_t K, int adt, const void* A, bool a_t, int64_t lda,
                 int bdt, const void* B, bool b_t, int64_t ldb, int cdt, void* C, int64_t ldc,
                 int epi) {
  GemmDesc g;
  g.M = M; g.N = N; g.K = K;
  g.adt = adt; g.A = A;
  if (!a_t) { g.sam = lda; g.sak = 1; } else { g.sam = 1; g.sak = lda; }
  g.bdt = bdt; g.B = B;
  if (!b_t) { g.sbk = ldb; g.sbn = 1; } else { g.sbk = 1; g.sbn = ldb; }
  g.cdt = cdt; g.C = C; g.ldc = ldc;
  g.epi = epi;
  g.err = tl_status;
  return g;
}

// A product that sums over tokens (a weight gradient): K blocks of kTokenBlock rows.
GemmDesc over_tokens(GemmDesc g) {
  g.kblk = kTokenBlock;
  return g;
}

sbp_status check_layer_cfg(const sbp_layer_cfg* L) {
  if (!L) return fail(SBP_ERR_INVALID_ARG, "cfg is NULL");
  if (L->batch <= 0 || L->seq_len <= 0 || L->d_model <= 0 || L->n_heads <= 0 ||
      L->n_kv_heads <= 0 || L->head_dim <= 0 || L->ffn <= 0)
    return fail(SBP_ERR_INVALID_ARG, "all layer dimensions must be positive");
  if (L->num_chunks < 1 || (int64_t)L->num_chunks > L->seq_len)
    return fail(SBP_ERR_INVALID_ARG, "need 1 <= num_chunks <= seq_len (got %d, T=%lld)",
                L->num_chunks, (long long)L->seq_len);
  if (L->n_heads % L->n_kv_heads != 0)
    return fail(SBP_ERR_INVALID_ARG, "n_heads %% n_kv_heads != 0");
  if (L->dtype != SBP_F32 && L->dtype != SBP_BF16)
    return fail(SBP_ERR_INVALID_ARG, "unknown dtype %d", L->dtype);
  if (L->head_dim % 2 != 0 || L->head_dim > 256)
    return fail(SBP_ERR_UNSUPPORTED, "head_dim must be even and <= 256");
  if (!(L->rms_eps >= 0.f)) return fail(SBP_ERR_INVALID_ARG, "rms_eps must be >= 0");
  if (!(L->rope_theta > 0.0)) return fail(SBP_ERR_INVALID_ARG, "rope_theta must be > 0");
  if (L->dtype == SBP_BF16) {
    const int64_t dq = L->n_heads * L->head_dim, dkv = L->n_kv_heads * L->head_dim;
    if (L->d_model % 8 || dq % 8 || dkv % 8 || L->ffn % 8)
      return fail(SBP_ERR_UNSUPPORTED, "bf16 needs d_model, heads*head_dim, ffn % 8 == 0");
  }
  return SBP_OK;
}

sbp_status check_weights(const sbp_layer_weights* w, bool* has_bias) {
  if (!w) return fail(SBP_ERR_INVALID_ARG, "weights is NULL");
  const void* req[] = {w->ln1_g, w->wq, w->wk, w->wv, w->wo, w->ln2_g, w->w_gate, w->w_up,
                       w->w_down};
  for (const void* p : req) {
    if (!p) return fail(SBP_ERR_INVALID_ARG, "a required weight pointer is NULL");
    if (!aligned16(p)) return fail(SBP_ERR_INVALID_ARG, "weight pointer not 16-byte aligned");
  }
  const int nb = (w->bq != nullptr) + (w->bk != nullptr) + (w->bv != nullptr);
  if (nb != 0 && nb != 3) return fail(SBP_ERR_INVALID_ARG, "bq/bk/bv must be all set or all NULL");
  *has_bias = nb == 3;
  return SBP_OK;
}

// Fused Q / K / V projections of a chunk (qkv_fused): part QKV_Q, QKV_KV or QKV_ALL.
sbp_status qkv_project(const sbp_layer_cfg& L, const sbp_layer_weights& w, const LayerPlan& p,
                       int64_t s, int64_t Tc, int part, cudaStream_t st) {
  const int dt = L.dtype;
  const int64_t B = L.batch, T = L.seq_len, d = L.d_model;
  const int64_t dq = L.n_heads * L.head_dim, dkv = L.n_kv_heads * L.head_dim;
  const int64_t R = B * Tc;
  (void)B;
  auto proj = [&](int64_t N, const void* W, const void* bias, void* out, int64_t rT,
                  bool rope) -> sbp_status {
    GemmDesc g = mk_gemm(R, N, d, dt, p.n1, false, d, dt, W, true, d, DT_BF16, out, N, EPI_ROPE);
    g.bias = bias; g.bias_dt = dt;
    g.cosb = rope ? p.cosb : nullptr;
    g.sinb = rope ? p.sinb : nullptr;
    g.r_Tc = Tc; g.r_s = s; g.r_T = rT;
    SBP_CK(gemm(g, st));
    return SBP_OK;
  };
  sbp_status r = SBP_OK;
  if (part != QKV_KV && (r = proj(dq, w.wq, w.bq, p.q, 0, true)) != SBP_OK) return r;
  if (part != QKV_Q) {
    if ((r = proj(dkv, w.wk, w.bk, p.Kp, T, true)) != SBP_OK) return r;
    if ((r = proj(dkv, w.wv, w.bv, p.Vp, T, false)) != SBP_OK) return r;
  }
  return SBP_OK;
}

// RMSNorm-1 and the K/V projections of one chunk: fills n1, rstd1 and the chunk's rows of the
// K/V prefix.  xc is the chunk's input rows [B * Tc, d] (contiguous).
sbp_status layer_chunk_kv(const sbp_layer_cfg& L, const sbp_layer_weights& w, const LayerPlan& p,
                          const void* xc, int64_t s, int64_t Tc, cudaStream_t st) {
  const int dt = L.dtype;
  const int64_t B = L.batch, T = L.seq_len, d = L.d_model;
  const int64_t H = L.n_heads, Hkv = L.n_kv_heads, hd = L.head_dim;
  const int64_t dq = H * hd, dkv = Hkv * hd, W3 = dq + 2 * dkv;
  const int64_t R = B * Tc;
  SBP_CK(rmsnorm_fwd(R, d, dt, xc, dt, w.ln1_g, dt, p.n1, p.rstd1, L.rms_eps, st));
  if (qkv_fused(L)) return qkv_project(L, w, p, s, Tc, QKV_KV, st);
  GemmDesc g = mk_gemm(R, dkv, d, dt, p.n1, false, d, dt, w.wk, true, d, DT_F32, p.qkv + dq, W3,
                       EPI_STORE);
  g.bias = w.bk; g.bias_dt = dt;
  SBP_CK(gemm(g, st));
  g = mk_gemm(R, dkv, d, dt, p.n1, false, d, dt, w.wv, true, d, DT_F32, p.qkv + dq + dkv, W3,
              EPI_STORE);
  g.bias = w.bv; g.bias_dt = dt;
  SBP_CK(gemm(g, st));
  SBP_CK(qkv_post(R, Tc, s, T, H, Hkv, hd, p.qkv, dt, p.q, p.Kp, p.Vp, p.cosb, p.sinb, st,
                  QKV_KV));
  return SBP_OK;
}

// Forward recompute of one chunk: fills n1, rstd1, q, K/V prefix rows, o, alse, hbuf (= h),
// n2, rstd2, gu and m.  xc is the chunk's input rows [B * Tc, d] (contiguous).  With
// kv_ready the whole K/V prefix is already in place: only the query projection is computed.
sbp_status layer_chunk_forward(const sbp_layer_cfg& L, const sbp_layer_weights& w,
                               const LayerPlan& p, const void* xc, int64_t s, int64_t Tc,
                               cudaStream_t st, bool kv_ready = false) {
  const int dt = L.dtype;
  const int64_t B = L.batch, T = L.seq_len, d = L.d_model, f = L.ffn;
  const int64_t H = L.n_heads, Hkv = L.n_kv_heads, hd = L.head_dim;
  const int64_t dq = H * hd, dkv = Hkv * hd, W3 = dq + 2 * dkv;
  const int64_t R = B * Tc;
  SBP_CK(rmsnorm_fwd(R, d, dt, xc, dt, w.ln1_g, dt, p.n1, p.rstd1, L.rms_eps, st));
  if (qkv_fused(L)) {
    const sbp_status r = qkv_project(L, w, p, s, Tc, kv_ready ? QKV_Q : QKV_ALL, st);
    if (r != SBP_OK) return r;
  } else {
    GemmDesc g = mk_gemm(R, dq, d, dt, p.n1, false, d, dt, w.wq, true, d, DT_F32, p.qkv, W3,
                         EPI_STORE);
    g.bias = w.bq; g.bias_dt = dt;
    SBP_CK(gemm(g, st));
    if (kv_ready) {
      SBP_CK(qkv_post(R, Tc, s, T, H, Hkv, hd, p.qkv, dt, p.q, p.Kp, p.Vp, p.cosb, p.sinb, st,
                      QKV_Q));
    } else {
      g = mk_gemm(R, dkv, d, dt, p.n1, false, d, dt, w.wk, true, d, DT_F32, p.qkv + dq, W3,
                  EPI_STORE);
      g.bias = w.bk; g.bias_dt = dt;
      SBP_CK(gemm(g, st));
      g = mk_gemm(R, dkv, d, dt, p.n1, false, d, dt, w.wv, true, d, DT_F32, p.qkv + dq + dkv,
                  W3, EPI_STORE);
      g.bias = w.bv; g.bias_dt = dt;
      SBP_CK(gemm(g, st));
      SBP_CK(qkv_post(R, Tc, s, T, H, Hkv, hd, p.qkv, dt, p.q, p.Kp, p.Vp, p.cosb, p.sinb, st));
    }
  }
  // the forward's key-range split parks partials in dq and delta, which only the backward
  // of the same chunk fills, after this call
  AttnFwdSplit sc;
  sc.part = p.dq;
  sc.ml = p.delta;
  sc.flags = p.aflags;
  SBP_CK(attn_fwd(B, T, Tc, s, H, Hkv, hd, dt, p.q, p.Kp, p.Vp, p.o, p.alse, sc, st));
  SBP_CK(copy_cast(R * d, dt, xc, DT_F32, p.hbuf, st));
  SBP_CK(gemm(mk_gemm(R, d, dq, dt, p.o, false, dq, dt, w.wo, true, dq, DT_F32, p.hbuf, d,
                      EPI_ACC), st));
  SBP_CK(rmsnorm_fwd(R, d, DT_F32, p.hbuf, dt, w.ln2_g, dt, p.n2, p.rstd2, L.rms_eps, st));
  SBP_CK(gemm(mk_gemm(R, f, d, dt, p.n2, false, d, dt, w.w_gate, true, d, dt, p.gu, 2 * f,
                      EPI_STORE), st));
  // the up projection; on the tensor-core path its epilogue also forms m = silu(g) u
  GemmDesc gup = mk_gemm(R, f, d, dt, p.n2, false, d, dt, w.w_up, true, d, dt,
                         static_cast<char*>(p.gu) + f * dt_size(dt), 2 * f, EPI_SWIGLU_FWD);
  gup.aux = p.gu; gup.aux_ld = 2 * f;
  gup.C2 = p.m; gup.ldc2 = f;
  if (dt == DT_BF16 && gemm_tc_supported(gup)) {
    SBP_CK(gemm(gup, st));
  } else {
    gup.epi = EPI_STORE;
    SBP_CK(gemm(gup, st));
    SBP_CK(swiglu_fwd(R, f, dt, p.gu, p.m, st));
  }
  return SBP_OK;
}

sbp_status check_ws(void* ws, size_t have, size_t need) {
  if (!ws) return fail(SBP_ERR_INVALID_ARG, "workspace is NULL");
  if (((uintptr_t)ws & 255u) != 0) return fail(SBP_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (have < need)
    return fail(SBP_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", have, need);
  return SBP_OK;
}

}  // namespace

namespace sbp {
// Lets other translation units of the library report a message through sbp_last_error().
void set_last_error(const char* msg) { g_err = msg ? msg : ""; }
int* status_word() { return tl_status; }
}  // namespace sbp

namespace {

// Host-resident per-token inputs of the LM-head backward: each chunk's rows are copied into one
// of two staging blocks of the workspace on a side stream while the previous chunk computes.
struct HostIn {
  const char* h;          // [N, d] host
  const int32_t* y;       // [N] host
  const float* w;         // [N] host
  char* sh[2];            // staging blocks [Rmax, d]
  int32_t* sy[2];
  float* sw[2];
};

void host_carve(Carver& c, int64_t N, int64_t d, int D, int dt, HostIn& hin) {
  const int64_t Rmax = chunk_max(N, D);
  for (int b = 0; b < 2; ++b) {
    hin.sh[b] = static_cast<char*>(c.take_bytes((size_t)Rmax * d * dt_size(dt)));
    hin.sy[b] = c.take<int32_t>(Rmax);
    hin.sw[b] = c.take<float>(Rmax);
  }
}

sbp_status lmhead_check(int64_t N, int64_t d, int64_t V, int D, sbp_dtype dt,
                        std::initializer_list<const void*> ptrs) {
  if (N <= 0 || d <= 0 || V <= 0) return fail(SBP_ERR_INVALID_ARG, "sizes must be positive");
  if (D < 1 || (int64_t)D > N)
    return fail(SBP_ERR_INVALID_ARG, "need 1 <= num_chunks <= n_tokens");
  if (dt != SBP_F32 && dt != SBP_BF16) return fail(SBP_ERR_INVALID_ARG, "unknown dtype");
  if (dt == SBP_BF16 && d % 8 != 0) return fail(SBP_ERR_UNSUPPORTED, "bf16 needs hidden % 8 == 0");
  for (const void* q : ptrs) {
    if (!q) return fail(SBP_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned16(q)) return fail(SBP_ERR_INVALID_ARG, "a pointer is not 16-byte aligned");
  }
  return SBP_OK;
}

// Rows [s, e) of a chunk staged at `base` (row s at base[0]) addressed by their global row index.
template <typename T>
const T* as_global_rows(const void* base, int64_t s, int64_t row_bytes) {
  return reinterpret_cast<const T*>(reinterpret_cast<uintptr_t>(base) -
                                    (uintptr_t)(s * row_bytes));
}

sbp_status lmhead_backward_run(int64_t N, int64_t d, int64_t V, int D, sbp_dtype dt,
                               const void* hidden_states, const void* weight,
                               const int32_t* targets, const float* loss_weights,
                               float* loss_out, float* d_hidden, float* d_weight, CePlan& p,
                               const HostIn* hin, cudaStream_t st) {
  const int64_t es = dt_size(dt);
  SidePool* sp = side_pool();
  if (!sp) return fail(SBP_ERR_CUDA, "could not create the side streams");
  std::lock_guard<std::recursive_mutex> side_lock(sp->mu);
  // staging: ev[16 + b] = block b holds its chunk, ev[18 + b] = block b has been gathered
  auto stage = [&](int i) -> cudaError_t {
    int64_t s0, e0;
    chunk_range(N, D, i, s0, e0);
    const int b = i & 1;
    cudaError_t e = cudaSuccess;
    if (i >= 2) e = cudaStreamWaitEvent(sp->s[2], sp->ev[18 + b], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(hin->sh[b], hin->h + s0 * d * es, (size_t)(e0 - s0) * d * es,
                          cudaMemcpyHostToDevice, sp->s[2]);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(hin->sy[b], hin->y + s0, sizeof(int32_t) * (size_t)(e0 - s0),
                          cudaMemcpyHostToDevice, sp->s[2]);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(hin->sw[b], hin->w + s0, sizeof(float) * (size_t)(e0 - s0),
                          cudaMemcpyHostToDevice, sp->s[2]);
    if (e == cudaSuccess) e = cudaEventRecord(sp->ev[16 + b], sp->s[2]);
    return e;
  };
  if (hin) {
    SBP_CK(cudaEventRecord(sp->ev[7], st));        // the side stream starts after the caller
    SBP_CK(cudaStreamWaitEvent(sp->s[2], sp->ev[7], 0));
    SBP_CK(stage(0));
    if (D > 1) SBP_CK(stage(1));
  }
  for (int i = 0; i < D; ++i) {
    int64_t s, e;
    chunk_range(N, D, i, s, e);
    const int64_t Rc = e - s;
    const void* hid = hidden_states;
    const int32_t* tg = targets;
    const float* lw = loss_weights;
    if (hin) {
      const int b = i & 1;
      SBP_CK(cudaStreamWaitEvent(st, sp->ev[16 + b], 0));
      hid = as_global_rows<char>(hin->sh[b], s, d * es);
      tg = as_global_rows<int32_t>(hin->sy[b], s, sizeof(int32_t));
      lw = as_global_rows<float>(hin->sw[b], s, sizeof(float));
    }
    SBP_CK(ce_compact(s, e, V, tg, lw, p.idx, p.count, p.status, st));
    SBP_CK(ce_gather(Rc, d, dt, hid, p.idx, p.count, tg, lw, p.hc, p.yc, p.wc, p.zy, p.lse, st));
    if (hin) {
      // the chunk's rows now live in the compacted buffers: its staging block may be refilled
      SBP_CK(cudaEventRecord(sp->ev[18 + (i & 1)], st));
      if (i + 2 < D) SBP_CK(stage(i + 2));
    }
    SBP_CK(zero_rows(s, e, d, d_hidden, st));
    // pass 1: per-row log-sum-exp over the vocabulary (logits stay in GEMM tiles)
    GemmDesc g = mk_gemm(Rc, V, d, dt, p.hc, false, d, dt, weight, true, d, DT_F32, nullptr, 0,
                         EPI_LSE);
    g.dynM = p.count; g.tgt = p.yc; g.col0 = 0; g.pmax = p.pmax; g.psum = p.psum;
    g.pld = p.tiles; g.zy = p.zy;
    SBP_CK(gemm(g, st));
    SBP_CK(ce_finish(Rc, p.tiles, p.pmax, p.psum, p.tiles, p.count, p.wc, p.zy, p.lse,
                     p.row_loss, loss_out, i == 0, st));
    // pass 2, one vocabulary block at a time: G = w (softmax - onehot) on the caller's stream,
    // then dH += G W_b and dW_b += G^T H on the two side streams while the next block's G is
    // formed in the other buffer (dH stays in vocabulary order on its stream).
    SBP_CK(cudaEventRecord(sp->ev[0], st));
    SBP_CK(cudaStreamWaitEvent(sp->s[0], sp->ev[0], 0));
    SBP_CK(cudaStreamWaitEvent(sp->s[1], sp->ev[0], 0));
    int blk = 0;
    for (int64_t vb = 0; vb < V; vb += p.Vb, ++blk) {
      const int buf = blk & 1;
      const int64_t nb = (V - vb) < p.Vb ? (V - vb) : p.Vb;
      const char* Wb = static_cast<const char*>(weight) + vb * d * dt_size(dt);
      if (blk >= 2) {   // the products of block blk - 2 have read this buffer
        SBP_CK(cudaStreamWaitEvent(st, sp->ev[3 + buf], 0));
        SBP_CK(cudaStreamWaitEvent(st, sp->ev[5 + buf], 0));
      }
      GemmDesc gg = mk_gemm(Rc, nb, d, dt, p.hc, false, d, dt, Wb, true, d, dt, p.G[buf], nb,
                            EPI_CEGRAD);
      gg.dynM = p.count; gg.lse = p.lse; gg.tgt = p.yc; gg.wt = p.wc; gg.col0 = vb;
      SBP_CK(gemm(gg, st));
      SBP_CK(cudaEventRecord(sp->ev[1 + buf], st));
      SBP_CK(cudaStreamWaitEvent(sp->s[0], sp->ev[1 + buf], 0));
      GemmDesc gh = mk_gemm(Rc, d, nb, dt, p.G[buf], false, nb, dt, Wb, false, d, DT_F32,
                            d_hidden, d, vb == 0 ? EPI_STORE : EPI_ACC);
      gh.dynM = p.count; gh.crow = p.idx;
      SBP_CK(gemm(gh, sp->s[0]));
      SBP_CK(cudaEventRecord(sp->ev[3 + buf], sp->s[0]));
      SBP_CK(cudaStreamWaitEvent(sp->s[1], sp->ev[1 + buf], 0));
      GemmDesc gw = mk_gemm(nb, d, Rc, dt, p.G[buf], true, nb, dt, p.hc, false, d, DT_F32,
                            d_weight + vb * d, d, EPI_ACC);
      gw.dynK = p.count;
      gw.kblk = kTokenBlock;
      SBP_CK(gemm(gw, sp->s[1]));
      SBP_CK(cudaEventRecord(sp->ev[5 + buf], sp->s[1]));
    }
    // join: the next chunk reuses the compacted rows and the row map
    SBP_CK(cudaEventRecord(sp->ev[3], sp->s[0]));
    SBP_CK(cudaEventRecord(sp->ev[5], sp->s[1]));
    SBP_CK(cudaStreamWaitEvent(st, sp->ev[3], 0));
    SBP_CK(cudaStreamWaitEvent(st, sp->ev[5], 0));
  }
  return SBP_OK;
}

}  // namespace

extern "C" {

const char* sbp_last_error(void) { return g_err.c_str(); }

const char* sbp_version(void) { return "sbp 0.1 (sm_100a)"; }

sbp_status sbp_chunk_bounds(int64_t seq_len, int num_chunks, int64_t* bounds) {
  if (!bounds) return fail(SBP_ERR_INVALID_ARG, "bounds is NULL");
  if (num_chunks < 1 || seq_len < 1 || (int64_t)num_chunks > seq_len)
    return fail(SBP_ERR_INVALID_ARG, "need 1 <= num_chunks <= seq_len");
  for (int i = 0; i < num_chunks; ++i) {
    int64_t s, e;
    chunk_range(seq_len, num_chunks, i, s, e);
    bounds[i] = s;
    if (i == num_chunks - 1) bounds[num_chunks] = e;
  }
  return SBP_OK;
}

sbp_status sbp_get_device_status(void* workspace, void* stream) {
  if (!workspace) return fail(SBP_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h = 0;
  SBP_CK(cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, st));
  SBP_CK(cudaStreamSynchronize(st));
  SBP_CK(cudaMemsetAsync(workspace, 0, sizeof(int), st));
  if (h == DEV_OK) return SBP_OK;
  if (h == DEV_BAD_TARGET)
    return fail(SBP_ERR_BAD_TARGET, "a target outside [0, vocab) had a nonzero loss weight");
  if (h == DEV_TIMEOUT) return fail(SBP_ERR_DEVICE_TIMEOUT, "a device-side wait gave up");
  return fail(SBP_ERR_CUDA, "unknown device status %d", h);
}

// ------------------------------------------------------------------------------- LM head
size_t sbp_lmhead_ce_workspace_size(int64_t n_tokens, int64_t hidden, int64_t vocab,
                                    int num_chunks, sbp_dtype dt) {
  if (n_tokens <= 0 || hidden <= 0 || vocab <= 0 || num_chunks < 1 ||
      (int64_t)num_chunks > n_tokens)
    return 0;
  Carver c(nullptr);
  CePlan p;
  ce_carve(c, n_tokens, hidden, vocab, num_chunks, dt, p);
  return c.off;
}

sbp_status sbp_lmhead_ce_backward_stream(int64_t N, int64_t d, int64_t V, int D, sbp_dtype dt,
                                         const void* hidden_states, const void* weight,
                                         const int32_t* targets, const float* loss_weights,
                                         float* loss_out, float* d_hidden, float* d_weight,
                                         void* workspace, size_t workspace_bytes,
                                         void* stream) {
  if (sbp_status r = lmhead_check(N, d, V, D, dt, {hidden_states, weight, targets, loss_weights,
                                                   loss_out, d_hidden, d_weight}))
    return r;
  const size_t need = sbp_lmhead_ce_workspace_size(N, d, V, D, dt);
  if (sbp_status s = check_ws(workspace, workspace_bytes, need)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  CePlan p;
  ce_carve(c, N, d, V, D, dt, p);
  tl_status = p.status;
  SBP_CK(cudaMemsetAsync(p.status, 0, sizeof(int), st));
  return lmhead_backward_run(N, d, V, D, dt, hidden_states, weight, targets, loss_weights,
                             loss_out, d_hidden, d_weight, p, nullptr, st);
}

size_t sbp_lmhead_ce_workspace_size_host(int64_t N, int64_t d, int64_t V, int D, sbp_dtype dt) {
  if (sbp_lmhead_ce_workspace_size(N, d, V, D, dt) == 0) return 0;
  Carver c(nullptr);
  CePlan p;
  ce_carve(c, N, d, V, D, dt, p);
  HostIn hin;
  host_carve(c, N, d, D, dt, hin);
  return c.off;
}

sbp_status sbp_lmhead_ce_backward_stream_host(int64_t N, int64_t d, int64_t V, int D,
                                              sbp_dtype dt, const void* hidden_states_host,
                                              const void* weight, const int32_t* targets_host,
                                              const float* loss_weights_host, float* loss_out,
                                              float* d_hidden, float* d_weight, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  if (sbp_status r = lmhead_check(N, d, V, D, dt, {hidden_states_host, weight, targets_host,
                                                   loss_weights_host, loss_out, d_hidden,
                                                   d_weight}))
    return r;
  const size_t need = sbp_lmhead_ce_workspace_size_host(N, d, V, D, dt);
  if (sbp_status s = check_ws(workspace, workspace_bytes, need)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  CePlan p;
  ce_carve(c, N, d, V, D, dt, p);
  HostIn hin;
  host_carve(c, N, d, D, dt, hin);
  hin.h = static_cast<const char*>(hidden_states_host);
  hin.y = targets_host;
  hin.w = loss_weights_host;
  tl_status = p.status;
  SBP_CK(cudaMemsetAsync(p.status, 0, sizeof(int), st));
  return lmhead_backward_run(N, d, V, D, dt, nullptr, weight, nullptr, nullptr, loss_out,
                             d_hidden, d_weight, p, &hin, st);
}

sbp_status sbp_lmhead_ce_forward_stream(int64_t N, int64_t d, int64_t V, int D, sbp_dtype dt,
                                        const void* hidden_states, const void* weight,
                                        const int32_t* targets, const float* loss_weights,
                                        float* token_ce, float* loss_out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (N <= 0 || d <= 0 || V <= 0) return fail(SBP_ERR_INVALID_ARG, "sizes must be positive");
  if (D < 1 || (int64_t)D > N)
    return fail(SBP_ERR_INVALID_ARG, "need 1 <= num_chunks <= n_tokens");
  if (dt != SBP_F32 && dt != SBP_BF16) return fail(SBP_ERR_INVALID_ARG, "unknown dtype");
  if (dt == SBP_BF16 && d % 8 != 0) return fail(SBP_ERR_UNSUPPORTED, "bf16 needs hidden % 8 == 0");
  const void* ptrs[] = {hidden_states, weight, targets, loss_weights, token_ce};
  for (const void* q : ptrs) {
    if (!q) return fail(SBP_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned16(q)) return fail(SBP_ERR_INVALID_ARG, "a pointer is not 16-byte aligned");
  }
  const size_t need = sbp_lmhead_ce_workspace_size(N, d, V, D, dt);
  if (sbp_status s = check_ws(workspace, workspace_bytes, need)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  CePlan p;
  ce_carve(c, N, d, V, D, dt, p);
  tl_status = p.status;
  SBP_CK(cudaMemsetAsync(p.status, 0, sizeof(int), st));
  float* lo = loss_out ? loss_out : p.loss_tmp;
  for (int i = 0; i < D; ++i) {
    int64_t s, e;
    chunk_range(N, D, i, s, e);
    const int64_t Rc = e - s;
    SBP_CK(ce_compact(s, e, V, targets, loss_weights, p.idx, p.count, p.status, st));
    SBP_CK(ce_gather(Rc, d, dt, hidden_states, p.idx, p.count, targets, loss_weights, p.hc, p.yc,
                     p.wc, p.zy, p.lse, st));
    // per-row log-sum-exp over the vocabulary (logits stay in GEMM tiles), as in the backward
    GemmDesc g = mk_gemm(Rc, V, d, dt, p.hc, false, d, dt, weight, true, d, DT_F32, nullptr, 0,
                         EPI_LSE);
    g.dynM = p.count; g.tgt = p.yc; g.col0 = 0; g.pmax = p.pmax; g.psum = p.psum;
    g.pld = p.tiles; g.zy = p.zy;
    SBP_CK(gemm(g, st));
    SBP_CK(ce_finish(Rc, p.tiles, p.pmax, p.psum, p.tiles, p.count, p.wc, p.zy, p.lse,
                     p.row_loss, lo, i == 0, st));
    SBP_CK(ce_token_scatter(s, e, Rc, p.idx, p.count, p.lse, p.zy, token_ce, st));
  }
  return SBP_OK;
}

// ------------------------------------------------------------------------------- DPO
size_t sbp_dpo_workspace_size(int64_t P) {
  if (P < 1) return 0;
  Carver c(nullptr);
  c.take_bytes(kStatusBytes);
  c.take<float>(2 * P);     // sequence log-probabilities when the caller keeps none
  c.take<float>(P);         // per-pair loss terms
  return c.off;
}

sbp_status sbp_dpo_token_weights(int64_t P, int64_t T, const float* token_ce,
                                 const float* mask, const float* ref_logp, float beta,
                                 float* loss_out, float* seq_logp, float* weights,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (P < 1 || T < 1) return fail(SBP_ERR_INVALID_ARG, "n_pairs and seq_len must be positive");
  if (!(beta > 0.f)) return fail(SBP_ERR_INVALID_ARG, "beta must be positive");
  if (!token_ce || !mask || !ref_logp || !loss_out || !weights)
    return fail(SBP_ERR_INVALID_ARG, "a required pointer is NULL");
  if (sbp_status s = check_ws(workspace, workspace_bytes, sbp_dpo_workspace_size(P))) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  int* status = static_cast<int*>(c.take_bytes(kStatusBytes));
  float* lp_tmp = c.take<float>(2 * P);
  float* terms = c.take<float>(P);
  SBP_CK(cudaMemsetAsync(status, 0, sizeof(int), st));
  SBP_CK(dpo_weights(P, T, token_ce, mask, ref_logp, beta, seq_logp ? seq_logp : lp_tmp, terms,
                     loss_out, weights, st));
  return SBP_OK;
}

// ------------------------------------------------------------------------------- layer
size_t sbp_decoder_layer_workspace_size(const sbp_layer_cfg* cfg) {
  if (check_layer_cfg(cfg) != SBP_OK) return 0;
  Carver c(nullptr);
  LayerPlan p;
  layer_carve(c, *cfg, p);
  return c.off;
}

// The streamed layer backward in either chunk order.  Forward order (chunks 0 .. D-1) grows the
// K/V prefix chunk by chunk and backpropagates the K/V projections after the loop, once every
// later chunk has added its dK/dV.  Reverse order (D-1 .. 0) computes the whole K/V prefix
// first; when chunk i is reached every chunk that attends to its keys is done, so its K/V
// projection backward runs inside the same iteration, on the n1 rows already in place.
static sbp_status layer_backward_run(const sbp_layer_cfg* cfg, const sbp_layer_weights* w,
                                     const void* x, const float* dy, float* dx,
                                     const sbp_layer_grads* gr, void* workspace,
                                     size_t workspace_bytes, void* stream, bool reverse) {
  if (sbp_status s = check_layer_cfg(cfg)) return s;
  bool has_bias = false;
  if (sbp_status s = check_weights(w, &has_bias)) return s;
  if (!gr) return fail(SBP_ERR_INVALID_ARG, "grads is NULL");
  {
    float* req[] = {gr->ln1_g, gr->wq, gr->wk, gr->wv, gr->wo, gr->ln2_g, gr->w_gate, gr->w_up,
                    gr->w_down};
    for (float* q : req)
      if (!q || !aligned16(q)) return fail(SBP_ERR_INVALID_ARG, "grad pointer NULL or misaligned");
    const int nb = (gr->bq != nullptr) + (gr->bk != nullptr) + (gr->bv != nullptr);
    if ((has_bias && nb != 3) || (!has_bias && nb != 0))
      return fail(SBP_ERR_INVALID_ARG, "bias grads must be set exactly when biases are");
  }
  const void* io[] = {x, dy, dx};
  for (const void* q : io)
    if (!q || !aligned16(q)) return fail(SBP_ERR_INVALID_ARG, "x/dy/dx NULL or misaligned");
  const sbp_layer_cfg& L = *cfg;
  const size_t need = sbp_decoder_layer_workspace_size(cfg);
  if (sbp_status s = check_ws(workspace, workspace_bytes, need)) return s;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  LayerPlan p;
  layer_carve(c, L, p);
  const int dt = L.dtype;
  const size_t es = dt_size(dt);
  const int64_t B = L.batch, T = L.seq_len, d = L.d_model, f = L.ffn;
  const int64_t H = L.n_heads, Hkv = L.n_kv_heads, hd = L.head_dim;
  const int64_t dq = H * hd, dkv = Hkv * hd;
  const int D = L.num_chunks;

  tl_status = p.status;
  SBP_CK(cudaMemsetAsync(p.status, 0, sizeof(int), st));
  SBP_CK(rope_table(T, hd, L.rope_theta, p.cosb, p.sinb, st));
  SBP_CK(cudaMemsetAsync(p.dKp, 0, sizeof(float) * (size_t)B * T * dkv, st));
  SBP_CK(cudaMemsetAsync(p.dVp, 0, sizeof(float) * (size_t)B * T * dkv, st));
  if (!reverse) {
    // key/value rows past the current prefix are read (and masked) by the last key tile of a
    // query tile: give them finite contents
    SBP_CK(cudaMemsetAsync(p.Kp, 0, es * (size_t)B * T * dkv, st));
    SBP_CK(cudaMemsetAsync(p.Vp, 0, es * (size_t)B * T * dkv, st));
  }

  // Weight-gradient products run on two side streams next to the chain of data gradients on
  // the caller's stream; each chunk ends with a join (its buffers are reused by the next one).
  SidePool* sp = side_pool();
  if (!sp) return fail(SBP_ERR_CUDA, "could not create the side streams");
  std::lock_guard<std::recursive_mutex> side_lock(sp->mu);
  auto fork_to = [&](int k, int ev) -> cudaError_t {
    cudaError_t e = cudaEventRecord(sp->ev[ev], st);
    return e == cudaSuccess ? cudaStreamWaitEvent(sp->s[k], sp->ev[ev], 0) : e;
  };
  auto join_all = [&]() -> cudaError_t {
    cudaError_t e = cudaEventRecord(sp->ev[12], sp->s[0]);
    if (e == cudaSuccess) e = cudaEventRecord(sp->ev[13], sp->s[1]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, sp->ev[12], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, sp->ev[13], 0);
    return e;
  };
  cudaStream_t s0 = sp->s[0], s1 = sp->s[1];

  // K/V projection backward of the chunk [s, s + Tc) once its dK/dV rows are final (n1 holds
  // that chunk's RMSNorm-1 output): dW_k, dW_v (and the bias sums) accumulate, and
  // dK_pre W_k + dV W_v is stored into dn1 or, with acc, added to it.
  auto kv_backward = [&](int64_t s, int64_t Tc, bool acc) -> sbp_status {
    const int64_t R = B * Tc;
    // without biases the fp32 chunk rows of dK / dV are not needed: the bf16 path reads the
    // prefix rows, rotates dK and writes the hi + lo operands in one pass each
    const bool fused = dt == DT_BF16 && !has_bias &&
                       gather_split_ok(hd, dkv, p.dKp, p.khi, p.klo, p.cosb, p.sinb) &&
                       gather_split_ok(hd, dkv, p.dVp, p.vhi, p.vlo, p.cosb, p.sinb);
    if (fused) {
      SBP_CK(gather_rope_inv_split(B, T, Tc, s, Hkv, hd, p.dKp, p.khi, p.klo, p.cosb, p.sinb, st));
      SBP_CK(gather_split_bf16(B, T, Tc, s, dkv, p.dVp, p.vhi, p.vlo, st));
    } else {
      SBP_CK(gather_rope_inv(B, T, Tc, s, Hkv, hd, p.dKp, p.dkpre, p.cosb, p.sinb, st));
      SBP_CK(gather_chunk(B, T, Tc, s, dkv, DT_F32, p.dVp, p.dvg, st));
    }
    if (dt == DT_BF16) {
      // dK/dV are fp32 sums over chunks; their bf16 operands carry a hi + lo pair so that the
      // products do not depend on where the fp32 sum happened to round
      if (!fused) {
        SBP_CK(split_bf16(R * dkv, p.dkpre, p.khi, p.klo, st));
        SBP_CK(split_bf16(R * dkv, p.dvg, p.vhi, p.vlo, st));
      }
      const void* parts[4] = {p.khi, p.klo, p.vhi, p.vlo};
      const void* wts[4] = {w->wk, w->wk, w->wv, w->wv};
      float* grs[4] = {gr->wk, gr->wk, gr->wv, gr->wv};
      SBP_CK(fork_to(0, 8));
      for (int k = 0; k < 4; ++k)
        SBP_CK(gemm(over_tokens(mk_gemm(dkv, d, R, DT_BF16, parts[k], true, dkv, dt, p.n1, false,
                                        d, DT_F32, grs[k], d, EPI_ACC)), s0));
      for (int k = 0; k < 4; ++k)
        SBP_CK(gemm(mk_gemm(R, d, dkv, DT_BF16, parts[k], false, dkv, dt, wts[k], false, d,
                            DT_F32, p.dn1, d, k == 0 && !acc ? EPI_STORE : EPI_ACC), st));
    } else {
      SBP_CK(gemm(mk_gemm(R, d, dkv, DT_F32, p.dkpre, false, dkv, dt, w->wk, false, d, DT_F32,
                          p.dn1, d, acc ? EPI_ACC : EPI_STORE), st));
      SBP_CK(gemm(mk_gemm(R, d, dkv, DT_F32, p.dvg, false, dkv, dt, w->wv, false, d, DT_F32,
                          p.dn1, d, EPI_ACC), st));
      SBP_CK(gemm(over_tokens(mk_gemm(dkv, d, R, DT_F32, p.dkpre, true, dkv, dt, p.n1, false, d,
                                      DT_F32, gr->wk, d, EPI_ACC)), st));
      SBP_CK(gemm(over_tokens(mk_gemm(dkv, d, R, DT_F32, p.dvg, true, dkv, dt, p.n1, false, d,
                                      DT_F32, gr->wv, d, EPI_ACC)), st));
    }
    if (has_bias) {
      SBP_CK(colsum_acc(R, dkv, p.dkpre, gr->bk, p.cpart, st));
      SBP_CK(colsum_acc(R, dkv, p.dvg, gr->bv, p.cpart, st));
    }
    return SBP_OK;
  };

  if (reverse) {
    // the K/V prefix of the whole sequence, chunk by chunk
    for (int j = 0; j < D; ++j) {
      int64_t s, e;
      chunk_range(T, D, j, s, e);
      const int64_t Tc = e - s;
      const void* xc = static_cast<const char*>(x) + s * d * es;
      if (B > 1) {
        SBP_CK(gather_chunk(B, T, Tc, s, d, dt, x, p.xg, st));
        xc = p.xg;
      }
      if (sbp_status r = layer_chunk_kv(L, *w, p, xc, s, Tc, st)) return r;
    }
  }

  for (int ii = 0; ii < D; ++ii) {
    const int i = reverse ? D - 1 - ii : ii;
    int64_t s, e;
    chunk_range(T, D, i, s, e);
    const int64_t Tc = e - s, R = B * Tc;
    // a single sequence's chunk is contiguous: use it in place, no gather / scatter
    const void* xc = static_cast<const char*>(x) + s * d * es;
    const float* dyc = dy + s * d;
    float* dxc = dx + s * d;
    if (B > 1) {
      SBP_CK(gather_chunk(B, T, Tc, s, d, dt, x, p.xg, st));
      SBP_CK(gather_chunk(B, T, Tc, s, d, DT_F32, dy, p.dyg, st));
      xc = p.xg;
      dyc = p.dyg;
      dxc = p.dxg;
    }
    if (sbp_status r = layer_chunk_forward(L, *w, p, xc, s, Tc, st, reverse)) return r;
    // ---- MLP backward.  fp32 gradients enter the tensor cores as bf16 operands (rounded
    // per element, so the rounding does not depend on the chunking).
    const bool b16 = dt == DT_BF16;
    const void* dY = dyc;
    int dYdt = DT_F32;
    if (b16) {
      SBP_CK(copy_cast(R * d, DT_F32, dyc, DT_BF16, p.dyg16, st));
      dY = p.dyg16;
      dYdt = DT_BF16;
    }
    SBP_CK(fork_to(0, 8));
    SBP_CK(gemm(over_tokens(mk_gemm(d, f, R, dYdt, dY, true, d, dt, p.m, false, f, DT_F32,
                                    gr->w_down, f, EPI_ACC)), s0));
    {
      // dM = dY W_d with the SwiGLU backward fused into the product's epilogue:
      // (dG, dU) = dM * (u sigma'(g) ..., silu(g)) written straight into dgu
      GemmDesc gd = mk_gemm(R, f, d, dYdt, dY, false, d, dt, w->w_down, false, f, dt, p.dgu,
                            2 * f, EPI_SWIGLU_BWD);
      gd.aux = p.gu;
      gd.aux_ld = 2 * f;
      gd.aux_off = f;
      SBP_CK(gemm(gd, st));
    }
    const char* dU = static_cast<const char*>(p.dgu) + f * es;
    SBP_CK(gemm(mk_gemm(R, d, f, dt, p.dgu, false, 2 * f, dt, w->w_gate, false, d, DT_F32, p.dn2,
                        d, EPI_STORE), st));
    SBP_CK(gemm(mk_gemm(R, d, f, dt, dU, false, 2 * f, dt, w->w_up, false, d, DT_F32, p.dn2, d,
                        EPI_ACC), st));
    SBP_CK(fork_to(1, 9));
    SBP_CK(gemm(over_tokens(mk_gemm(f, d, R, dt, p.dgu, true, 2 * f, dt, p.n2, false, d, DT_F32,
                                    gr->w_gate, d, EPI_ACC)), s1));
    SBP_CK(gemm(over_tokens(mk_gemm(f, d, R, dt, dU, true, 2 * f, dt, p.n2, false, d, DT_F32,
                                    gr->w_up, d, EPI_ACC)), s1));
    SBP_CK(rmsnorm_bwd(R, d, DT_F32, p.hbuf, dt, w->ln2_g, p.rstd2, p.dn2, dyc, p.dh, 0,
                       gr->ln2_g, p.rpart, st));
    // ---- attention output projection backward
    const void* dH = p.dh;
    int dHdt = DT_F32;
    if (b16) {
      SBP_CK(copy_cast(R * d, DT_F32, p.dh, DT_BF16, p.dh16, st));
      dH = p.dh16;
      dHdt = DT_BF16;
    }
    SBP_CK(fork_to(0, 10));
    SBP_CK(gemm(over_tokens(mk_gemm(d, dq, R, dHdt, dH, true, d, dt, p.o, false, dq, DT_F32,
                                    gr->wo, dq, EPI_ACC)), s0));
    SBP_CK(gemm(mk_gemm(R, dq, d, dHdt, dH, false, d, dt, w->wo, false, dq, dt, p.dO, dq,
                        EPI_STORE), st));
    // ---- attention backward over the causal prefix; dK/dV accumulate in fp32
    SBP_CK(attn_bwd(B, T, Tc, s, H, Hkv, hd, dt, p.q, p.Kp, p.Vp, p.o, p.dO, p.alse, p.delta,
                    p.dq, p.dKp, p.dVp, st));
    SBP_CK(rope_inv_f32(R, Tc, s, H, hd, p.dq, p.cosb, p.sinb, st));
    // ---- q projection backward
    // dQ of a query row is a fixed-order sum over its key tiles (the same at every D), so a
    // plain per-element bf16 rounding is D-independent
    const void* dQ = p.dq;
    int dQdt = DT_F32;
    if (b16) {
      SBP_CK(copy_cast(R * dq, DT_F32, p.dq, DT_BF16, p.dq16, st));
      dQ = p.dq16;
      dQdt = DT_BF16;
    }
    SBP_CK(fork_to(1, 11));
    SBP_CK(gemm(over_tokens(mk_gemm(dq, d, R, dQdt, dQ, true, dq, dt, p.n1, false, d, DT_F32,
                                    gr->wq, d, EPI_ACC)), s1));
    if (has_bias) SBP_CK(colsum_acc(R, dq, p.dq, gr->bq, p.cpart, s1));
    SBP_CK(gemm(mk_gemm(R, d, dq, dQdt, dQ, false, dq, dt, w->wq, false, d, DT_F32, p.dn1, d,
                        EPI_STORE), st));
    // in reverse order this chunk's dK/dV rows are final: its K/V part joins dn1 here
    if (reverse)
      if (sbp_status r = kv_backward(s, Tc, true)) return r;
    SBP_CK(rmsnorm_bwd(R, d, dt, xc, dt, w->ln1_g, p.rstd1, p.dn1, p.dh, dxc, 0, gr->ln1_g,
                       p.rpart, st));
    if (B > 1) SBP_CK(scatter_chunk_f32(B, T, Tc, s, d, p.dxg, dx, 0, st));
    SBP_CK(join_all());
  }
  if (reverse) return SBP_OK;
  // ---- K/V projection backward, chunk by chunk, once every later chunk has added its dK/dV
  for (int j = 0; j < D; ++j) {
    int64_t s, e;
    chunk_range(T, D, j, s, e);
    const int64_t Tc = e - s, R = B * Tc;
    const void* xc = static_cast<const char*>(x) + s * d * es;
    if (B > 1) {
      SBP_CK(gather_chunk(B, T, Tc, s, d, dt, x, p.xg, st));
      xc = p.xg;
    }
    SBP_CK(rmsnorm_fwd(R, d, dt, xc, dt, w->ln1_g, dt, p.n1, p.rstd1, L.rms_eps, st));
    if (sbp_status r = kv_backward(s, Tc, false)) return r;
    if (B > 1) {
      SBP_CK(rmsnorm_bwd(R, d, dt, xc, dt, w->ln1_g, p.rstd1, p.dn1, nullptr, p.dxg, 0,
                         gr->ln1_g, p.rpart, st));
      SBP_CK(scatter_chunk_f32(B, T, Tc, s, d, p.dxg, dx, 1, st));
    } else {
      SBP_CK(rmsnorm_bwd(R, d, dt, xc, dt, w->ln1_g, p.rstd1, p.dn1, nullptr, dx + s * d, 1,
                         gr->ln1_g, p.rpart, st));
    }
    SBP_CK(join_all());
  }
  return SBP_OK;
}

sbp_status sbp_decoder_layer_backward_stream(const sbp_layer_cfg* cfg,
                                             const sbp_layer_weights* w, const void* x,
                                             const float* dy, float* dx,
                                             const sbp_layer_grads* gr, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  return layer_backward_run(cfg, w, x, dy, dx, gr, workspace, workspace_bytes, stream, false);
}

sbp_status sbp_decoder_layer_backward_stream_reverse(const sbp_layer_cfg* cfg,
                                                     const sbp_layer_weights* w, const void* x,
                                                     const float* dy, float* dx,
                                                     const sbp_layer_grads* gr,
                                                     void* workspace, size_t workspace_bytes,
                                                     void* stream) {
  return layer_backward_run(cfg, w, x, dy, dx, gr, workspace, workspace_bytes, stream, true);
}

sbp_status sbp_decoder_layer_forward_stream(const sbp_layer_cfg* cfg,
                                            const sbp_layer_weights* w, const void* x, void* y,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream) {
  if (sbp_status s = check_layer_cfg(cfg)) return s;
  bool has_bias = false;
  if (sbp_status s = check_weights(w, &has_bias)) return s;
  if (!x || !y || !aligned16(x) || !aligned16(y))
    return fail(SBP_ERR_INVALID_ARG, "x/y NULL or misaligned");
  const sbp_layer_cfg& L = *cfg;
  const size_t need = sbp_decoder_layer_workspace_size(cfg);
  if (sbp_status s = check_ws(workspace, workspace_bytes, need)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  LayerPlan p;
  layer_carve(c, L, p);
  const int dt = L.dtype;
  const int64_t B = L.batch, T = L.seq_len, d = L.d_model, f = L.ffn;
  tl_status = p.status;
  SBP_CK(cudaMemsetAsync(p.status, 0, sizeof(int), st));
  SBP_CK(rope_table(T, L.head_dim, L.rope_theta, p.cosb, p.sinb, st));
  {
    const size_t kvb = dt_size(dt) * (size_t)B * T * L.n_kv_heads * L.head_dim;
    SBP_CK(cudaMemsetAsync(p.Kp, 0, kvb, st));
    SBP_CK(cudaMemsetAsync(p.Vp, 0, kvb, st));
  }
  for (int i = 0; i < L.num_chunks; ++i) {
    int64_t s, e;
    chunk_range(T, L.num_chunks, i, s, e);
    const int64_t Tc = e - s, R = B * Tc;
    const void* xc = static_cast<const char*>(x) + s * d * dt_size(dt);
    if (B > 1) {
      SBP_CK(gather_chunk(B, T, Tc, s, d, dt, x, p.xg, st));
      xc = p.xg;
    }
    if (sbp_status r = layer_chunk_forward(L, *w, p, xc, s, Tc, st)) return r;
    SBP_CK(gemm(mk_gemm(R, d, f, dt, p.m, false, f, dt, w->w_down, true, f, DT_F32, p.hbuf, d,
                        EPI_ACC), st));
    if (B > 1) {
      SBP_CK(copy_cast(R * d, DT_F32, p.hbuf, dt, p.xg, st));
      SBP_CK(scatter_chunk(B, T, Tc, s, d, dt, p.xg, y, st));
    } else {
      SBP_CK(copy_cast(R * d, DT_F32, p.hbuf, dt, static_cast<char*>(y) + s * d * dt_size(dt),
                       st));
    }
  }
  return SBP_OK;
}

// ------------------------------------------------------------------------------- support
sbp_status sbp_rmsnorm_forward(int64_t rows, int64_t cols, sbp_dtype dt, float eps,
                               const void* x, const void* g, void* y, float* rstd,
                               void* stream) {
  if (rows <= 0 || cols <= 0) return fail(SBP_ERR_INVALID_ARG, "sizes must be positive");
  if (!x || !g || !y) return fail(SBP_ERR_INVALID_ARG, "x/g/y is NULL");
  SBP_CK(rmsnorm_fwd(rows, cols, dt, x, dt, g, dt, y, rstd, eps,
                     static_cast<cudaStream_t>(stream)));
  return SBP_OK;
}

size_t sbp_rmsnorm_backward_workspace_size(int64_t rows, int64_t cols) {
  (void)rows;
  return rmsnorm_bwd_partial_floats(cols) * sizeof(float);
}

sbp_status sbp_rmsnorm_backward(int64_t rows, int64_t cols, sbp_dtype dt, const void* x,
                                const void* g, const float* rstd, const float* dy, float* dx,
                                int accumulate, float* dg, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (rows <= 0 || cols <= 0) return fail(SBP_ERR_INVALID_ARG, "sizes must be positive");
  if (!x || !g || !rstd || !dy || !dx || !workspace)
    return fail(SBP_ERR_INVALID_ARG, "a required pointer is NULL");
  if (workspace_bytes < sbp_rmsnorm_backward_workspace_size(rows, cols))
    return fail(SBP_ERR_WORKSPACE, "workspace too small");
  SBP_CK(rmsnorm_bwd(rows, cols, dt, x, dt, g, rstd, dy, nullptr, dx, accumulate, dg,
                     static_cast<float*>(workspace), static_cast<cudaStream_t>(stream)));
  return SBP_OK;
}

sbp_status sbp_embedding_forward(int64_t rows, int64_t cols, int64_t vocab, sbp_dtype dt,
                                 const int32_t* ids, const void* table, void* y, void* stream) {
  if (rows <= 0 || cols <= 0 || vocab <= 0) return fail(SBP_ERR_INVALID_ARG, "bad sizes");
  if (!ids || !table || !y) return fail(SBP_ERR_INVALID_ARG, "a required pointer is NULL");
  SBP_CK(embed_fwd(rows, cols, vocab, dt, ids, table, y, static_cast<cudaStream_t>(stream)));
  return SBP_OK;
}

size_t sbp_embedding_backward_workspace_size(int64_t rows, int64_t vocab) {
  return embed_bwd_ws_ints(rows, vocab) * sizeof(int);
}

sbp_status sbp_embedding_backward(int64_t rows, int64_t cols, int64_t vocab,
                                  const int32_t* ids, const float* dy, float* d_table,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (rows <= 0 || cols <= 0 || vocab <= 0) return fail(SBP_ERR_INVALID_ARG, "bad sizes");
  if (!ids || !dy || !d_table || !workspace)
    return fail(SBP_ERR_INVALID_ARG, "a required pointer is NULL");
  if (workspace_bytes < sbp_embedding_backward_workspace_size(rows, vocab))
    return fail(SBP_ERR_WORKSPACE, "workspace too small");
  SBP_CK(embed_bwd(rows, cols, vocab, ids, dy, d_table, static_cast<int*>(workspace),
                   static_cast<cudaStream_t>(stream)));
  return SBP_OK;
}

// ------------------------------------------------------------------------------- debug
sbp_status sbp_debug_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, int a_trans,
                               int64_t lda, const void* B, int b_trans, int64_t ldb, float* C,
                               int64_t ldc, int accumulate, int path, int64_t kblk,
                               void* workspace, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return fail(SBP_ERR_INVALID_ARG, "sizes must be positive");
  if (!A || !B || !C || !workspace) return fail(SBP_ERR_INVALID_ARG, "NULL pointer");
  if (path < 0 || path > 4) return fail(SBP_ERR_INVALID_ARG, "path must be 0 .. 4");
  if (kblk < 0 || kblk % 64 != 0)
    return fail(SBP_ERR_INVALID_ARG, "kblk must be 0 or a positive multiple of 64");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  tl_status = static_cast<int*>(workspace);
  GemmDesc g = mk_gemm(M, N, K, DT_BF16, A, a_trans != 0, lda, DT_BF16, B, b_trans != 0, ldb,
                       DT_F32, C, ldc, accumulate ? EPI_ACC : EPI_STORE);
  g.path = path;
  g.kblk = kblk;
  if (path >= 2 && !gemm_tc_supported(g))
    return fail(SBP_ERR_UNSUPPORTED, "layout not supported by the tensor-core GEMM");
  if (path == 4 && kblk % 128 != 0)
    return fail(SBP_ERR_UNSUPPORTED, "the CTA-pair GEMM takes K blocks of whole 128-column stages");
  SBP_CK(gemm(g, st));
  return SBP_OK;
}

sbp_status sbp_debug_gemm_stall_bf16(int64_t M, int64_t N, int64_t K, const void* A,
                                     const void* B, float* C, int64_t wait_limit_ns,
                                     void* workspace, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return fail(SBP_ERR_INVALID_ARG, "sizes must be positive");
  if (!A || !B || !C || !workspace) return fail(SBP_ERR_INVALID_ARG, "NULL pointer");
  if (wait_limit_ns < 100000 || wait_limit_ns > 2000000000)
    return fail(SBP_ERR_INVALID_ARG, "wait_limit_ns must be in [1e5, 2e9]");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  tl_status = static_cast<int*>(workspace);
  GemmDesc g = mk_gemm(M, N, K, DT_BF16, A, false, K, DT_BF16, B, true, K, DT_F32, C, N,
                       EPI_STORE);
  g.path = 3;
  g.stall_wait_ns = wait_limit_ns;
  if (!gemm_tc_supported(g))
    return fail(SBP_ERR_UNSUPPORTED, "layout not supported by the tensor-core GEMM");
  SBP_CK(gemm(g, st));
  return SBP_OK;
}

sbp_status sbp_debug_attn_fwd_bf16(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H,
                                   int64_t Hkv, int64_t hd, const void* q, const void* Kp,
                                   const void* Vp, void* o, float* lse, int path, void* workspace,
                                   void* stream) {
  if (B <= 0 || T <= 0 || Tc <= 0 || s < 0 || s + Tc > T || H <= 0 || Hkv <= 0 || H % Hkv ||
      hd <= 0 || hd % 2 || hd > 256)
    return fail(SBP_ERR_INVALID_ARG, "bad attention sizes");
  if (!q || !Kp || !Vp || !o || !lse || !workspace) return fail(SBP_ERR_INVALID_ARG, "NULL pointer");
  if (path < 0 || path > 2) return fail(SBP_ERR_INVALID_ARG, "path must be 0, 1 or 2");
  if (path == 2 && !attn_tc_supported(hd, DT_BF16, q, Kp, Vp, o))
    return fail(SBP_ERR_UNSUPPORTED, "the tensor-core attention needs head_dim 128 and aligned rows");
  tl_status = static_cast<int*>(workspace);
  // the split scratch follows the status word: part, ml, flags
  AttnFwdSplit sc;
  sc.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
  sc.ml = sc.part + B * Tc * H * hd;
  sc.flags = reinterpret_cast<int*>(sc.ml + 2 * B * Tc * H);
  SBP_CK(attn_fwd(B, T, Tc, s, H, Hkv, hd, DT_BF16, q, Kp, Vp, o, lse, sc,
                  static_cast<cudaStream_t>(stream), path));
  return SBP_OK;
}

sbp_status sbp_debug_attn_bwd_bf16(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H,
                                   int64_t Hkv, int64_t hd, const void* q, const void* Kp,
                                   const void* Vp, const void* o, const void* dO,
                                   const float* lse, float* dq, float* dKp, float* dVp,
                                   int path, void* workspace, void* stream) {
  if (B <= 0 || T <= 0 || Tc <= 0 || s < 0 || s + Tc > T || H <= 0 || Hkv <= 0 || H % Hkv ||
      hd <= 0 || hd % 2 || hd > 256)
    return fail(SBP_ERR_INVALID_ARG, "bad attention sizes");
  if (!q || !Kp || !Vp || !o || !dO || !lse || !dq || !dKp || !dVp || !workspace)
    return fail(SBP_ERR_INVALID_ARG, "NULL pointer");
  if (path < 0 || path > 2) return fail(SBP_ERR_INVALID_ARG, "path must be 0, 1 or 2");
  if (path == 2 && !attn_bwd_tc_supported(hd, DT_BF16, q, Kp, Vp, o, dO, dq))
    return fail(SBP_ERR_UNSUPPORTED, "the tensor-core attention needs head_dim 128 and aligned rows");
  tl_status = static_cast<int*>(workspace);
  float* delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
  // (the caller provides kStatusBytes + 4 * attn_bwd_scratch_floats(B, Tc, H) bytes)
  SBP_CK(attn_bwd(B, T, Tc, s, H, Hkv, hd, DT_BF16, q, Kp, Vp, o, dO, lse, delta, dq, dKp, dVp,
                  static_cast<cudaStream_t>(stream), path));
  return SBP_OK;
}

}  // extern "C"
