/*
 * sbp_debug.h -- test hooks of libsbp (not part of the streamed-backward API).
 *
 * The paper has no counterpart: these calls exist so that the tests can check a single
 * building block of the library (the GEMM engine) against a reference, path by path.
 */
#ifndef SBP_DEBUG_H_
#define SBP_DEBUG_H_

#include <stddef.h>
#include <stdint.h>

#include "sbp.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * C[m, n] (+)= sum_k op(A)[m, k] * op(B)[k, n] with bf16 A and B and fp32 C, all row-major:
 *   a_trans = 0: A is [M, K] with leading dimension lda;  1: A is [K, M] (op(A) = A^T)
 *   b_trans = 0: B is [K, N] with leading dimension ldb;  1: B is [N, K] (op(B) = B^T)
 * C is [M, N] with leading dimension ldc; accumulate = 0 overwrites, 1 adds.
 * path: 0 = automatic, 1 = CUDA cores, 2 = tensor cores (either kernel), 3 = tensor cores with
 * one CTA per 128 x 256 tile, 4 = tensor cores with a CTA pair per 256 x 256 tile
 * (SBP_ERR_UNSUPPORTED for 2..4 if the layout is not one the tensor-core kernels
 * take, and for 4 if kblk is not a multiple of 128, the pair kernel's stage depth; path 0 and
 * 2 then take the single-CTA kernel).  kblk = 0 sums all of K in one accumulator; kblk > 0
 * (a multiple of 64, else
 * SBP_ERR_INVALID_ARG) adds the partial products of consecutive K blocks of that length into
 * C one after another, in fp32 (the rounding the weight-gradient products over tokens use).
 * `workspace` (>= 256 bytes, device) receives the device status word (see
 * sbp_get_device_status).  Device pointers, queued on `stream`.
 */
sbp_status sbp_debug_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, int a_trans,
                               int64_t lda, const void* B, int b_trans, int64_t ldb, float* C,
                               int64_t ldc, int accumulate, int path, int64_t kblk,
                               void* workspace, void* stream);

/*
 * Test of the bounded waits (failure detection without a GPU fault).  Launches the single-CTA
 * tensor-core GEMM of C = A B^T (A [M, K], B [N, K], both bf16 row-major with leading
 * dimension K; C [M, N] fp32) with its producer told to issue no copy at all and every
 * mbarrier wait bounded by `wait_limit_ns` (1e5 .. 2e9 ns, else SBP_ERR_INVALID_ARG).  The MMA
 * issuer's first operand wait therefore runs out with no copy and no MMA in flight; the kernel
 * takes its timeout exit (every role winds down, TMEM is freed) and raises SBP_ERR_DEVICE_TIMEOUT
 * in the status word at the start of `workspace` (>= 256 bytes, zeroed by the caller), which
 * sbp_get_device_status reports.  C is not written.  The same launch path as a normal GEMM,
 * so a context that passes this call keeps working.  Device pointers, queued on `stream`.
 */
sbp_status sbp_debug_gemm_stall_bf16(int64_t M, int64_t N, int64_t K, const void* A,
                                     const void* B, float* C, int64_t wait_limit_ns,
                                     void* workspace, void* stream);

/*
 * Causal GQA attention forward of one query chunk over its key prefix (bf16):
 *   q  [B * Tc, H, hd]  (chunk rows; row r is position s + r % Tc of sequence r / Tc)
 *   Kp, Vp [B, T, Hkv, hd] (keys/values of whole sequences; positions < s + Tc are read)
 *   o  [B * Tc, H, hd] bf16 out;  lse [B * Tc, H] fp32 out (natural log of the softmax sum)
 * path: 0 automatic, 1 CUDA cores, 2 tensor cores (head_dim 128 only).
 * `workspace` (device, 16-byte aligned) holds the 256-byte status word and then the scratch
 * of the tensor-core path's key-range split: 256 + 4 * B * Tc * H * (hd + 2) + 8 * B * H * P
 * bytes, P = ceil(ceil(Tc / 128) / 2) query-tile pairs.  Query rows whose keys reach past a
 * quarter of the sequence (key tile ceil(ceil(T / 128) / 4)) are computed as two partial
 * softmaxes over the keys before and after that point and combined, in that order, by the
 * second of the two CTAs to finish; the split point depends on T only, so a row's result does
 * not depend on the chunking.
 */
sbp_status sbp_debug_attn_fwd_bf16(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H,
                                   int64_t Hkv, int64_t hd, const void* q, const void* Kp,
                                   const void* Vp, void* o, float* lse, int path, void* workspace,
                                   void* stream);

/*
 * Backward of sbp_debug_attn_fwd_bf16 given its o and lse and the upstream dO [B*Tc, H, hd]
 * (bf16): dq [B*Tc, H, hd] fp32 is overwritten; dKp, dVp [B, T, Hkv, hd] fp32 are accumulated
 * (+=) for key positions < s + Tc.  `workspace` needs 256 + 8 * H * B * ceil(Tc / 128) * 128
 * bytes (and at least 256 + 4 * B * Tc * H).
 */
sbp_status sbp_debug_attn_bwd_bf16(int64_t B, int64_t T, int64_t Tc, int64_t s, int64_t H,
                                   int64_t Hkv, int64_t hd, const void* q, const void* Kp,
                                   const void* Vp, const void* o, const void* dO,
                                   const float* lse, float* dq, float* dKp, float* dVp,
                                   int path, void* workspace, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SBP_DEBUG_H_ */
