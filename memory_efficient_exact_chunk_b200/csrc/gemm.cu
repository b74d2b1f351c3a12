// GEMM dispatch: bf16 x bf16 products in a layout TMA can tile go to the tcgen05 kernel,
// everything else (fp32 operands, mixed fp32/bf16 operands, unaligned views) to the CUDA cores.
#include "sbp_internal.cuh"

namespace sbp {

cudaError_t gemm_simt(const GemmDesc& g, cudaStream_t st);
cudaError_t gemm_tc(const GemmDesc& g, int* err, cudaStream_t st);
cudaError_t gemm_tc_pair(const GemmDesc& g, int* err, cudaStream_t st);

// The CTA-pair kernel needs enough 256 x 256 tiles to occupy every SM pair, and K blocks
// (kblk) that are whole 128-column stages.
static bool use_pair(const GemmDesc& g) {
  const int64_t tiles = ((g.M + 255) / 256) * ((g.N + 255) / 256);
  return g.path != 3 && tiles >= 74 && g.kblk % 128 == 0;
}

cudaError_t gemm(const GemmDesc& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (g.kblk < 0 || (g.kblk > 0 && (g.kblk % 64 != 0 || (g.epi != EPI_STORE && g.epi != EPI_ACC))))
    return cudaErrorInvalidValue;
  const bool tc = g.path != 1 && gemm_tc_supported(g);
  if (!tc && (g.path >= 2 || g.epi == EPI_ROPE || g.epi == EPI_SWIGLU_FWD))
    return cudaErrorNotSupported;
  const int kind = tc ? PROF_GEMM_TC : PROF_GEMM_SIMT;
  prof_mark_begin(kind, st);
  const cudaError_t e = tc ? ((g.path == 4 || (g.path == 0 && use_pair(g))) ? gemm_tc_pair(g, g.err, st)
                                                                            : gemm_tc(g, g.err, st))
                           : gemm_simt(g, st);
  prof_mark_end(kind, st);
  return e;
}

}  // namespace sbp
