// GEMM dispatch: bf16 x bf16 products in a layout TMA can tile go to the tcgen05 kernel,
// everything else (fp32 operands, mixed fp32/bf16 operands, unaligned views) to the CUDA cores.
#include "sbp_internal.cuh"

namespace sbp {

cudaError_t gemm_simt(const GemmDesc& g, cudaStream_t st);
cudaError_t gemm_tc(const GemmDesc& g, int* err, cudaStream_t st);

cudaError_t gemm(const GemmDesc& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  const bool tc = g.path != 1 && gemm_tc_supported(g);
  if (!tc && g.path == 2) return cudaErrorNotSupported;
  const int kind = tc ? PROF_GEMM_TC : PROF_GEMM_SIMT;
  prof_mark_begin(kind, st);
  const cudaError_t e = tc ? gemm_tc(g, g.err, st) : gemm_simt(g, st);
  prof_mark_end(kind, st);
  return e;
}

}  // namespace sbp
