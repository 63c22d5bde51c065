// Tensor-core grouped GEMM path of the routed layer (tcgen05 block-scaled MMA).
#include "ffn_gemm.cuh"

namespace nvfp4moe {

bool gemm_path_available() { return false; }

nvfp4moe_status launch_gemm_ffn(const GemmFfnArgs&, cudaStream_t) {
  return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "tensor-core grouped GEMM path not built");
}

}  // namespace nvfp4moe
