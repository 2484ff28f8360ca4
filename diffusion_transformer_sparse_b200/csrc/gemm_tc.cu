// Tensor-core (tcgen05) projection GEMM.
#include "common.cuh"

namespace ptdit {
bool gemm_tc_supported(const GemmArgs &) { return false; }
cudaError_t launch_gemm_tc(const GemmArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace ptdit
