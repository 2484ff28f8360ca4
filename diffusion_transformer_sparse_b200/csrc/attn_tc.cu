// Tensor-core (tcgen05) attention core.
#include "common.cuh"

namespace ptdit {
bool attention_tc_supported(const AttnArgs &) { return false; }
cudaError_t launch_attention_tc(const AttnArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace ptdit
