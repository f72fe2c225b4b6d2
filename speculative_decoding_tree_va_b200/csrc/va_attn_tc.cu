// Tensor-core (tcgen05) bf16 tree-verify attention -- placeholder until the
// sm_100a kernel lands; reports "not supported" so no silent fallback exists.
#include "va_common.cuh"

namespace va {
cudaError_t launch_attn_tc(const va_attn_args&, int, float*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace va
