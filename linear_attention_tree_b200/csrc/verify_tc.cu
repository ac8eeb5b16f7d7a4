// Tensor-core tree verification (placeholder until the tcgen05 kernel lands).
#include "tv_internal.cuh"

namespace tv {
cudaError_t launch_verify_tc(const VerifyArgs &, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace tv
