// stubs.cu -- launchers of kernels not built yet; never reached (the planner
// does not route work to them).
#include "kernels.h"
namespace rpa {
cudaError_t launch_decode(const Problem &, const DecodeItem *, int, float *, float *, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_combine(const Problem &, const CombineItem *, int, const float *, const float *,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_prefill(const Problem &, const PrefillTile *, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace rpa
