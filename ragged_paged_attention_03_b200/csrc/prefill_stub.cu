// prefill_stub.cu -- launcher of the tensor-core prefill kernel until it
// exists; the planner does not route work to it.
#include "kernels.h"
namespace rpa {
cudaError_t launch_prefill(const Problem &, const PrefillTile *, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace rpa
