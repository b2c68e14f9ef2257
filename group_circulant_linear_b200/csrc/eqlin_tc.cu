// eqlin_tc.cu -- tcgen05 (5th-generation tensor core) kernels; placeholder.
#include "eqlin_internal.cuh"

namespace eqlin {
bool tc_supported(const Handle&, bool) { return false; }
cudaError_t launch_tc_apply(const Handle&, bool, const void*, void*, int64_t, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace eqlin
