// Tensor-core (tcgen05) attention kernels: not yet built.
#include "common.cuh"

namespace moba {
bool tc_supported(const Dims&) { return false; }
cudaError_t launch_history_tc(const Dims&, const Chunk&, const void*, const void*, const void*,
                              const int32_t*, const Regroup&, const Partials&, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_current_tc(const Dims&, const Chunk&, const void*, const void*, const void*,
                              const int32_t*, const int32_t*, const Partials&, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_dense_tc(const Dims&, const void*, const void*, const void*, const int32_t*,
                            void*, float*, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace moba
