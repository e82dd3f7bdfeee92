// Tensor-core k-means assignment (placeholder until the tcgen05 kernel lands).
#include "kmeans_tc.cuh"
#include "internal.h"

namespace svg {
bool kmeans_tc_supported(int, int) { return false; }
size_t kmeans_tc_ws_bytes(int, int, int, int) { return 0; }
cudaError_t kmeans_tc_prepare_rows(const void*, int, int, int, void*, cudaStream_t) { return cudaSuccess; }
cudaError_t kmeans_assign_tc(const void*, int, int, int, int, const float*, int32_t*, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace svg
