// Tensor-core hybrid attention (placeholder until the tcgen05 kernel lands).
#include "attn_tc.cuh"

namespace svg {
bool attn_tc_supported(int, int) { return false; }
size_t attn_tc_ws_bytes(int, int, int, int, int) { return 0; }
cudaError_t attn_tc_run(const void*, const void*, const void*, const int32_t*, const int32_t*,
                        const int32_t*, const float*, const float*, const int32_t*, const int32_t*,
                        int, int, int, int, int, int, float, void*, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace svg
