// Tensor-core (tcgen05) k-means assignment for bf16 tokens; see kmeans_tc.cu.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace svg {
bool kmeans_tc_supported(int d, int C);
// Supported shape, at least one full tile of tokens, 16-byte aligned tokens
// and a driver that encodes TMA maps.
bool kmeans_tc_usable(const void* X, int N, int d, int C);
size_t kmeans_tc_ws_bytes(int H, int N, int d, int C);
// Once per k-means call: per-token norms used by the rounding bound.
cudaError_t kmeans_tc_prepare_rows(const void* X, int H, int N, int d, void* ws, cudaStream_t st);
// One assignment pass against float32 centroids `cent` [H,C,d].
cudaError_t kmeans_assign_tc(const void* X, int H, int N, int d, int C, const float* cent,
                             int32_t* labels, void* ws, cudaStream_t st);
}  // namespace svg
