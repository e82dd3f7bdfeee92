// Semantic k-means of queries / keys (SVG-EAR review, step (1): "Flash
// k-means" clustering; gist.science summary 2.A).  Lloyd iterations:
//   assign: label(x) = argmin_c ||x - mu_c||^2   (ties -> smaller c)
//   update: mu_c = mean of the x labelled c      (empty c keeps mu_c)
// `iters` assign->update rounds, then a final assignment.
//
// Assignment has two implementations:
//  * bf16 inputs: a tcgen05 tensor-core GEMM of the token tile against the
//    bf16-rounded centroids with an argmin epilogue; every token whose
//    best/second-best scores lie within the proven rounding bound is
//    re-decided in float64 (kmeans_tc.cu), so labels equal the exact argmin.
//  * float32 inputs: float64 distances on the CUDA cores (k_assign_exact).
// The update is a deterministic segmented mean over the counting-sort order
// (no float atomics), accumulated in float64.
#include "common.cuh"
#include "internal.h"
#include "kmeans_tc.cuh"

namespace svg {

namespace {

template <typename T, int D>
__global__ void k_init_deterministic(const T* __restrict__ X, int N, int C, float* __restrict__ cent) {
  const int h = blockIdx.y, c = blockIdx.x;
  const long long src = (long long)c * N / C;
  for (int t = threadIdx.x; t < D; t += blockDim.x)
    cent[((size_t)h * C + c) * D + t] = to_f(X[((size_t)h * N + src) * D + t]);
}

// float64 distances for every (token, centroid); 64 tokens per block.
template <typename T, int D>
__global__ void __launch_bounds__(64) k_assign_exact(const T* __restrict__ X, const float* __restrict__ cent,
                                                     int N, int C, int32_t* __restrict__ labels) {
  constexpr int CT = 16, BT = 64;
  __shared__ float xs[D][BT];
  __shared__ float cs[CT][D];
  const int h = blockIdx.y, i0 = blockIdx.x * BT, tid = threadIdx.x;
  const T* Xh = X + (size_t)h * N * D;
  for (int e = tid; e < BT * D; e += BT) {
    const int r = e / D, t = e % D;
    xs[t][r] = (i0 + r < N) ? to_f(Xh[(size_t)(i0 + r) * D + t]) : 0.f;
  }
  double best = 1.0e300;
  int bi = 0;
  const float* ch = cent + (size_t)h * C * D;
  for (int c0 = 0; c0 < C; c0 += CT) {
    __syncthreads();
    const int nc = min(CT, C - c0);
    for (int e = tid; e < nc * D; e += BT) cs[e / D][e % D] = ch[(size_t)c0 * D + e];
    __syncthreads();
    for (int cc = 0; cc < nc; ++cc) {
      double acc = 0.0;
#pragma unroll 16
      for (int t = 0; t < D; ++t) {
        const double df = (double)xs[t][tid] - (double)cs[cc][t];
        acc = fma(df, df, acc);
      }
      if (acc < best) { best = acc; bi = c0 + cc; }
    }
  }
  if (i0 + tid < N) labels[(size_t)h * N + i0 + tid] = bi;
}

// Segmented float64 mean over the sorted membership list of cluster c.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_update(const T* __restrict__ X, const int32_t* __restrict__ perm,
                                                const int32_t* __restrict__ off, int N, int C,
                                                float* __restrict__ cent) {
  constexpr int PER = D / 32;
  constexpr int NW = 8;
  __shared__ double red[NW][D];
  const int h = blockIdx.y, c = blockIdx.x;
  const int beg = off[(size_t)h * (C + 1) + c], end = off[(size_t)h * (C + 1) + c + 1];
  if (beg >= end) return;  // empty cluster keeps its centroid
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* Xh = X + (size_t)h * N * D + lane * PER;
  const int32_t* ph = perm + (size_t)h * N;
  double acc[PER];
#pragma unroll
  for (int t = 0; t < PER; ++t) acc[t] = 0.0;
  int r = beg + w;
  for (; r + 7 * NW < end; r += 8 * NW) {
    int idx[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) idx[u] = ph[r + u * NW];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if constexpr (PER == 4) {
        float4 v = ld4(Xh + (size_t)idx[u] * D);
        acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
      } else {
        float2 v = ld2(Xh + (size_t)idx[u] * D);
        acc[0] += v.x; acc[1] += v.y;
      }
    }
  }
  // at most eight rows of this warp remain: one predicated batch (loads in
  // flight together), added in the same row order as before
  {
    int idx[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) idx[u] = r + u * NW < end ? ph[r + u * NW] : -1;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (idx[u] < 0) continue;
      if constexpr (PER == 4) {
        float4 v = ld4(Xh + (size_t)idx[u] * D);
        acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
      } else {
        float2 v = ld2(Xh + (size_t)idx[u] * D);
        acc[0] += v.x; acc[1] += v.y;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < PER; ++t) red[w][lane * PER + t] = acc[t];
  __syncthreads();
  const double inv = 1.0 / (double)(end - beg);
  for (int t = threadIdx.x; t < D; t += blockDim.x) {
    double s = 0.0;
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) s += red[ww][t];
    cent[((size_t)h * C + c) * D + t] = (float)(s * inv);
  }
}

template <typename T, int D>
cudaError_t run_t(const T* X, int H, int N, int C, int iters, const float* init, float* cent,
                  int32_t* labels, int32_t* counts, int32_t* offsets, int32_t* perm, char* sort_ws,
                  void* tc_ws, bool use_tc, cudaStream_t st) {
  if (init) {
    cudaError_t e = cudaMemcpyAsync(cent, init, (size_t)H * C * D * sizeof(float),
                                    cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  } else {
    k_init_deterministic<T, D><<<dim3(C, H), 128, 0, st>>>(X, N, C, cent); note_launch();
  }
  auto do_assign = [&]() -> cudaError_t {
    if (use_tc) return kmeans_assign_tc(X, H, N, D, C, cent, labels, tc_ws, st);
    k_assign_exact<T, D><<<dim3((N + 63) / 64, H), 64, 0, st>>>(X, cent, N, C, labels); note_launch();
    return cudaGetLastError();
  };
  if (use_tc) {
    cudaError_t e = kmeans_tc_prepare_rows(X, H, N, D, tc_ws, st);
    if (e != cudaSuccess) return e;
  }
  for (int it = 0; it < iters; ++it) {
    cudaError_t e = do_assign();
    if (e != cudaSuccess) return e;
    e = cluster_sort(labels, H, N, C, counts, offsets, perm, sort_ws, st);
    if (e != cudaSuccess) return e;
    k_update<T, D><<<dim3(C, H), 256, 0, st>>>(X, perm, offsets, N, C, cent); note_launch();
  }
  cudaError_t e = do_assign();
  if (e != cudaSuccess) return e;
  return cluster_sort(labels, H, N, C, counts, offsets, perm, sort_ws, st);
}

}  // namespace

size_t kmeans_ws_bytes(int H, int N, int d, int C) {
  Carve cv(nullptr);
  cv.take<int32_t>((size_t)H * N);        // perm
  cv.take<int32_t>((size_t)H * (C + 1));  // offsets
  cv.take<char>(sort_ws_bytes(H, N, C));
  cv.take<char>(kmeans_tc_ws_bytes(H, N, d, C));
  return cv.used();
}

cudaError_t kmeans_run(const void* X, int dtype, int H, int N, int d, int C, int iters,
                       const float* init, float* cent, int32_t* labels, int32_t* counts,
                       int32_t* offsets_out, int32_t* perm_out, void* ws, cudaStream_t st) {
  Carve cv(ws);
  int32_t* perm = cv.take<int32_t>((size_t)H * N);
  int32_t* offs = cv.take<int32_t>((size_t)H * (C + 1));
  char* sws = cv.take<char>(sort_ws_bytes(H, N, C));
  void* tws = cv.take<char>(kmeans_tc_ws_bytes(H, N, d, C));
  if (perm_out) perm = perm_out;
  if (offsets_out) offs = offsets_out;
  if (dtype == DT_BF16) {
    const bf16* x = static_cast<const bf16*>(X);
    const bool tc = kmeans_tc_usable(X, N, d, C);
    if (d == 128) return run_t<bf16, 128>(x, H, N, C, iters, init, cent, labels, counts, offs, perm, sws, tws, tc, st);
    return run_t<bf16, 64>(x, H, N, C, iters, init, cent, labels, counts, offs, perm, sws, tws, tc, st);
  }
  const float* x = static_cast<const float*>(X);
  if (d == 128) return run_t<float, 128>(x, H, N, C, iters, init, cent, labels, counts, offs, perm, sws, tws, false, st);
  return run_t<float, 64>(x, H, N, C, iters, init, cent, labels, counts, offs, perm, sws, tws, false, st);
}

}  // namespace svg
