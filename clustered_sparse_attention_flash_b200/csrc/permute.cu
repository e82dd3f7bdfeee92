// Token reordering so that every cluster is contiguous (SVG-EAR review,
// step (1)), plus the value centroids and per-key terms the value-aware error
// estimate uses (review step (2); gist.science summary 2.B).
// Both kernels are HBM-bound row copies / row reductions.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace svg {

namespace {

// Xp[h][n] = X[h][perm[h][n]], 16-byte chunks, grid-stride.
__global__ void k_gather(const uint4* __restrict__ X, const int32_t* __restrict__ perm, int H, int N,
                         int cpr, uint4* __restrict__ Xp) {
  const long long total = (long long)H * N * cpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / cpr;
    const int ch = (int)(e - row * cpr);
    const int h = (int)(row / N);
    const int src = perm[row];
    Xp[e] = X[((long long)h * N + src) * cpr + ch];
  }
}

// One block per (cluster, head): vbar = float64 mean of the cluster's rows
// (stored as float32), then per row (vbar - v)^2, (vbar - v).v, v.v.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_value_stats(const T* __restrict__ Vp, const int32_t* __restrict__ off,
                                                     int H, int N, int C, float* __restrict__ Vbar,
                                                     float* __restrict__ ks) {
  constexpr int PER = D / 32, NW = 8;
  __shared__ double red[NW][D];
  __shared__ float vb[D];
  const int h = blockIdx.y, c = blockIdx.x;
  const int beg = off[(size_t)h * (C + 1) + c], end = off[(size_t)h * (C + 1) + c + 1];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* Vh = Vp + (size_t)h * N * D + lane * PER;
  double acc[PER];
#pragma unroll
  for (int t = 0; t < PER; ++t) acc[t] = 0.0;
  // eight rows per warp in flight; each batch is summed in float32 (fixed
  // pairwise order) and added to the float64 accumulators once
  for (int r0 = beg + w; r0 < end; r0 += 8 * NW) {
    float x[8][PER];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const bool in = r0 + u * NW < end;
      if constexpr (PER == 4) {
        const float4 v = in ? ld4(Vh + (size_t)(r0 + u * NW) * D) : make_float4(0.f, 0.f, 0.f, 0.f);
        x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
      } else {
        const float2 v = in ? ld2(Vh + (size_t)(r0 + u * NW) * D) : make_float2(0.f, 0.f);
        x[u][0] = v.x; x[u][1] = v.y;
      }
    }
#pragma unroll
    for (int t = 0; t < PER; ++t)
      acc[t] += (double)(((x[0][t] + x[1][t]) + (x[2][t] + x[3][t])) + ((x[4][t] + x[5][t]) + (x[6][t] + x[7][t])));
  }
#pragma unroll
  for (int t = 0; t < PER; ++t) red[w][lane * PER + t] = acc[t];
  __syncthreads();
  const double inv = end > beg ? 1.0 / (double)(end - beg) : 0.0;
  for (int t = threadIdx.x; t < D; t += blockDim.x) {
    double s = 0.0;
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) s += red[ww][t];
    const float m = (float)(s * inv);
    vb[t] = m;
    if (Vbar) Vbar[((size_t)h * C + c) * D + t] = m;
  }
  __syncthreads();
  if (!ks) return;
  float mv[PER];
#pragma unroll
  for (int t = 0; t < PER; ++t) mv[t] = vb[lane * PER + t];
  const size_t plane = (size_t)H * N;
  // per-key scalars, four rows per warp in flight with independent reductions
  constexpr int RB = 4;
  for (int r0 = beg + w; r0 < end; r0 += RB * NW) {
    float s1[RB], s2[RB], s3[RB];
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      const int r = r0 + u * NW;
      float v[PER];
      if constexpr (PER == 4) {
        const float4 q = r < end ? ld4(Vh + (size_t)r * D) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
      } else {
        const float2 q = r < end ? ld2(Vh + (size_t)r * D) : make_float2(0.f, 0.f);
        v[0] = q.x; v[1] = q.y;
      }
      s1[u] = 0.f; s2[u] = 0.f; s3[u] = 0.f;
#pragma unroll
      for (int t = 0; t < PER; ++t) {
        const float dv = mv[t] - v[t];
        s1[u] = fmaf(dv, dv, s1[u]);
        s2[u] = fmaf(dv, v[t], s2[u]);
        s3[u] = fmaf(v[t], v[t], s3[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        s1[u] += __shfl_xor_sync(0xffffffffu, s1[u], o);
        s2[u] += __shfl_xor_sync(0xffffffffu, s2[u], o);
        s3[u] += __shfl_xor_sync(0xffffffffu, s3[u], o);
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int r = r0 + u * NW;
        if (r < end) {
          const size_t i = (size_t)h * N + r;
          ks[i] = s1[u];
          ks[plane + i] = s2[u];
          ks[2 * plane + i] = s3[u];
        }
      }
    }
  }
}

}  // namespace

cudaError_t gather_rows(const void* X, int dtype, const int32_t* perm, int H, int N, int d,
                        void* Xp, cudaStream_t st) {
  const int esz = dtype == DT_BF16 ? 2 : 4;
  const int cpr = d * esz / 16;
  const long long total = (long long)H * N * cpr;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 148LL * 16);
  k_gather<<<(int)std::max<long long>(blocks, 1), threads, 0, st>>>(
      static_cast<const uint4*>(X), perm, H, N, cpr, static_cast<uint4*>(Xp)); note_launch();
  return cudaGetLastError();
}

cudaError_t value_stats(const void* Vp, int dtype, const int32_t* off, int H, int N, int d, int C,
                        float* Vbar, float* key_scalars, cudaStream_t st) {
  dim3 g(C, H);
  if (dtype == DT_BF16) {
    if (d == 128) { k_value_stats<bf16, 128><<<g, 256, 0, st>>>(static_cast<const bf16*>(Vp), off, H, N, C, Vbar, key_scalars); note_launch(); }
    else { k_value_stats<bf16, 64><<<g, 256, 0, st>>>(static_cast<const bf16*>(Vp), off, H, N, C, Vbar, key_scalars); note_launch(); }
  } else {
    if (d == 128) { k_value_stats<float, 128><<<g, 256, 0, st>>>(static_cast<const float*>(Vp), off, H, N, C, Vbar, key_scalars); note_launch(); }
    else { k_value_stats<float, 64><<<g, 256, 0, st>>>(static_cast<const float*>(Vp), off, H, N, C, Vbar, key_scalars); note_launch(); }
  }
  return cudaGetLastError();
}

}  // namespace svg
