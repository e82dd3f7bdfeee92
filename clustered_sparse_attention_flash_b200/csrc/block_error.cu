// Value-aware block error with the query-centroid proxy (SVG-EAR review,
// step (2); gist.science summary 2.B, "lightweight probe", O(C_q N_k d)).
//
//   eps^2(a,j) = || A vbar_c - B_j v_j ||^2,  A = e^{s qbar_a.kbar_c - M_a},
//                                              B_j = e^{s qbar_a.k_j - M_a}
//   E[a,c]     = (1/|k_c|) sum_{j in c} eps^2(a,j)
//
// The norm is expanded with per-key terms precomputed by the permute step
// (s1 = ||vbar-v||^2, s2 = (vbar-v).v, s3 = ||v||^2) around A:
//   A vbar - B v = A (vbar - v) + (A - B) v,  A - B = -A expm1(u),
//   u = s qbar_a.(k_j - kbar_c),
//   eps^2 = A^2 s1 + 2 A (A-B) s2 + (A-B)^2 s3.
// This is exact algebra; the form keeps full relative accuracy when the
// cluster is tight (u -> 0, v -> vbar) where a^2|vbar|^2 - 2ab vbar.v + b^2|v|^2
// would cancel.  Logits never leave registers.
//
// Two ablation signals share the launch sequence: the value-agnostic error
// (s1, s2, s3) = (0, 0, 1), i.e. eps^2 = (A - B)^2, and the estimated
// attention mass of each key cluster, |k_c| A normalised over the row, which
// needs only the centroid logits.
#include <mutex>

#include "../../include/svgear.h"
#include "common.cuh"
#include "internal.h"

namespace svg {

namespace {

// L[a][c] = s qbar_a.kbar_c (float64 dot, stored float32) for a tile of
// 32 query centroids x 32 key centroids per block (both staged in shared
// memory); each thread owns one query centroid and four key centroids.
template <int D>
__global__ void __launch_bounds__(256) k_centroid_logits(const float* __restrict__ Qbar,
                                                         const float* __restrict__ Kbar, int Cq, int Ck,
                                                         float scale, float* __restrict__ L) {
  __shared__ float qs[32][D + 1];
  __shared__ float ks[32][D + 1];
  const int h = blockIdx.z, a0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int e = threadIdx.x; e < 32 * D; e += blockDim.x) {
    const int r = e / D, t = e % D;
    qs[r][t] = a0 + r < Cq ? Qbar[((size_t)h * Cq + a0 + r) * D + t] : 0.f;
    ks[r][t] = c0 + r < Ck ? Kbar[((size_t)h * Ck + c0 + r) * D + t] : 0.f;
  }
  __syncthreads();
  const int ar = threadIdx.x & 31, cg = threadIdx.x >> 5;  // query row, group of 4 key rows
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
  for (int t = 0; t < D; ++t) {
    const double q = qs[ar][t];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = fma(q, (double)ks[cg * 4 + i][t], acc[i]);
  }
  const int a = a0 + ar;
  if (a < Cq)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = c0 + cg * 4 + i;
      if (c < Ck) L[((size_t)h * Cq + a) * Ck + c] = (float)(acc[i] * (double)scale);
    }
}

// M[a] = max over non-empty c of L[a][c]: one warp per (a, head).
__global__ void __launch_bounds__(256) k_logit_max(const float* __restrict__ L, const int32_t* __restrict__ k_off,
                                                   int H, int Cq, int Ck, float* __restrict__ M) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= H * Cq) return;
  const int h = row / Cq;
  const int32_t* off = k_off + (size_t)h * (Ck + 1);
  const float* Lr = L + (size_t)row * Ck;
  float mx = -INFINITY;
  for (int c = lane; c < Ck; c += 32)
    if (off[c + 1] > off[c]) mx = fmaxf(mx, Lr[c]);
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) M[row] = mx;
}

// Estimated attention mass: E[a][c] = |k_c| e^{L[a][c] - M[a]} / row sum over
// the non-empty clusters (0 for empty ones).  One warp per (a, head); the row
// sum is accumulated in float64.
__global__ void __launch_bounds__(256) k_block_mass(const float* __restrict__ L, const float* __restrict__ M,
                                                    const int32_t* __restrict__ k_off, int H, int Cq, int Ck,
                                                    float* __restrict__ E) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= H * Cq) return;
  const int h = row / Cq;
  const int32_t* off = k_off + (size_t)h * (Ck + 1);
  const float* Lr = L + (size_t)row * Ck;
  float* Er = E + (size_t)row * Ck;
  const float m = M[row];
  double sum = 0.0;
  for (int c = lane; c < Ck; c += 32) {
    const int n = off[c + 1] - off[c];
    const float w = n > 0 ? (float)n * expf(Lr[c] - m) : 0.f;
    Er[c] = w;
    sum += (double)w;
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = (float)(1.0 / sum);  // sum >= 1: the maximising cluster has n >= 1, e^0
  for (int c = lane; c < Ck; c += 32) Er[c] *= inv;
}

// One block per (key cluster c, head); thread t owns query cluster a = t (+128k).
// Keys of c stream through shared memory as k_j - kbar_c.
template <typename T, int D>
__global__ void __launch_bounds__(128) k_block_error(const float* __restrict__ Qbar,
                                                     const float* __restrict__ Kbar,
                                                     const T* __restrict__ Kp,
                                                     const int32_t* __restrict__ k_off,
                                                     const float* __restrict__ ks, const float* __restrict__ L,
                                                     const float* __restrict__ M, int H, int Nk, int Cq,
                                                     int Ck, float scale, int value_agnostic,
                                                     float* __restrict__ E) {
  constexpr int KT = 32;
  __shared__ __align__(16) float dk[KT][D];
  __shared__ float sc[3][KT];
  __shared__ float kb[D];
  const int h = blockIdx.y, c = blockIdx.x;
  const int beg = k_off[(size_t)h * (Ck + 1) + c], end = k_off[(size_t)h * (Ck + 1) + c + 1];
  if (beg >= end) {
    for (int a = threadIdx.x; a < Cq; a += blockDim.x) E[((size_t)h * Cq + a) * Ck + c] = 0.f;
    return;
  }
  for (int t = threadIdx.x; t < D; t += blockDim.x) kb[t] = Kbar[((size_t)h * Ck + c) * D + t];
  const size_t plane = (size_t)H * Nk;
  const T* Kh = Kp + (size_t)h * Nk * D;
  for (int a0 = 0; a0 < Cq; a0 += blockDim.x) {
    const int a = a0 + threadIdx.x;
    const bool act = a < Cq;
    float q[D];
    float A = 0.f;
    if (act) {
      const float* qb = Qbar + ((size_t)h * Cq + a) * D;
#pragma unroll
      for (int t = 0; t < D; t += 4) {
        float4 v = ld4(qb + t);
        q[t] = v.x * scale; q[t + 1] = v.y * scale; q[t + 2] = v.z * scale; q[t + 3] = v.w * scale;
      }
      A = expf(L[((size_t)h * Cq + a) * Ck + c] - M[(size_t)h * Cq + a]);
    } else {
#pragma unroll
      for (int t = 0; t < D; ++t) q[t] = 0.f;
    }
    double acc = 0.0;
    for (int j0 = beg; j0 < end; j0 += KT) {
      const int nk = min(KT, end - j0);
      __syncthreads();
      for (int e = threadIdx.x; e < nk * D; e += blockDim.x) {
        const int r = e / D, t = e % D;
        dk[r][t] = to_f(Kh[(size_t)(j0 + r) * D + t]) - kb[t];
      }
      for (int e = threadIdx.x; e < 3 * nk; e += blockDim.x) {
        const int w = e / nk, r = e % nk;
        sc[w][r] = value_agnostic ? (w == 2 ? 1.f : 0.f) : ks[w * plane + (size_t)h * Nk + j0 + r];
      }
      __syncthreads();
      if (act) {
        for (int r = 0; r < nk; ++r) {
          float u = 0.f;
#pragma unroll
          for (int t = 0; t < D; t += 4) {
            const float4 k4 = *reinterpret_cast<const float4*>(&dk[r][t]);
            u = fmaf(q[t], k4.x, u); u = fmaf(q[t + 1], k4.y, u);
            u = fmaf(q[t + 2], k4.z, u); u = fmaf(q[t + 3], k4.w, u);
          }
          const float amb = -A * expm1f(u);
          float e2 = A * A * sc[0][r] + 2.f * A * amb * sc[1][r] + amb * amb * sc[2][r];
          acc += (double)fmaxf(e2, 0.f);
        }
      }
    }
    if (act) E[((size_t)h * Cq + a) * Ck + c] = (float)(acc / (double)(end - beg));
  }
}

}  // namespace

size_t block_error_ws_bytes(int H, int Cq, int Ck, int d, int dtype) {
  size_t n = align_up((size_t)H * Cq * Ck * sizeof(float), 256);
  // reserved whenever the shape allows the tensor-core kernel (no device query here)
  if (block_error_tc_shape_ok(dtype, d, Cq)) n += align_up(block_error_tc_ws_bytes(H, d), 256);
  return n;
}

cudaError_t block_error_run(const float* Qbar, const float* Kbar, const float* Vbar,
                            const void* Kp, const void* Vp, const int32_t* k_off,
                            const float* key_scalars, int dtype, int H, int Nk, int d, int Cq,
                            int Ck, float scale, float* E, float* M, void* ws, cudaStream_t st,
                            int router, bool allow_tc) {
  (void)Vbar; (void)Vp;  // their contribution enters through key_scalars
  float* L = static_cast<float*>(ws);
  const dim3 lg((Ck + 31) / 32, (Cq + 31) / 32, H);
  if (d == 128) { k_centroid_logits<128><<<lg, 256, 0, st>>>(Qbar, Kbar, Cq, Ck, scale, L); note_launch(); }
  else { k_centroid_logits<64><<<lg, 256, 0, st>>>(Qbar, Kbar, Cq, Ck, scale, L); note_launch(); }
  k_logit_max<<<(H * Cq + 7) / 8, 256, 0, st>>>(L, k_off, H, Cq, Ck, M); note_launch();
  if (router == SVGEAR_ROUTE_MASS) {
    k_block_mass<<<(H * Cq + 7) / 8, 256, 0, st>>>(L, M, k_off, H, Cq, Ck, E); note_launch();
    return cudaGetLastError();
  }
  const int vagn = router == SVGEAR_ROUTE_ERROR_NOV;
  if (allow_tc && block_error_tc_supported(dtype, d, Cq, Nk)) {
    char* qhl = static_cast<char*>(ws) + align_up((size_t)H * Cq * Ck * sizeof(float), 256);
    return block_error_tc_run(Qbar, Kp, k_off, key_scalars, L, M, H, Nk, d, Cq, Ck, scale, E, qhl, st,
                              vagn != 0);
  }
  dim3 g(Ck, H);
  if (dtype == DT_BF16) {
    if (d == 128) { k_block_error<bf16, 128><<<g, 128, 0, st>>>(Qbar, Kbar, static_cast<const bf16*>(Kp), k_off, key_scalars, L, M, H, Nk, Cq, Ck, scale, vagn, E); note_launch(); }
    else { k_block_error<bf16, 64><<<g, 128, 0, st>>>(Qbar, Kbar, static_cast<const bf16*>(Kp), k_off, key_scalars, L, M, H, Nk, Cq, Ck, scale, vagn, E); note_launch(); }
  } else {
    if (d == 128) { k_block_error<float, 128><<<g, 128, 0, st>>>(Qbar, Kbar, static_cast<const float*>(Kp), k_off, key_scalars, L, M, H, Nk, Cq, Ck, scale, vagn, E); note_launch(); }
    else { k_block_error<float, 64><<<g, 128, 0, st>>>(Qbar, Kbar, static_cast<const float*>(Kp), k_off, key_scalars, L, M, H, Nk, Cq, Ck, scale, vagn, E); note_launch(); }
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the centroid-logit scratch lives in a file-scope
// device array instead of a caller workspace.  Every GPU that loads the
// library holds this array until the process exits.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 21;  // 8 MiB: H*Cq*Ck <= 2,097,152
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the symbol name is only a host-side handle).
static float* noalloc_scratch(cudaError_t* err) {
  static std::mutex mu;
  static float* cache[64] = {nullptr};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) { *err = cudaErrorInvalidDevice; return nullptr; }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    cache[dev] = static_cast<float*>(ptr);
  }
  return cache[dev];
}

}  // namespace svg

extern "C" int svgear_block_error_noalloc(const float* Qbar, const float* Kbar, const float* Vbar,
                                          const void* Kp, const void* Vp, const int32_t* k_off,
                                          const float* key_scalars, const svgear_params* p, float* E,
                                          float* M, void* stream) {
  using namespace svg;
  const int r = params_status(p);
  if (r != SVGEAR_OK) return r;
  if (!Qbar || !Kbar || !k_off || !E || !M) return SVGEAR_ERR_INVALID;
  if (p->router != SVGEAR_ROUTE_MASS && !Kp) return SVGEAR_ERR_INVALID;
  if (p->router == SVGEAR_ROUTE_ERROR && !key_scalars) return SVGEAR_ERR_INVALID;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(Qbar) | reinterpret_cast<uintptr_t>(Kbar) |
                        reinterpret_cast<uintptr_t>(Kp);
  if (mis & 15u) return SVGEAR_ERR_INVALID;
  if ((size_t)p->H * (size_t)p->Cq * (size_t)p->Ck > kNoAllocScratchFloats) return SVGEAR_ERR_WORKSPACE;
  cudaError_t e = cudaSuccess;
  float* L = noalloc_scratch(&e);
  if (!L) return SVGEAR_ERR_CUDA;
  const float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
  // the static scratch holds the centroid logits only: CUDA-core block error
  e = block_error_run(Qbar, Kbar, Vbar, Kp, Vp, k_off, key_scalars, p->dtype, p->H, p->Nk, p->d, p->Cq,
                      p->Ck, scale, E, M, L, static_cast<cudaStream_t>(stream), p->router, false);
  return e == cudaSuccess ? SVGEAR_OK : SVGEAR_ERR_CUDA;
}
