// Error-aware routing under the density budget rho (SVG-EAR review, step (3);
// gist.science summary 2.B "Selektion"): per query cluster, key clusters are
// ordered by error-to-cost ratio (descending, smaller index first on ties)
// and the longest prefix whose key count fits floor(rho * N_k) is routed to
// exact attention.  One block per (query cluster, head): bitonic sort of
// 64-bit keys in shared memory, then a block scan of the cluster sizes.
#include "common.cuh"
#include "internal.h"

namespace svg {

namespace {

constexpr int kMaxCk = 4096;

__device__ __forceinline__ uint32_t ordered(float x) {
  // monotone map float -> uint32 for non-negative and negative values alike
  uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(1024) k_route(const float* __restrict__ E, const int32_t* __restrict__ k_counts,
                                                const int32_t* __restrict__ q_counts, int Cq, int Ck,
                                                long long budget, uint8_t* __restrict__ mask,
                                                int32_t* __restrict__ sel, int32_t* __restrict__ n_sel,
                                                unsigned long long* __restrict__ exec_pairs) {
  __shared__ unsigned long long key[kMaxCk];
  __shared__ long long wsum[32];
  __shared__ long long wmax[32];
  __shared__ int cnt_ok[32];
  const int h = blockIdx.y, a = blockIdx.x, T = blockDim.x;
  const float* Er = E + ((size_t)h * Cq + a) * Ck;
  const int32_t* kc = k_counts + (size_t)h * Ck;
  int P = 1;
  while (P < Ck) P <<= 1;
  for (int i = threadIdx.x; i < P; i += T) {
    unsigned long long k = ~0ull;  // padding and empty clusters sort last
    if (i < Ck && kc[i] > 0) {
      float e = Er[i];
      if (!(e >= 0.f)) e = 0.f;       // NaN / negative rounding -> 0
      const uint32_t hi = 0xFFFFFFFFu - ordered(e);  // descending ratio
      k = ((unsigned long long)hi << 32) | (uint32_t)i;  // then ascending index
    }
    key[i] = k;
  }
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P; i += T) {
        const int l = i ^ j;
        if (l > i) {
          const unsigned long long x = key[i], y = key[l];
          const bool up = (i & k) == 0;
          if ((x > y) == up) { key[i] = y; key[l] = x; }
        }
      }
      __syncthreads();
    }
  }
  // inclusive scan of the sizes in routing order (blocked per thread)
  const int per = (Ck + T - 1) / T;
  const int beg = threadIdx.x * per, end = min(Ck, beg + per);
  long long s = 0;
  for (int i = beg; i < end; ++i) {
    const unsigned long long k = key[i];
    s += (k == ~0ull) ? 0 : kc[(uint32_t)k];
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  long long v = s;
  for (int o = 1; o < 32; o <<= 1) {
    long long u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) wsum[w] = v;
  __syncthreads();
  if (w == 0) {
    long long t = (lane < (T >> 5)) ? wsum[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      long long u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    wsum[lane] = t;
  }
  __syncthreads();
  long long run = v - s + (w > 0 ? wsum[w - 1] : 0);
  int ok = 0;
  long long fit = 0;  // largest running total that still fits
  for (int i = beg; i < end; ++i) {
    const unsigned long long k = key[i];
    const bool valid = k != ~0ull;
    run += valid ? kc[(uint32_t)k] : 0;
    if (valid && run <= budget) { ++ok; fit = run; }
  }
  // the prefix rule: running totals are non-decreasing, so the routed set is
  // the first n entries of the order
  for (int o = 16; o > 0; o >>= 1) {
    ok += __shfl_xor_sync(0xffffffffu, ok, o);
    fit = max(fit, __shfl_xor_sync(0xffffffffu, fit, o));
  }
  if (lane == 0) { cnt_ok[w] = ok; wmax[w] = fit; }
  __syncthreads();
  int n = 0;
  long long routed = 0;
  for (int ww = 0; ww < (T >> 5); ++ww) { n += cnt_ok[ww]; routed = max(routed, wmax[ww]); }
  uint8_t* mr = mask + ((size_t)h * Cq + a) * Ck;
  int32_t* sr = sel + ((size_t)h * Cq + a) * Ck;
  for (int i = threadIdx.x; i < Ck; i += T) mr[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += T) {
    const int c = (int)(uint32_t)key[i];
    mr[c] = 1;
    sr[i] = c;
  }
  if (threadIdx.x == 0) {
    n_sel[(size_t)h * Cq + a] = n;
    const long long pairs = routed * (long long)q_counts[(size_t)h * Cq + a];
    if (pairs) atomicAdd(exec_pairs + h, (unsigned long long)pairs);
  }
}

}  // namespace

cudaError_t route_run(const float* E, const int32_t* k_counts, const int32_t* q_counts, int H,
                      int Nk, int Cq, int Ck, float rho, uint8_t* mask, int32_t* sel,
                      int32_t* n_sel, int64_t* exec_pairs, cudaStream_t st) {
  if (Ck > kMaxCk) return cudaErrorInvalidValue;
  const long long budget = (long long)floor((double)rho * (double)Nk);
  cudaError_t e = cudaMemsetAsync(exec_pairs, 0, (size_t)H * sizeof(int64_t), st);
  if (e != cudaSuccess) return e;
  int T = 32;
  while (T < Ck && T < 1024) T <<= 1;
  k_route<<<dim3(Cq, H), T, 0, st>>>(E, k_counts, q_counts, Cq, Ck, budget, mask, sel, n_sel,
                                     reinterpret_cast<unsigned long long*>(exec_pairs)); note_launch();
  return cudaGetLastError();
}

}  // namespace svg
