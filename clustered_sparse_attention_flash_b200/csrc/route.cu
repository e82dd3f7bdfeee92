// Error-aware routing under the density budget rho (SVG-EAR review, step (3);
// gist.science summary 2.B "Selektion"): per query cluster, key clusters are
// ordered by error-to-cost ratio (descending, smaller index first on ties)
// and the longest prefix whose key count fits floor(rho * N_k) is routed to
// exact attention.  One block per (query cluster, head): bitonic sort of
// 64-bit keys in shared memory, then a block scan of the cluster sizes.
//
// Global budget (the knapsack form over all blocks of a head): every block
// (a, c) with |q_a|, |k_c| > 0 costs |q_a||k_c| pairs and is ranked by its
// unshifted ratio, compared as logf(E) + 2 M_a; the longest prefix of that
// order (equal keys: smaller a * Ck + c first) within floor(rho Nq Nk) pairs
// is routed.  k_route_global finds the cut with a four-pass radix select
// on the 32-bit ordered key (cost histograms per 8-bit digit), resolves the
// items equal to the cut key in index order with a chunked block scan, and
// leaves each row's routed key count in n_sel.  The order restricted to one
// row is that row's order under the same key, so k_route with that count as
// the row's budget routes exactly the selected clusters.
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

// Key of the global order: the unshifted ratio as logf(E) + 2 M (E = 0,
// negative rounding or NaN count as 0, i.e. -inf), mapped to uint32.
__device__ __forceinline__ uint32_t global_key(float e, float m) {
  if (!(e >= 0.f)) e = 0.f;
  return ordered(logf(e) + 2.f * m);
}

// row_budget (global mode) aliases n_sel: each block reads its row's entry
// before the barriers that precede its own write of n_sel.
__global__ void __launch_bounds__(1024) k_route(const float* __restrict__ E, const int32_t* __restrict__ k_counts,
                                                const int32_t* __restrict__ q_counts, int Cq, int Ck,
                                                long long budget, const float* __restrict__ M,
                                                const int32_t* row_budget, uint8_t* __restrict__ mask,
                                                int32_t* __restrict__ sel, int32_t* n_sel,
                                                unsigned long long* __restrict__ exec_pairs) {
  __shared__ unsigned long long key[kMaxCk];
  __shared__ long long wsum[32];
  __shared__ long long wmax[32];
  __shared__ int cnt_ok[32];
  const int h = blockIdx.y, a = blockIdx.x, T = blockDim.x;
  if (row_budget) budget = row_budget[(size_t)h * Cq + a];
  const float* Er = E + ((size_t)h * Cq + a) * Ck;
  const int32_t* kc = k_counts + (size_t)h * Ck;
  int P = 1;
  while (P < Ck) P <<= 1;
  for (int i = threadIdx.x; i < P; i += T) {
    unsigned long long k = ~0ull;  // padding and empty clusters sort last
    if (i < Ck && kc[i] > 0) {
      float e = Er[i];
      if (!(e >= 0.f)) e = 0.f;       // NaN / negative rounding -> 0
      const uint32_t hi = 0xFFFFFFFFu - (M ? global_key(e, M[(size_t)h * Cq + a]) : ordered(e));  // descending ratio
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

// Block-wide inclusive scan of one long long per thread (blockDim.x a
// multiple of 32, at most 1024); every thread must call it.
__device__ long long block_incl_scan(long long v, long long* wsum, long long* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int o = 1; o < 32; o <<= 1) {
    const long long u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) wsum[w] = v;
  __syncthreads();
  if (w == 0) {
    long long t = lane < nw ? wsum[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    wsum[lane] = t;
  }
  __syncthreads();
  const long long r = v + (w > 0 ? wsum[w - 1] : 0);
  *total = wsum[nw - 1];
  __syncthreads();
  return r;
}

// One block per head: per-row routed key counts of the global-budget order
// (written to row_budget [H, Cq]).
__global__ void __launch_bounds__(1024) k_route_global(const float* __restrict__ E, const float* __restrict__ M,
                                                       const int32_t* __restrict__ k_counts,
                                                       const int32_t* __restrict__ q_counts, int Cq, int Ck,
                                                       long long budget, int32_t* __restrict__ row_budget) {
  __shared__ unsigned long long hist[256];
  __shared__ long long wsum[32];
  __shared__ uint32_t s_prefix, s_bits;
  __shared__ long long s_rem;
  __shared__ int s_all;
  const int h = blockIdx.x, T = blockDim.x, tid = threadIdx.x;
  const float* Eh = E + (size_t)h * Cq * Ck;
  const float* Mh = M + (size_t)h * Cq;
  const int32_t* kc = k_counts + (size_t)h * Ck;
  const int32_t* qc = q_counts + (size_t)h * Cq;
  int32_t* rb = row_budget + (size_t)h * Cq;
  const long long n = (long long)Cq * Ck;
  for (int a = tid; a < Cq; a += T) rb[a] = 0;
  if (tid == 0) { s_prefix = 0u; s_bits = 0u; s_rem = budget; s_all = 0; }
  __syncthreads();
  // radix select, most significant digit first: the digit whose items make
  // the running cost (higher keys first) pass the remaining budget
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += T) hist[i] = 0ull;
    __syncthreads();
    const uint32_t pre = s_prefix, bits = s_bits;
    for (long long i = tid; i < n; i += T) {
      const int a = (int)(i / Ck), c = (int)(i - (long long)a * Ck);
      const int q = qc[a], k = kc[c];
      if (q > 0 && k > 0) {
        const uint32_t u = global_key(Eh[i], Mh[a]);
        if ((u & bits) == pre) atomicAdd(&hist[(u >> shift) & 255u], (unsigned long long)q * (unsigned long long)k);
      }
    }
    __syncthreads();
    if (tid == 0) {
      const unsigned long long rem = (unsigned long long)s_rem;
      unsigned long long cum = 0ull;
      int b = -1;
      for (int bin = 255; bin >= 0; --bin) {
        if (cum + hist[bin] > rem) { b = bin; break; }
        cum += hist[bin];
      }
      if (b < 0) {
        s_all = 1;  // every item fits (first pass only: later passes split a bin that did not)
      } else {
        s_rem = (long long)(rem - cum);
        s_prefix = pre | ((uint32_t)b << shift);
        s_bits = bits | (0xFFu << shift);
      }
    }
    __syncthreads();
    if (s_all) break;
  }
  const bool all = s_all != 0;
  const uint32_t t = s_prefix;
  const long long rem = s_rem;
  // items above the cut key (or all of them)
  for (long long i = tid; i < n; i += T) {
    const int a = (int)(i / Ck), c = (int)(i - (long long)a * Ck);
    const int q = qc[a], k = kc[c];
    if (q > 0 && k > 0 && (all || global_key(Eh[i], Mh[a]) > t)) atomicAdd(&rb[a], k);
  }
  if (all) return;
  // items equal to the cut key, in index order, while the running cost fits
  long long carry = 0;
  for (long long base = 0; base < n; base += T) {
    const long long i = base + tid;
    long long cost = 0;
    int a = 0, k = 0;
    if (i < n) {
      a = (int)(i / Ck);
      const int c = (int)(i - (long long)a * Ck);
      const int q = qc[a];
      k = kc[c];
      if (q > 0 && k > 0 && global_key(Eh[i], Mh[a]) == t) cost = (long long)q * k;
    }
    long long total = 0;
    const long long incl = block_incl_scan(cost, wsum, &total);
    if (cost > 0 && carry + incl <= rem) atomicAdd(&rb[a], k);
    carry += total;
    if (carry > rem) break;  // uniform: every thread holds the same carry
  }
}

}  // namespace

long long route_global_budget(float rho, long long Nq, long long Nk) {
  // floor(rho * Nq * Nk) exactly: rho = f 2^ex with f in [0.5, 1), so
  // rho = m 2^(ex - 24) for the integer m = f 2^24 < 2^24
  if (!(rho > 0.f) || Nq <= 0 || Nk <= 0) return 0;
  int ex = 0;
  const float f = frexpf(rho, &ex);
  const unsigned long long m = (unsigned long long)ldexpf(f, 24);
  const unsigned __int128 prod = (unsigned __int128)m * (unsigned long long)Nq * (unsigned long long)Nk;
  const int sh = 24 - ex;
  if (sh >= 128) return 0;
  if (sh <= 0) return (long long)(prod << (-sh));
  return (long long)(prod >> sh);
}

cudaError_t route_run(const float* E, const int32_t* k_counts, const int32_t* q_counts, int H,
                      int Nk, int Cq, int Ck, float rho, uint8_t* mask, int32_t* sel,
                      int32_t* n_sel, int64_t* exec_pairs, cudaStream_t st, const float* M_global,
                      int Nq) {
  if (Ck > kMaxCk) return cudaErrorInvalidValue;
  const long long budget = (long long)floor((double)rho * (double)Nk);
  cudaError_t e = cudaMemsetAsync(exec_pairs, 0, (size_t)H * sizeof(int64_t), st);
  if (e != cudaSuccess) return e;
  if (M_global) {
    k_route_global<<<H, 1024, 0, st>>>(E, M_global, k_counts, q_counts, Cq, Ck,
                                       route_global_budget(rho, Nq, Nk), n_sel);
    note_launch();
  }
  int T = 32;
  while (T < Ck && T < 1024) T <<= 1;
  k_route<<<dim3(Cq, H), T, 0, st>>>(E, k_counts, q_counts, Cq, Ck, budget, M_global,
                                     M_global ? n_sel : nullptr, mask, sel, n_sel,
                                     reinterpret_cast<unsigned long long*>(exec_pairs)); note_launch();
  return cudaGetLastError();
}

}  // namespace svg
