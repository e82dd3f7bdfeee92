// Tensor-core k-means assignment for bf16 tokens (SVG-EAR review, step (1):
// "Flash k-means" clustering of queries and keys).
//
// For a tile of 128 tokens the scores x . mu_c of every centroid come from
// tcgen05 MMAs (A = token tile, B = bf16-rounded centroids resident in shared
// memory, fp32 accumulators in tensor memory).  The epilogue forms
// s_c = ||mu_c||^2 - 2 x.mu_c and keeps, per token, the running minimum and
// every centroid whose score lies within 2B of it, where B bounds the score
// error: rounding the centroid to bf16 moves x.mu by at most ||x|| ||mu - bf16(mu)||,
// the fp32 accumulation by at most 2^-14 ||x|| ||bf16(mu)||, plus the
// rounding of ||mu||^2 and of the epilogue FMA.  A single survivor is the exact
// argmin; otherwise the token goes on a list that k_refine re-decides with
// float64 distances (smaller index on equal distance), so labels equal the
// exact argmin.
//
// Block of 12 warps: warp 0 allocates tensor memory and issues MMAs, warps 1-3
// copy tiles (cp.async into the 128-byte-swizzled layout), warps 4-7 and 8-11
// are two epilogue warpgroups that take alternate 256-column accumulator slots.
// The epilogue reads each slot twice: a branch-free minimum pass, then a pass
// that lists every column inside the window of the minimum.
#include <algorithm>
#include <cfloat>

#include "internal.h"
#include "kmeans_tc.cuh"
#include "tc_common.cuh"

namespace svg {

namespace {

constexpr int BM = 128;
constexpr int KC = 6;                     // candidate list capacity per token
constexpr int kThreads = 384;
constexpr int kProducers = 96;
constexpr int kCentBytesMax = 128 * 1024;
constexpr int kSlotCols = 256;
constexpr int kRefineInts = 4 + KC;   // h, row, n (-1 = overflow), pad, candidates

__host__ __device__ inline int round16(int x) { return (x + 15) & ~15; }

struct Bounds {  // per head
  float dmax;    // max_c ||mu_c - bf16(mu_c)||
  float mmax;    // max_c ||bf16(mu_c)||
  float nmax;    // max_c ||mu_c||^2
  float pad;
};

// Per head: bf16 copy of the centroids (zero rows up to Cpad), ||mu||^2
// (+inf on padding rows) and the error-bound maxima.
template <int D>
__global__ void __launch_bounds__(256) k_prep_centroids(const float* __restrict__ cent, int C, int Cpad,
                                                        bf16* __restrict__ cb, float* __restrict__ cnorm,
                                                        Bounds* __restrict__ bounds) {
  __shared__ float red[3][8];
  const int h = blockIdx.x, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float dmax = 0.f, mmax = 0.f, nmax = 0.f;
  for (int c = w; c < Cpad; c += 8) {
    double dn = 0.0, mb = 0.0, n2 = 0.0;
    for (int t = lane; t < D; t += 32) {
      const float m = c < C ? cent[((size_t)h * C + c) * D + t] : 0.f;
      const bf16 b = __float2bfloat16_rn(m);
      cb[((size_t)h * Cpad + c) * D + t] = b;
      const double bd = (double)__bfloat162float(b);
      dn += ((double)m - bd) * ((double)m - bd);
      mb += bd * bd;
      n2 += (double)m * (double)m;
    }
    for (int o = 16; o > 0; o >>= 1) {
      dn += __shfl_xor_sync(0xffffffffu, dn, o);
      mb += __shfl_xor_sync(0xffffffffu, mb, o);
      n2 += __shfl_xor_sync(0xffffffffu, n2, o);
    }
    if (lane == 0) cnorm[(size_t)h * Cpad + c] = c < C ? (float)n2 : INFINITY;
    if (c < C) {
      dmax = fmaxf(dmax, (float)sqrt(dn));
      mmax = fmaxf(mmax, (float)sqrt(mb));
      nmax = fmaxf(nmax, (float)n2);
    }
  }
  if (lane == 0) { red[0][w] = dmax; red[1][w] = mmax; red[2][w] = nmax; }
  __syncthreads();
  if (threadIdx.x == 0) {
    Bounds b{0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < 8; ++i) {
      b.dmax = fmaxf(b.dmax, red[0][i]);
      b.mmax = fmaxf(b.mmax, red[1][i]);
      b.nmax = fmaxf(b.nmax, red[2][i]);
    }
    // round the maxima up a little so the bound stays an upper bound
    b.dmax *= 1.0001f; b.mmax *= 1.0001f; b.nmax *= 1.0001f;
    bounds[h] = b;
  }
}

// ||x_i|| per token (float, rounded up slightly), once per k-means call.
template <int D>
__global__ void k_row_norms(const bf16* __restrict__ X, long long rows, float* __restrict__ xn) {
  const long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  float s = 0.f;
  for (int t = lane * 2; t < D; t += 64) {
    const float2 v = ld2(X + r * D + t);
    s = fmaf(v.x, v.x, fmaf(v.y, v.y, s));
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) xn[r] = sqrtf(s) * 1.00001f;
}

// Per-token candidate state: minimum score, number of listed candidates and
// an overflow flag in registers; the list (KC entries per epilogue thread,
// strided by the 256 epilogue threads) in shared memory.
struct Cands {
  float best;
  int n;
  int over;
};

// Drop listed candidates that fell out of the window after `best` decreased.
__device__ __forceinline__ void cand_compact(Cands& st, float W, float* ls, int* lc) {
  int m = 0;
  for (int i = 0; i < min(st.n, KC); ++i) {
    const float v = ls[i * 256];
    if (v <= st.best + W) { ls[m * 256] = v; lc[m * 256] = lc[i * 256]; ++m; }
  }
  st.n = m;
}

__device__ __forceinline__ void cand_push(Cands& st, float s, int c, float* ls, int* lc) {
  if (st.n < KC) { ls[st.n * 256] = s; lc[st.n * 256] = c; }
  else st.over = 1;
  ++st.n;
}

// Pass 1: minimum score over 32 columns (branch-free).
__device__ __forceinline__ float min32(const uint32_t (&v)[32], const float* cn) {
  float m = INFINITY;
#pragma unroll
  for (int q = 0; q < 32; q += 4) {
    const float4 n4 = *reinterpret_cast<const float4*>(cn + q);
    const float a = fmaf(-2.f, __uint_as_float(v[q]), n4.x), b = fmaf(-2.f, __uint_as_float(v[q + 1]), n4.y);
    const float c = fmaf(-2.f, __uint_as_float(v[q + 2]), n4.z), d = fmaf(-2.f, __uint_as_float(v[q + 3]), n4.w);
    m = fminf(m, fminf(fminf(a, b), fminf(c, d)));
  }
  return m;
}

// Pass 2: list every column whose score is within the fixed threshold.
template <int G>
__device__ __forceinline__ void collect(Cands& st, const uint32_t (&v)[G], const float* cn, int cbase, int C,
                                        float thr, float* ls, int* lc) {
#pragma unroll
  for (int q = 0; q < G; ++q) {
    const float sq = fmaf(-2.f, __uint_as_float(v[q]), cn[q]);
    if (sq <= thr && cbase + q < C) cand_push(st, sq, cbase + q, ls, lc);
  }
}

// Rows the tensor-core pass left ambiguous: one warp per row computes float64
// distances ||x - mu_c||^2 to each listed candidate (to every centroid when
// the list overflowed) and keeps the smallest (smaller index on ties).
template <int D>
__global__ void __launch_bounds__(256) k_refine(const bf16* __restrict__ X, const float* __restrict__ cent,
                                                int N, int C, const int* __restrict__ refine,
                                                const int* __restrict__ count, int32_t* __restrict__ labels) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  const int total = *count;
  for (int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += nw) {
    const int* e = refine + (size_t)w * kRefineInts;
    const int h = e[0], row = e[1], n = e[2];
    float xv[PER];
    {
      const bf16* xr = X + ((size_t)h * N + row) * D + lane * PER;
      if constexpr (PER == 4) {
        const float4 v = ld4(xr);
        xv[0] = v.x; xv[1] = v.y; xv[2] = v.z; xv[3] = v.w;
      } else {
        const float2 v = ld2(xr);
        xv[0] = v.x; xv[1] = v.y;
      }
    }
    const int cnt = n < 0 ? C : n;
    double best = 1e300;
    int bc = 0;
    for (int i = 0; i < cnt; ++i) {
      const int c = n < 0 ? i : e[3 + i];
      const float* mu = cent + ((size_t)h * C + c) * D + lane * PER;
      double acc = 0.0;
#pragma unroll
      for (int t = 0; t < PER; ++t) {
        const double df = (double)xv[t] - (double)mu[t];
        acc = fma(df, df, acc);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (acc < best || (acc == best && c < bc)) { best = acc; bc = c; }
    }
    if (lane == 0) labels[(size_t)h * N + row] = bc;
  }
}

template <int D>
struct Smem {
  static constexpr int kXBytes = BM * D * 2;
  // offsets within the 1024-aligned dynamic shared memory
  __host__ __device__ static int cent_off() { return 0; }
  __host__ __device__ static int x_off(int Cpad) { return (Cpad * D * 2 + 1023) & ~1023; }
  __host__ __device__ static int cn_off(int Cpad) { return x_off(Cpad) + 2 * kXBytes; }
  __host__ __device__ static int merge_off(int Cpad) { return cn_off(Cpad) + ((Cpad * 4 + 15) & ~15); }
  __host__ __device__ static int list_off(int Cpad) { return merge_off(Cpad) + BM * 4 * 4; }
  __host__ __device__ static int bar_off(int Cpad) { return list_off(Cpad) + 2 * KC * 256 * 4; }
  // at least 120 KB so that only one block (and one 512-column tensor-memory
  // allocation) lives on an SM
  static int total(int Cpad) { return std::max(bar_off(Cpad) + 16 * 8 + 1024, 120 * 1024); }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_assign_tc(const bf16* __restrict__ X, const bf16* __restrict__ cb, const float* __restrict__ cnorm,
                const Bounds* __restrict__ bounds, const float* __restrict__ xnorm,
                const float* __restrict__ cent, int N, int C, int Cpad, int tiles_per_cta,
                int32_t* __restrict__ labels, int* __restrict__ refine, int* __restrict__ refine_count,
                int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using S = Smem<D>;
  uint8_t* cent_s = smem + S::cent_off();
  uint8_t* x_s = smem + S::x_off(Cpad);
  float* cn_s = reinterpret_cast<float*>(smem + S::cn_off(Cpad));
  int* merge = reinterpret_cast<int*>(smem + S::merge_off(Cpad));
  float* list_s = reinterpret_cast<float*>(smem + S::list_off(Cpad));
  int* list_c = reinterpret_cast<int*>(smem + S::list_off(Cpad) + KC * 256 * 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::bar_off(Cpad));
  uint64_t* cent_full = bars + 0;
  uint64_t* x_full = bars + 1;     // [2]
  uint64_t* x_empty = bars + 3;    // [2]
  uint64_t* acc_full = bars + 5;   // [2]
  uint64_t* acc_empty = bars + 7;  // [2]
  uint64_t* done = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 11);

  const int h = blockIdx.y;
  const int T = (N + BM - 1) / BM;
  const int t0 = blockIdx.x * tiles_per_cta;
  const int nt = min(tiles_per_cta, T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = (Cpad + kSlotCols - 1) / kSlotCols;
  constexpr int CPR = D / 8;  // 16-byte chunks per row

  if (threadIdx.x == 0) {
    tc::mbar_init(cent_full, kProducers);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(x_full + i, kProducers);
      tc::mbar_init(x_empty + i, 1);
      tc::mbar_init(acc_full + i, 1);
      tc::mbar_init(acc_empty + i, 128);
    }
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  for (int c = threadIdx.x; c < Cpad; c += blockDim.x) cn_s[c] = cnorm[(size_t)h * Cpad + c];
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = tc::mbar_wait(cent_full, 0, abort_flag, status);
      const uint32_t cent_a = tc::smem_u32(cent_s);
      const uint32_t cregion = (uint32_t)Cpad * 128u;
      for (int t = 0; ok && t < nt; ++t) {
        const int stage = t & 1;
        ok = tc::mbar_wait(x_full + stage, (t >> 1) & 1, abort_flag, status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t xa = tc::smem_u32(x_s + stage * S::kXBytes);
        for (int j = 0; j < nchunk; ++j) {
          const int g = t * nchunk + j, slot = g & 1, use = g >> 1;
          ok = tc::mbar_wait(acc_empty + slot, (use & 1) ^ 1, abort_flag, status);
          if (!ok) break;
          tc::tc_fence_after();
          const int n0 = j * kSlotCols, nj = min(kSlotCols, Cpad - n0);
          const uint32_t id = tc::idesc_bf16(BM, nj, false, false);
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t a = tc::desc_kmajor(xa, BM * 128u, k);
            const uint64_t b = tc::desc_kmajor(cent_a + (uint32_t)n0 * 128u, cregion, k);
            tc::mma_ss(tmem + (uint32_t)(slot * kSlotCols), a, b, id, k > 0 ? 1u : 0u);
          }
          tc::mma_commit(acc_full + slot);
        }
        tc::mma_commit(x_empty + stage);
      }
      tc::mma_commit(done);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ----------------------------------------------------------- producers
    const int pt = threadIdx.x - 32;
    const uint32_t cent_a = tc::smem_u32(cent_s);
    const bf16* cbh = cb + (size_t)h * Cpad * D;
    for (int e = pt; e < Cpad * CPR; e += kProducers) {
      const int r = e / CPR, c = e % CPR;
      tc::cp_async16(cent_a + tc::sw128_offset(r, c, Cpad), cbh + (size_t)r * D + c * 8, 16);
    }
    tc::cp_async_wait_all();
    tc::fence_proxy_async();
    tc::mbar_arrive(cent_full);
    const bf16* Xh = X + (size_t)h * N * D;
    for (int t = 0; t < nt; ++t) {
      const int stage = t & 1;
      if (!tc::mbar_wait(x_empty + stage, ((t >> 1) & 1) ^ 1, abort_flag, status)) break;
      const uint32_t xa = tc::smem_u32(x_s + stage * S::kXBytes);
      const int row0 = (t0 + t) * BM;
      for (int e = pt; e < BM * CPR; e += kProducers) {
        const int r = e / CPR, c = e % CPR;
        const bool valid = row0 + r < N;
        const bf16* src = Xh + (size_t)(valid ? row0 + r : 0) * D + c * 8;
        tc::cp_async16(xa + tc::sw128_offset(r, c, BM), src, valid ? 16u : 0u);
      }
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
      tc::mbar_arrive(x_full + stage);
    }
    tc::cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - 4) >> 2;           // 0 or 1
    const int r = ((warp & 3) << 5) + lane;   // TMEM lane == tile row
    const Bounds bd = bounds[h];
    for (int t = 0; t < nt; ++t) {
      const int row = (t0 + t) * BM + r;
      const float xn = row < N ? xnorm[(size_t)h * N + row] : 0.f;
      const float B = 2.f * xn * (bd.dmax + 6.1035e-5f * bd.mmax) +
                      9.5367e-7f * (bd.nmax + 2.f * xn * bd.mmax) + 1e-30f;
      const float W = 2.f * B;
      const int et = threadIdx.x - 128;  // epilogue thread 0..255
      float* ls = list_s + et;
      int* lc = list_c + et;
      Cands st{INFINITY, 0, 0};
      bool mine = false;
      for (int j = 0; j < nchunk; ++j) {
        const int g = t * nchunk + j, slot = g & 1, use = g >> 1;
        if (slot != wg) continue;
        mine = true;
        if (!tc::mbar_wait_warp(acc_full + slot, use & 1, abort_flag, status)) break;
        tc::tc_fence_after();
        const int n0 = j * kSlotCols, nj = min(kSlotCols, Cpad - n0);
        const uint32_t base = tc::taddr(tmem, (uint32_t)((warp & 3) << 5), (uint32_t)(slot * kSlotCols));
        const int n32 = nj & ~31;
        // pass 1: chunk minimum (padding columns score +inf)
        float m = INFINITY;
        for (int c0 = 0; c0 < n32; c0 += 32) {
          uint32_t v[32];
          tc::tmem_ld32(base + (uint32_t)c0, v);
          tc::tmem_ld_wait();
          m = fminf(m, min32(v, cn_s + n0 + c0));
        }
        if (n32 < nj) {
          uint32_t v[16];
          tc::tmem_ld16(base + (uint32_t)n32, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) m = fminf(m, fmaf(-2.f, __uint_as_float(v[q]), cn_s[n0 + n32 + q]));
        }
        if (m < st.best) {
          st.best = m;
          if (st.n) cand_compact(st, W, ls, lc);
        }
        // pass 2: every column within the window of the running minimum
        const float thr = st.best + W;
        for (int c0 = 0; c0 < n32; c0 += 32) {
          uint32_t v[32];
          tc::tmem_ld32(base + (uint32_t)c0, v);
          tc::tmem_ld_wait();
          collect<32>(st, v, cn_s + n0 + c0, n0 + c0, C, thr, ls, lc);
        }
        if (n32 < nj) {
          uint32_t v[16];
          tc::tmem_ld16(base + (uint32_t)n32, v);
          tc::tmem_ld_wait();
          collect<16>(st, v, cn_s + n0 + n32, n0 + n32, C, thr, ls, lc);
        }
        tc::tc_fence_before();
        tc::mbar_arrive(acc_empty + slot);
      }
      // on abort keep walking the tiles (waits now return at once) so that
      // both warpgroups pass the same named barriers
      bool finalize = mine;
      if (nchunk >= 2) {
        int* mrow = merge + r * 4;
        if (wg == 1) { mrow[0] = __float_as_int(st.best); mrow[2] = st.n; mrow[3] = st.over; }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (wg == 0) {
          const float ob = __int_as_float(mrow[0]);
          const int on = mrow[2];
          st.over |= mrow[3];
          if (ob < st.best) {
            st.best = ob;
            if (st.n) cand_compact(st, W, ls, lc);
          }
          const float thr = st.best + W;
          for (int i = 0; i < min(on, KC); ++i) {
            const float os = list_s[i * 256 + et + 128];
            if (os <= thr) cand_push(st, os, list_c[i * 256 + et + 128], ls, lc);
          }
          if (on > KC) st.over = 1;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        finalize = wg == 0;
      }
      if (!finalize || row >= N || *abort_flag) continue;
      // the listed candidate with the smallest score (smaller index on ties)
      cand_compact(st, W, ls, lc);
      int label = 0;
      float bs = INFINITY;
      for (int i = 0; i < min(st.n, KC); ++i) {
        const float v = ls[i * 256];
        const int c = lc[i * 256];
        if (v < bs || (v == bs && c < label)) { bs = v; label = c; }
      }
      labels[(size_t)h * N + row] = label;
      if (st.n > 1 || st.over) {
        // several centroids within the bound: decided later in float64
        const int k = atomicAdd(refine_count, 1);
        int* e = refine + (size_t)k * kRefineInts;
        e[0] = h; e[1] = row; e[2] = st.over ? -1 : st.n;
        for (int i = 0; i < min(st.n, KC); ++i) e[3 + i] = lc[i * 256];
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::mbar_wait_warp(done, 0, abort_flag, status);
    __syncwarp();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool kmeans_tc_supported(int d, int C) {
  if (d != 64 && d != 128) return false;
  return round16(C) * d * 2 <= kCentBytesMax;
}

// Workspace: token norms [H,N] first (they only depend on H, N), then the
// per-iteration centroid copy, norms and bounds, and the list of rows left
// for the float64 pass with its counter.
struct TcWs {
  float* xn;
  bf16* cb;
  float* cn;
  Bounds* bd;
  int* refine;
  int* refine_count;
};

static size_t tc_layout(int H, int N, int d, int C, TcWs* out, void* ws) {
  Carve cv(ws);
  const int Cpad = round16(C);
  TcWs w;
  w.xn = cv.take<float>((size_t)H * N);
  w.cb = cv.take<bf16>((size_t)H * Cpad * d);
  w.cn = cv.take<float>((size_t)H * Cpad);
  w.bd = cv.take<Bounds>(H);
  w.refine = cv.take<int>((size_t)H * N * kRefineInts);
  w.refine_count = cv.take<int>(1);
  if (out) *out = w;
  return cv.used();
}

size_t kmeans_tc_ws_bytes(int H, int N, int d, int C) {
  if (!kmeans_tc_supported(d, C)) return 0;
  return tc_layout(H, N, d, C, nullptr, nullptr);
}

cudaError_t kmeans_tc_prepare_rows(const void* Xv, int H, int N, int d, void* ws, cudaStream_t st) {
  float* xn = static_cast<float*>(ws);  // first buffer of the layout above
  const bf16* X = static_cast<const bf16*>(Xv);
  const long long rows = (long long)H * N;
  if (d == 128) { k_row_norms<128><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(X, rows, xn); note_launch(); }
  else { k_row_norms<64><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(X, rows, xn); note_launch(); }
  return cudaGetLastError();
}

cudaError_t kmeans_assign_tc(const void* Xv, int H, int N, int d, int C, const float* cent,
                             int32_t* labels, void* ws, cudaStream_t st) {
  TcWs w;
  tc_layout(H, N, d, C, &w, ws);
  const int Cpad = round16(C);
  const bf16* X = static_cast<const bf16*>(Xv);
  const int T = (N + BM - 1) / BM;
  const int tpc = std::max(1, std::min(16, (int)((long long)H * T / (2 * 148))));
  const int gx = (T + tpc - 1) / tpc;
  cudaError_t e = cudaMemsetAsync(w.refine_count, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  if (d == 128) {
    k_prep_centroids<128><<<H, 256, 0, st>>>(cent, C, Cpad, w.cb, w.cn, w.bd); note_launch();
    const int smem = Smem<128>::total(Cpad);
    e = cudaFuncSetAttribute(k_assign_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_assign_tc<128><<<dim3(gx, H), kThreads, smem, st>>>(X, w.cb, w.cn, w.bd, w.xn, cent, N, C, Cpad, tpc,
                                                           labels, w.refine, w.refine_count, status_word());
    note_launch();
    k_refine<128><<<148 * 8, 256, 0, st>>>(X, cent, N, C, w.refine, w.refine_count, labels); note_launch();
  } else {
    k_prep_centroids<64><<<H, 256, 0, st>>>(cent, C, Cpad, w.cb, w.cn, w.bd); note_launch();
    const int smem = Smem<64>::total(Cpad);
    e = cudaFuncSetAttribute(k_assign_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_assign_tc<64><<<dim3(gx, H), kThreads, smem, st>>>(X, w.cb, w.cn, w.bd, w.xn, cent, N, C, Cpad, tpc,
                                                          labels, w.refine, w.refine_count, status_word());
    note_launch();
    k_refine<64><<<148 * 8, 256, 0, st>>>(X, cent, N, C, w.refine, w.refine_count, labels); note_launch();
  }
  return cudaGetLastError();
}

}  // namespace svg
