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
// argmin; otherwise the survivors are re-decided with float64 distances
// (smaller index on equal distance), so labels equal the exact argmin.
//
// Block of 12 warps: warp 0 allocates tensor memory and issues MMAs, warps 1-3
// copy tiles (cp.async into the 128-byte-swizzled layout), warps 4-7 and 8-11
// are two epilogue warpgroups that take alternate 256-column accumulator slots.
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

struct Cands {
  float best;
  int bc;
  int n;
  int over;
  float s[KC];
  int c[KC];
};

__device__ __forceinline__ void cand_init(Cands& st) {
  st.best = INFINITY; st.bc = 0; st.n = 0; st.over = 0;
}

__device__ __forceinline__ void cand_compact(Cands& st, float W) {
  int m = 0;
  for (int i = 0; i < st.n; ++i)
    if (st.s[i] <= st.best + W) { st.s[m] = st.s[i]; st.c[m] = st.c[i]; ++m; }
  st.n = m;
}

__device__ __forceinline__ void cand_add(Cands& st, float s, int c, float W) {
  if (s < st.best || (s == st.best && c < st.bc)) { st.best = s; st.bc = c; }
  if (st.n == KC) cand_compact(st, W);
  if (st.n == KC) { st.over = 1; return; }
  st.s[st.n] = s; st.c[st.n] = c; ++st.n;
}

template <int D>
__device__ double exact_dist(const bf16* __restrict__ xrow, const float* __restrict__ mu) {
  double acc = 0.0;
#pragma unroll 4
  for (int t = 0; t < D; t += 4) {
    const float4 x = ld4(xrow + t);
    const float4 m = *reinterpret_cast<const float4*>(mu + t);
    double d0 = (double)x.x - m.x, d1 = (double)x.y - m.y, d2 = (double)x.z - m.z, d3 = (double)x.w - m.w;
    acc = fma(d0, d0, acc); acc = fma(d1, d1, acc); acc = fma(d2, d2, acc); acc = fma(d3, d3, acc);
  }
  return acc;
}

template <int D>
struct Smem {
  static constexpr int kXBytes = BM * D * 2;
  // offsets within the 1024-aligned dynamic shared memory
  __host__ __device__ static int cent_off() { return 0; }
  __host__ __device__ static int x_off(int Cpad) { return (Cpad * D * 2 + 1023) & ~1023; }
  __host__ __device__ static int cn_off(int Cpad) { return x_off(Cpad) + 2 * kXBytes; }
  __host__ __device__ static int merge_off(int Cpad) { return cn_off(Cpad) + ((Cpad * 4 + 15) & ~15); }
  __host__ __device__ static int bar_off(int Cpad) { return merge_off(Cpad) + BM * (4 + 2 * KC) * 4; }
  // at least 120 KB so that only one block (and one 512-column tensor-memory
  // allocation) lives on an SM
  static int total(int Cpad) { return std::max(bar_off(Cpad) + 16 * 8 + 1024, 120 * 1024); }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_assign_tc(const bf16* __restrict__ X, const bf16* __restrict__ cb, const float* __restrict__ cnorm,
                const Bounds* __restrict__ bounds, const float* __restrict__ xnorm,
                const float* __restrict__ cent, int N, int C, int Cpad, int tiles_per_cta,
                int32_t* __restrict__ labels, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using S = Smem<D>;
  uint8_t* cent_s = smem + S::cent_off();
  uint8_t* x_s = smem + S::x_off(Cpad);
  float* cn_s = reinterpret_cast<float*>(smem + S::cn_off(Cpad));
  int* merge = reinterpret_cast<int*>(smem + S::merge_off(Cpad));
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
    const float* ch = cent + (size_t)h * C * D;
    const bf16* Xh = X + (size_t)h * N * D;
    for (int t = 0; t < nt; ++t) {
      const int row = (t0 + t) * BM + r;
      const float xn = row < N ? xnorm[(size_t)h * N + row] : 0.f;
      const float B = 2.f * xn * (bd.dmax + 6.1035e-5f * bd.mmax) +
                      9.5367e-7f * (bd.nmax + 2.f * xn * bd.mmax) + 1e-30f;
      const float W = 2.f * B;
      Cands st;
      cand_init(st);
      bool mine = false;
      for (int j = 0; j < nchunk; ++j) {
        const int g = t * nchunk + j, slot = g & 1, use = g >> 1;
        if (slot != wg) continue;
        mine = true;
        if (!tc::mbar_wait(acc_full + slot, use & 1, abort_flag, status)) break;
        tc::tc_fence_after();
        const int n0 = j * kSlotCols, nj = min(kSlotCols, Cpad - n0);
        const uint32_t base = tc::taddr(tmem, (uint32_t)((warp & 3) << 5), (uint32_t)(slot * kSlotCols));
        int c0 = 0;
        for (; c0 + 32 <= nj; c0 += 32) {
          uint32_t v[32];
          tc::tmem_ld32(base + (uint32_t)c0, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int c = n0 + c0 + q;
            const float s = fmaf(-2.f, __uint_as_float(v[q]), cn_s[c]);
            if (c < C && s <= st.best + W) cand_add(st, s, c, W);
          }
        }
        if (c0 < nj) {  // 16-column tail
          uint32_t v[16];
          tc::tmem_ld16(base + (uint32_t)c0, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int c = n0 + c0 + q;
            const float s = fmaf(-2.f, __uint_as_float(v[q]), cn_s[c]);
            if (c < C && s <= st.best + W) cand_add(st, s, c, W);
          }
        }
        tc::tc_fence_before();
        tc::mbar_arrive(acc_empty + slot);
      }
      // on abort keep walking the tiles (waits now return at once) so that
      // both warpgroups pass the same named barriers
      // combine the two warpgroups' partial results when both saw this tile
      bool finalize = mine;
      if (nchunk >= 2) {
        int* mrow = merge + r * (4 + 2 * KC);
        if (wg == 1) {
          mrow[0] = __float_as_int(st.best); mrow[1] = st.bc; mrow[2] = st.n; mrow[3] = st.over;
          for (int i = 0; i < st.n; ++i) { mrow[4 + i] = __float_as_int(st.s[i]); mrow[4 + KC + i] = st.c[i]; }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (wg == 0) {
          const float ob = __int_as_float(mrow[0]);
          const int obc = mrow[1], on = mrow[2];
          st.over |= mrow[3];
          if (ob < st.best || (ob == st.best && obc < st.bc)) { st.best = ob; st.bc = obc; }
          for (int i = 0; i < on; ++i) cand_add(st, __int_as_float(mrow[4 + i]), mrow[4 + KC + i], W);
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        finalize = wg == 0;
      }
      if (!finalize || row >= N || *abort_flag) continue;
      cand_compact(st, W);
      int label = st.bc;
      if (st.over || st.n > 1) {
        const bf16* xr = Xh + (size_t)row * D;
        double bestd = 1e300;
        int bestc = 0;
        if (st.over) {
          for (int c = 0; c < C; ++c) {
            const double dd = exact_dist<D>(xr, ch + (size_t)c * D);
            if (dd < bestd) { bestd = dd; bestc = c; }
          }
        } else {
          for (int i = 0; i < st.n; ++i) {
            const int c = st.c[i];
            const double dd = exact_dist<D>(xr, ch + (size_t)c * D);
            if (dd < bestd || (dd == bestd && c < bestc)) { bestd = dd; bestc = c; }
          }
        }
        label = bestc;
      }
      labels[(size_t)h * N + row] = label;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::mbar_wait(done, 0, abort_flag, status);
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool kmeans_tc_supported(int d, int C) {
  if (d != 64 && d != 128) return false;
  return round16(C) * d * 2 <= kCentBytesMax;
}

// Workspace: token norms [H,N] first (they only depend on H, N), then the
// per-iteration centroid copy, norms and bounds.
static size_t tc_layout(int H, int N, int d, int C, bf16** cb, float** cn, Bounds** bd, float** xn,
                        void* ws) {
  Carve cv(ws);
  const int Cpad = round16(C);
  float* e = cv.take<float>((size_t)H * N);
  bf16* a = cv.take<bf16>((size_t)H * Cpad * d);
  float* b = cv.take<float>((size_t)H * Cpad);
  Bounds* c = cv.take<Bounds>(H);
  if (cb) { *cb = a; *cn = b; *bd = c; *xn = e; }
  return cv.used();
}

size_t kmeans_tc_ws_bytes(int H, int N, int d, int C) {
  if (!kmeans_tc_supported(d, C)) return 0;
  return tc_layout(H, N, d, C, nullptr, nullptr, nullptr, nullptr, nullptr);
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
  bf16 *cb; float *cn, *xn; Bounds* bd;
  tc_layout(H, N, d, C, &cb, &cn, &bd, &xn, ws);
  const int Cpad = round16(C);
  const bf16* X = static_cast<const bf16*>(Xv);
  const int T = (N + BM - 1) / BM;
  int tpc = std::max(1, std::min(16, (int)((long long)H * T / (2 * 148))));
  const int gx = (T + tpc - 1) / tpc;
  cudaError_t e;
  if (d == 128) {
    k_prep_centroids<128><<<H, 256, 0, st>>>(cent, C, Cpad, cb, cn, bd); note_launch();
    const int smem = Smem<128>::total(Cpad);
    e = cudaFuncSetAttribute(k_assign_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_assign_tc<128><<<dim3(gx, H), kThreads, smem, st>>>(X, cb, cn, bd, xn, cent, N, C, Cpad, tpc, labels,
                                                           status_word()); note_launch();
  } else {
    k_prep_centroids<64><<<H, 256, 0, st>>>(cent, C, Cpad, cb, cn, bd); note_launch();
    const int smem = Smem<64>::total(Cpad);
    e = cudaFuncSetAttribute(k_assign_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_assign_tc<64><<<dim3(gx, H), kThreads, smem, st>>>(X, cb, cn, bd, xn, cent, N, C, Cpad, tpc, labels,
                                                          status_word()); note_launch();
  }
  return cudaGetLastError();
}

}  // namespace svg
