// Tensor-core k-means assignment for bf16 tokens (SVG-EAR review, step (1):
// "Flash k-means" clustering of queries and keys).
//
// The nearest centroid of x is the one with the largest score
//   s_c = x . mu_c - ||mu_c||^2 / 2.
// For a tile of 128 tokens, x . mu_c comes from tcgen05 MMAs (A = token tile,
// B = bf16-rounded centroids resident in shared memory, fp32 accumulators in
// tensor memory, 128 centroid columns per accumulator slot).  The epilogue
// subtracts ||mu_c||^2 / 2, writes the column index into the low mantissa bits
// of the score (so one float carries score and index, and no two columns tie)
// and keeps, per token, the two largest packed scores b1 >= b2 exactly and an
// upper bound b2 >= b3 of the third largest.
//
// Every packed score is within E of the exact s_c (bf16 rounding of mu, the
// fp32 accumulation inside the MMA, the subtraction, the index bits; bound
// below), so the exact best column has a packed score >= b1 - 2E:
//   b2 <  b1 - 2E            -> the label is the column of b1 (exact);
//   b3 <  b1 - 2E <= b2      -> one of the columns of b1, b2: decided in float64
//                               (b3 bounds the third score from above, so no
//                               third column is within the bound);
//   otherwise                -> every centroid is checked in float64.
// Ties in float64 go to the smaller index, so labels equal the exact argmin.
//
// Block of 10 warps: warp 0 allocates tensor memory and issues MMAs, warp 1
// issues the TMA copies (centroid table once, token tiles through a ring of
// stages), warps 2-5 and 6-9 are two epilogue warpgroups that take alternate
// 128-column chunks.  When a tile has chunks in both warpgroups, the one that
// did not see the tile's last chunk hands its partial top three to the other
// through shared memory (mbarrier-synchronised, no lockstep).
//
// When the bf16 centroids do not fit in shared memory next to two token
// stages (d = 128 and more than 512 centroids), the centroids are taken in
// segments of whole 128-column chunks, one launch per segment: every launch
// but the last stores each token's top three (packed scores carry the global
// column index) to a [3][H][N] buffer, every launch but the first folds the
// stored top three in before its own decision or store, so the last launch
// decides over all centroids with the same rule.
#include <cuda.h>

#include <algorithm>
#include <cfloat>
#include <climits>

#include "internal.h"
#include "kmeans_tc.cuh"
#include "tc_common.cuh"

namespace svg {

namespace {

constexpr int BM = 128;                // tokens per tile (MMA M)
constexpr int kThreads = 320;
constexpr int kChunk = 128;            // accumulator columns per TMEM slot
constexpr int kSlots = 4;
constexpr int kMaxStages = 6;
constexpr int kSmemLimit = 232448;     // opt-in dynamic shared memory per block
constexpr int kMaxC = 1024;            // index bits packed into the score: at most 10
constexpr float kPadHalfNorm = 1e30f;  // ||mu||^2/2 of padding columns: never best, finite

__host__ __device__ inline int round16(int x) { return (x + 15) & ~15; }
__host__ __device__ inline int round128(int x) { return (x + 127) & ~127; }

struct Bounds {  // per head; non-negative floats, combined with integer atomicMax
  float dmax;    // max_c ||mu_c - bf16(mu_c)||
  float mmax;    // max_c ||bf16(mu_c)||
  float nmax;    // max_c ||mu_c||^2
  int pad;
};

// Shared-memory layout of the assignment kernel (offsets from a 1024-aligned base).
struct Lay {
  int cent, x, tab, merge, bars, total;
};
__host__ __device__ inline Lay layout(int D, int Cr, int Cpad, int stages) {
  Lay l;
  l.cent = 0;
  l.x = Cr * D * 2;                          // Cr is a multiple of 128: 1024-aligned
  l.tab = l.x + stages * BM * D * 2;
  l.merge = l.tab + Cpad * 8;
  l.bars = l.merge + 2 * 3 * BM * 4;
  l.total = l.bars + 32 * 8 + 1024;          // barriers, TMEM slot, abort flag; alignment slack
  return l;
}

// Per block of 32 centroid rows of one head: the bf16 copy (zero rows up to
// Cr), the table entry {||mu||^2 / 2, index} (padding columns up to Cpad get
// kPadHalfNorm), a transposed float32 copy [d][C] for the float64 pass, and
// the per-head maxima of the error bound.
template <int D>
__global__ void __launch_bounds__(256) k_prep_centroids(const float* __restrict__ cent, int C, int Cpad, int Cr,
                                                        bf16* __restrict__ cb, int2* __restrict__ table,
                                                        float* __restrict__ centT, Bounds* __restrict__ bounds) {
  __shared__ float tile[32][D + 1];
  __shared__ float red[3][8];
  const int h = blockIdx.y, c0 = blockIdx.x * 32;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < 32 * D; e += blockDim.x) {
    const int r = e / D, t = e % D, c = c0 + r;
    tile[r][t] = c < C ? cent[((size_t)h * C + c) * D + t] : 0.f;
  }
  __syncthreads();
  float dmax = 0.f, mmax = 0.f, nmax = 0.f;
  for (int r = w; r < 32; r += 8) {
    const int c = c0 + r;
    if (c >= Cr) break;
    double dn = 0.0, mb = 0.0, n2 = 0.0;
    for (int t = lane; t < D; t += 32) {
      const float m = tile[r][t];
      const bf16 b = __float2bfloat16_rn(m);
      cb[((size_t)h * Cr + c) * D + t] = b;
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
    if (lane == 0 && c < Cpad)
      table[(size_t)h * Cpad + c] = make_int2(__float_as_int(c < C ? (float)(0.5 * n2) : kPadHalfNorm), c);
    if (c < C) {
      dmax = fmaxf(dmax, (float)sqrt(dn));
      mmax = fmaxf(mmax, (float)sqrt(mb));
      nmax = fmaxf(nmax, (float)n2);
    }
  }
  for (int e = threadIdx.x; e < 32 * D; e += blockDim.x) {
    const int t = e / 32, r = e % 32, c = c0 + r;
    if (c < C) centT[((size_t)h * D + t) * C + c] = tile[r][t];
  }
  if (lane == 0) { red[0][w] = dmax; red[1][w] = mmax; red[2][w] = nmax; }
  __syncthreads();
  if (threadIdx.x < 3) {
    float m = 0.f;
    for (int i = 0; i < 8; ++i) m = fmaxf(m, red[threadIdx.x][i]);
    // rounded up a little so that the bound stays an upper bound
    atomicMax(reinterpret_cast<int*>(&bounds[h]) + threadIdx.x, __float_as_int(m * 1.0001f));
  }
}

// ||x_i|| per token (float, rounded up slightly), once per k-means call: D/8
// lanes per row, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) k_row_norms(const bf16* __restrict__ X, long long rows,
                                                   float* __restrict__ xn) {
  constexpr int LPR = D / 8, RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW; r0 < rows;
       r0 += nw * RPW) {
    const long long r = r0 + lane / LPR;
    float s = 0.f;
    if (r < rows) {
      const uint4 u = *reinterpret_cast<const uint4*>(X + r * D + (lane % LPR) * 8);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(w4[i] << 16), b = __uint_as_float(w4[i] & 0xffff0000u);
        s = fmaf(a, a, fmaf(b, b, s));
      }
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (r < rows && lane % LPR == 0) xn[r] = sqrtf(s) * 1.00001f;
  }
}

// Rows the tensor-core pass left with two candidates {c1, c2}: float64
// distances ||x - mu_c||^2 to both, the smaller wins (the smaller index on
// ties).  Eight lanes per row, four rows per warp.
template <int D>
__global__ void __launch_bounds__(256) k_refine2(const bf16* __restrict__ X, const float* __restrict__ cent,
                                                 int N, int C, const int4* __restrict__ list,
                                                 const int* __restrict__ count, int32_t* __restrict__ labels) {
  constexpr int PER = D / 8;  // dimensions per lane
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int total = *count;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int wb = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4; wb < total; wb += nwarps * 4) {
    const int gi = wb + (lane >> 3);
    const bool act = gi < total;
    int4 e = make_int4(0, 0, 0, 0);
    if (act) e = list[gi];
    double a0 = 0.0, a1 = 0.0;
    if (act) {
      const bf16* xr = X + ((size_t)e.x * N + e.y) * D + sub * PER;
      const float* m0 = cent + ((size_t)e.x * C + e.z) * D + sub * PER;
      const float* m1 = cent + ((size_t)e.x * C + e.w) * D + sub * PER;
#pragma unroll
      for (int t = 0; t < PER; t += 4) {
        const float2 xa = ld2(xr + t), xb = ld2(xr + t + 2);
        const float4 u = *reinterpret_cast<const float4*>(m0 + t);
        const float4 w = *reinterpret_cast<const float4*>(m1 + t);
        const double x4[4] = {xa.x, xa.y, xb.x, xb.y};
        const double u4[4] = {u.x, u.y, u.z, u.w}, w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const double du = x4[i] - u4[i], dw = x4[i] - w4[i];
          a0 = fma(du, du, a0);
          a1 = fma(dw, dw, a1);
        }
      }
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      a0 += __shfl_xor_sync(0xffffffffu, a0, o);
      a1 += __shfl_xor_sync(0xffffffffu, a1, o);
    }
    if (act && sub == 0)
      labels[(size_t)e.x * N + e.y] = (a1 < a0 || (a1 == a0 && e.w < e.z)) ? e.w : e.z;
  }
}

// Rows with three or more candidates, listed per head: every centroid is
// scanned in float32, eight rows at a time (a thread owns centroids tid,
// tid + blockDim, ... and keeps the eight rows' distances, so each coalesced
// load of the transposed centroids serves eight rows).  With d + 3 roundings
// per distance the float32 value is within (d + 3) 2^-24 of the exact one in
// relative terms, so every centroid whose float32 distance is within a
// relative 2e-5 of the row's smallest is a candidate: a single candidate is
// the nearest centroid, several (ties within the float32 error) are re-checked
// in float64 by their threads; the smallest float64 distance wins, the
// smaller index on ties.
constexpr int kFullRows = 8;
constexpr int kFullThreads = 256;

template <int D>
__global__ void __launch_bounds__(kFullThreads) k_refine_full(const bf16* __restrict__ X,
                                                              const float* __restrict__ cent,
                                                              const float* __restrict__ centT, int N, int C,
                                                              const int* __restrict__ list,
                                                              const int* __restrict__ counts,
                                                              int32_t* __restrict__ labels) {
  constexpr int R = kFullRows;
  constexpr int KMAX = kMaxC / kFullThreads;  // centroids per thread: blocks of 256 when C > 256
  __shared__ __align__(16) float xs[D][R];
  __shared__ float rmin[R][kFullThreads / 32];
  __shared__ double rbest[R][kFullThreads / 32];
  __shared__ int rbc[R][kFullThreads / 32];
  __shared__ int rcnt[R][kFullThreads / 32];
  __shared__ int rtie[R];
  const int h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  const int total = counts[h];
  const int* lh = list + (size_t)h * N;
  const float* cth = centT + (size_t)h * D * C;
  const float* ch = cent + (size_t)h * C * D;
  for (int base = blockIdx.x * R; base < total; base += gridDim.x * R) {
    for (int e = tid; e < D * R; e += blockDim.x) {
      const int r = e / D, t = e % D;
      xs[t][r] = base + r < total ? __bfloat162float(X[((size_t)h * N + lh[base + r]) * D + t]) : 0.f;
    }
    __syncthreads();
    float dl[KMAX][R];
    float dmin[R];
#pragma unroll
    for (int r = 0; r < R; ++r) dmin[r] = INFINITY;
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      const int c = k * blockDim.x + tid;
#pragma unroll
      for (int r = 0; r < R; ++r) dl[k][r] = INFINITY;
      if (k * (int)blockDim.x >= C) continue;
      if (c < C) {
        float acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll 16
        for (int t = 0; t < D; ++t) {
          const float m = cth[(size_t)t * C + c];
          const float4 xa = *reinterpret_cast<const float4*>(&xs[t][0]);
          const float4 xb = *reinterpret_cast<const float4*>(&xs[t][4]);
          const float xv[R] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const float df = xv[r] - m;
            acc[r] = fmaf(df, df, acc[r]);
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          dl[k][r] = acc[r];
          dmin[r] = fminf(dmin[r], acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dmin[r] = fminf(dmin[r], __shfl_xor_sync(0xffffffffu, dmin[r], o));
      if (lane == 0) rmin[r][warp] = dmin[r];
    }
    __syncthreads();
    // rows whose window holds a single centroid are decided; the others
    // (ties within the float32 error) go through float64
    float lim[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float g = INFINITY;
      for (int i = 0; i < nwarp; ++i) g = fminf(g, rmin[r][i]);
      lim[r] = g * (1.f + 2e-5f) + 1e-30f;
      int n = 0, cmin = INT_MAX;
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        const int c = k * blockDim.x + tid;
        if (c < C && dl[k][r] <= lim[r]) { ++n; cmin = min(cmin, c); }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        n += __shfl_xor_sync(0xffffffffu, n, o);
        cmin = min(cmin, __shfl_xor_sync(0xffffffffu, cmin, o));
      }
      if (lane == 0) { rcnt[r][warp] = n; rbc[r][warp] = cmin; }
    }
    __syncthreads();
    if (tid < R) {
      int n = 0, cmin = INT_MAX;
      for (int i = 0; i < nwarp; ++i) { n += rcnt[tid][i]; cmin = min(cmin, rbc[tid][i]); }
      rtie[tid] = n > 1;
      if (base + tid < total && n == 1) labels[(size_t)h * N + lh[base + tid]] = cmin;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!rtie[r] || base + r >= total) continue;  // block-uniform
      double best = DBL_MAX;
      int bc = INT_MAX;
#pragma unroll
      for (int k = 0; k < KMAX; ++k) {
        const int c = k * blockDim.x + tid;
        if (c < C && dl[k][r] <= lim[r]) {
          const float4* mu = reinterpret_cast<const float4*>(ch + (size_t)c * D);
          double a4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
          for (int t4 = 0; t4 < D / 4; ++t4) {
            const float4 m = mu[t4];
            const double d0 = (double)xs[4 * t4][r] - m.x, d1 = (double)xs[4 * t4 + 1][r] - m.y;
            const double d2 = (double)xs[4 * t4 + 2][r] - m.z, d3 = (double)xs[4 * t4 + 3][r] - m.w;
            a4[0] = fma(d0, d0, a4[0]); a4[1] = fma(d1, d1, a4[1]);
            a4[2] = fma(d2, d2, a4[2]); a4[3] = fma(d3, d3, a4[3]);
          }
          const double acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
          if (acc < best || (acc == best && c < bc)) { best = acc; bc = c; }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
        if (ob < best || (ob == best && oc < bc)) { best = ob; bc = oc; }
      }
      if (lane == 0) { rbest[r][warp] = best; rbc[r][warp] = bc; }
    }
    __syncthreads();
    if (tid < R && rtie[tid] && base + tid < total) {
      double bb = rbest[tid][0];
      int cc = rbc[tid][0];
      for (int i = 1; i < nwarp; ++i) {
        const double ob = rbest[tid][i];
        const int oc = rbc[tid][i];
        if (ob < bb || (ob == bb && oc < cc)) { bb = ob; cc = oc; }
      }
      labels[(size_t)h * N + lh[base + tid]] = cc;
    }
    __syncthreads();
  }
}

// Bound on |packed score - exact score| for a token of norm xn (see header):
// xn ||mu - bf16(mu)|| for the centroid rounding, 2^-14 xn ||bf16(mu)|| for the
// fp32 accumulation inside the MMA, a generous 2^-21 (||mu||^2 + 2 xn ||mu||)
// for the rounding of ||mu||^2/2 and of the subtraction, and 2^(bits-23) |s|
// for the index bits written over the mantissa.
__device__ __forceinline__ float score_error(float xn, const Bounds& b, float idx_rel) {
  const float mag = xn * b.mmax + 0.5f * b.nmax;
  return xn * (b.dmax + 6.1035156e-5f * b.mmax) + 4.7683716e-7f * (b.nmax + 2.f * xn * b.mmax) +
         idx_rel * mag * 1.0001f + 1e-30f;
}

// Insert two packed scores into the running top three (b1 >= b2 >= b3): the
// k-th largest of two sorted lists is the largest min(A_i, B_j) over i + j = k.
// b1 and b2 stay exact.  For the third, lo stands in for min(b1, lo): equal
// unless both new scores exceed b1, and never smaller, so b3 stays an upper
// bound of the third largest (and at most b2), which is all the decision and
// the merges need; it saves one instruction per pair of columns.
__device__ __forceinline__ void top3_add2(float& b1, float& b2, float& b3, float p0, float p1) {
  const float hi = fmaxf(p0, p1), lo = fminf(p0, p1);
  const float n3 = tc::fmax3(b3, fminf(b2, hi), lo);
  const float n2 = tc::fmax3(b2, fminf(b1, hi), lo);
  b1 = fmaxf(b1, hi);
  b2 = n2;
  b3 = n3;
}

template <int NV>
__device__ __forceinline__ void consume(const uint32_t (&v)[NV], const int4* __restrict__ tp, uint32_t keep,
                                        float& b1, float& b2, float& b3) {
#pragma unroll
  for (int q = 0; q < NV; q += 2) {
    const int4 e = tp[q >> 1];  // {||mu||^2/2, index} of two columns
    // both scores x.mu - ||mu||^2/2 in one two-wide subtraction
    uint64_t a2, n2, d2;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a2) : "r"(v[q]), "r"(v[q + 1]));
    asm("mov.b64 %0, {%1, %2};" : "=l"(n2) : "r"(e.x), "r"(e.z));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d2) : "l"(a2), "l"(n2));
    float s0, s1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(s0), "=f"(s1) : "l"(d2));
    const float p0 = __uint_as_float((__float_as_uint(s0) & keep) | (uint32_t)e.y);
    const float p1 = __uint_as_float((__float_as_uint(s1) & keep) | (uint32_t)e.w);
    top3_add2(b1, b2, b3, p0, p1);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_assign_tc(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmc,
                const int2* __restrict__ table, const Bounds* __restrict__ bounds,
                const float* __restrict__ xnorm, int N, int Cpad, int Cr, int stages, int tiles_per_cta,
                int nbits, int32_t* __restrict__ labels, int4* __restrict__ list2,
                int* __restrict__ list_full, int* __restrict__ counts, int* status, int tstride, int c_base,
                float* __restrict__ part, int pmode) {
  // Cpad / Cr: padded columns / resident rows of this launch's centroid
  // segment, which starts at global column c_base; tstride: the table's
  // per-head stride.  pmode bit 0: fold in the top three stored by the
  // previous segment; bit 1: store the top three instead of deciding.
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Lay L = layout(D, Cr, Cpad, stages);
  uint8_t* cent_s = smem + L.cent;
  uint8_t* x_s = smem + L.x;
  int2* tab = reinterpret_cast<int2*>(smem + L.tab);
  float* mbuf = reinterpret_cast<float*>(smem + L.merge);  // [2][3][BM]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* cent_full = bars;
  uint64_t* x_full = bars + 1;                  // [kMaxStages]
  uint64_t* x_empty = bars + 1 + kMaxStages;    // [kMaxStages]
  uint64_t* acc_full = bars + 13;               // [kSlots]
  uint64_t* acc_empty = bars + 17;              // [kSlots]
  uint64_t* merge_full = bars + 21;             // [2]
  uint64_t* merge_empty = bars + 23;            // [2]
  uint64_t* done = bars + 25;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 26);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 27);
  constexpr int kXBytes = BM * D * 2;

  const int h = blockIdx.y;
  const int T = (N + BM - 1) / BM;
  const int t0 = blockIdx.x * tiles_per_cta;
  const int nt = min(tiles_per_cta, T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = (Cpad + kChunk - 1) / kChunk;

  if (threadIdx.x == 0) {
    tc::mbar_init(cent_full, 1);
    for (int i = 0; i < stages; ++i) {
      tc::mbar_init(x_full + i, 1);
      tc::mbar_init(x_empty + i, 1);
    }
    for (int i = 0; i < kSlots; ++i) {
      tc::mbar_init(acc_full + i, 1);
      tc::mbar_init(acc_empty + i, 4);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(merge_full + i, 4);
      tc::mbar_init(merge_empty + i, 4);
    }
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  for (int c = threadIdx.x; c < Cpad; c += blockDim.x) tab[c] = table[(size_t)h * tstride + c_base + c];
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
    // The whole warp runs the loop (warp-uniform control and descriptor
    // arithmetic); one elected lane issues each tcgen05.mma and commit.
    const bool leader = tc::elect_one();
    bool ok = tc::mbar_wait_warp(cent_full, 0, abort_flag, status);
    const uint32_t cent_a = tc::smem_u32(cent_s);
    const uint32_t cregion = (uint32_t)Cr * 128u;
    int g = 0;
    for (int t = 0; ok && t < nt; ++t) {
      const int s = t % stages, k = t / stages;
      ok = tc::mbar_wait_warp(x_full + s, k & 1, abort_flag, status);
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t xa = tc::smem_u32(x_s + s * kXBytes);
      for (int j = 0; j < nch; ++j, ++g) {
        const int slot = g & (kSlots - 1), use = g >> 2;
        ok = tc::mbar_wait_warp(acc_empty + slot, (use & 1) ^ 1, abort_flag, status);
        if (!ok) break;
        tc::tc_fence_after();
        const int n0 = j * kChunk, nj = min(kChunk, Cpad - n0);
        const uint32_t id = tc::idesc_bf16(BM, nj, false, false);
        if (leader) {
#pragma unroll
          for (int k16 = 0; k16 < D / 16; ++k16) {
            const uint64_t a = tc::desc_kmajor(xa, BM * 128u, k16);
            const uint64_t b = tc::desc_kmajor(cent_a + (uint32_t)n0 * 128u, cregion, k16);
            tc::mma_ss(tmem + (uint32_t)(slot * kChunk), a, b, id, k16 > 0 ? 1u : 0u);
          }
          tc::mma_commit(acc_full + slot);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (leader) tc::mma_commit(x_empty + s);
      __syncwarp();
    }
    if (leader) tc::mma_commit(done);
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- TMA producer
    if (lane == 0) {
      tc::tma_prefetch_map(&tmx);
      tc::tma_prefetch_map(&tmc);
      const uint32_t cent_a = tc::smem_u32(cent_s);
      tc::mbar_arrive_expect_tx(cent_full, (uint32_t)(Cr * D * 2));
      for (int kh = 0; kh < D / 64; ++kh)
        for (int rb = 0; rb < Cr / 128; ++rb)
          tc::tma_load_3d(cent_a + (uint32_t)(kh * Cr * 128 + rb * 128 * 128), &tmc, kh * 64, c_base + rb * 128,
                          h, cent_full);
      for (int t = 0; t < nt; ++t) {
        const int s = t % stages, k = t / stages;
        if (!tc::mbar_wait(x_empty + s, (k & 1) ^ 1, abort_flag, status)) break;
        const uint32_t xa = tc::smem_u32(x_s + s * kXBytes);
        tc::mbar_arrive_expect_tx(x_full + s, (uint32_t)kXBytes);
        for (int kh = 0; kh < D / 64; ++kh)
          tc::tma_load_3d(xa + (uint32_t)(kh * BM * 128), &tmx, kh * 64, (t0 + t) * BM, h, x_full + s);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - 2) >> 2;           // 0 or 1: takes chunks g with g % 2 == wg
    const int quarter = warp & 3;             // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;        // tile row == TMEM lane
    const uint32_t keep = ~((1u << nbits) - 1u);
    const float idx_rel = ldexpf(1.f, nbits - 23);
    const Bounds bd = bounds[h];
    bool ok = true;
    for (int t = 0; t < nt && ok; ++t) {
      float b1 = -INFINITY, b2 = -INFINITY, b3 = -INFINITY;
      bool mine = false;
      for (int j = 0; j < nch; ++j) {
        const int g = t * nch + j;
        if ((g & 1) != wg) continue;
        mine = true;
        const int slot = g & (kSlots - 1), use = g >> 2;
        ok = tc::mbar_wait_warp(acc_full + slot, use & 1, abort_flag, status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t base = tc::taddr(tmem, (uint32_t)(quarter * 32), (uint32_t)(slot * kChunk));
        const int n0 = j * kChunk, nj = min(kChunk, Cpad - n0);
        const int4* tp = reinterpret_cast<const int4*>(tab + n0);
        int c0 = 0;
        for (; c0 + 64 <= nj; c0 += 64) {
          uint32_t va[32], vb[32];
          tc::tmem_ld32(base + (uint32_t)c0, va);
          tc::tmem_ld32(base + (uint32_t)(c0 + 32), vb);
          tc::tmem_ld_wait();
          consume<32>(va, tp + (c0 >> 1), keep, b1, b2, b3);
          consume<32>(vb, tp + ((c0 + 32) >> 1), keep, b1, b2, b3);
        }
        if (c0 + 32 <= nj) {
          uint32_t va[32];
          tc::tmem_ld32(base + (uint32_t)c0, va);
          tc::tmem_ld_wait();
          consume<32>(va, tp + (c0 >> 1), keep, b1, b2, b3);
          c0 += 32;
        }
        if (c0 < nj) {  // nj is a multiple of 16
          uint32_t va[16];
          tc::tmem_ld16(base + (uint32_t)c0, va);
          tc::tmem_ld_wait();
          consume<16>(va, tp + (c0 >> 1), keep, b1, b2, b3);
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(acc_empty + slot);
      }
      if (!ok || !mine) continue;
      // the tile's last chunk decides; the other warpgroup (if it had chunks
      // of this tile) hands over its partial top three
      const bool decider = ((t * nch + nch - 1) & 1) == wg;
      const int mb = t & 1;
      const uint32_t mpar = (uint32_t)(t >> 1) & 1u;
      float* mrow = mbuf + mb * 3 * BM + r;
      if (nch >= 2 && !decider) {
        ok = tc::mbar_wait_warp(merge_empty + mb, mpar ^ 1u, abort_flag, status);
        if (!ok) break;
        mrow[0] = b1; mrow[BM] = b2; mrow[2 * BM] = b3;
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(merge_full + mb);
        continue;
      }
      if (nch >= 2) {
        ok = tc::mbar_wait_warp(merge_full + mb, mpar, abort_flag, status);
        if (!ok) break;
        const float c1 = mrow[0], c2 = mrow[BM], c3 = mrow[2 * BM];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(merge_empty + mb);
        const float n3 = fmaxf(tc::fmax3(b3, fminf(b2, c1), fminf(b1, c2)), c3);
        const float n2 = tc::fmax3(b2, fminf(b1, c1), c2);
        b1 = fmaxf(b1, c1);
        b2 = n2;
        b3 = n3;
      }
      const int row = (t0 + t) * BM + r;
      if (pmode != 0) {
        const size_t plane = (size_t)gridDim.y * N, at = (size_t)h * N + row;
        if ((pmode & 1) && row < N) {  // the previous segments' top three
          const float c1 = part[at], c2 = part[plane + at], c3 = part[2 * plane + at];
          const float n3 = fmaxf(tc::fmax3(b3, fminf(b2, c1), fminf(b1, c2)), c3);
          const float n2 = tc::fmax3(b2, fminf(b1, c1), c2);
          b1 = fmaxf(b1, c1);
          b2 = n2;
          b3 = n3;
        }
        if (pmode & 2) {  // a later segment decides (pmode is uniform)
          if (row < N) { part[at] = b1; part[plane + at] = b2; part[2 * plane + at] = b3; }
          continue;
        }
      }
      int need = 0, lab = 0;
      if (row < N) {
        const float xn = xnorm[(size_t)h * N + row];
        const float thr = b1 - 2.02f * score_error(xn, bd, idx_rel);
        lab = (int)(__float_as_uint(b1) & ~keep);
        need = b2 >= thr ? (b3 >= thr ? -1 : 2) : 0;
        labels[(size_t)h * N + row] = lab;
      }
      // several centroids within the bound: listed for the float64 passes
      const uint32_t want2 = __ballot_sync(0xffffffffu, need == 2);
      const uint32_t wantf = __ballot_sync(0xffffffffu, need < 0);
      const uint32_t below = (1u << lane) - 1u;
      if (want2) {
        int base = 0;
        if (lane == 0) base = atomicAdd(counts, __popc(want2));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (need == 2)
          list2[base + __popc(want2 & below)] =
              make_int4(h, row, lab, (int)(__float_as_uint(b2) & ~keep));
      }
      if (wantf) {
        int base = 0;
        if (lane == 0) base = atomicAdd(counts + 1 + h, __popc(wantf));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (need < 0) list_full[(size_t)h * N + base + __popc(wantf & below)] = row;
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

// Token stages that fit next to a centroid segment of Cpad columns (Cr rows).
static int pick_stages(int d, int Cr, int Cpad) {
  int s = 0;
  while (s < kMaxStages && layout(d, Cr, Cpad, s + 1).total <= kSmemLimit) ++s;
  return s;
}

// Columns per launch: all of them (round128(C)) when they fit with two token
// stages, else the largest multiple of 128 that does (0: none).
static int segment_cols(int d, int C) {
  const int Cpad = round16(C), Cr = round128(C);
  if (pick_stages(d, Cr, Cpad) >= 2) return Cr;
  int s = Cr - kChunk;
  while (s >= kChunk && pick_stages(d, s, s) < 2) s -= kChunk;
  return s;
}

static bool segmented(int d, int C) { return segment_cols(d, C) < round16(C); }

bool kmeans_tc_supported(int d, int C) {
  if (d != 64 && d != 128) return false;
  if (C < 1 || C > kMaxC) return false;
  return segment_cols(d, C) >= kChunk;
}

bool kmeans_tc_usable(const void* X, int N, int d, int C) {
  return kmeans_tc_supported(d, C) && N >= BM && (reinterpret_cast<uintptr_t>(X) & 15u) == 0 &&
         tma_available();
}

// Workspace: token norms [H,N] first (they only depend on H, N), then the
// per-pass centroid copies and table, the bounds with the list counters right
// behind them (cleared together), and the lists of rows for the float64
// passes: two-candidate rows {h, row, c1, c2}, full-scan rows per head.
struct TcWs {
  float* xn;
  bf16* cb;
  int2* table;
  float* centT;
  Bounds* bd;
  int* counts;  // [0] two-candidate rows, [1 + h] full-scan rows of head h
  int4* list2;
  int* list_full;  // [H][N]
  float* part;     // [3][H][N] top three between centroid segments (segmented shapes only)
};

static size_t zeroed_bytes(int H) { return sizeof(Bounds) * H + sizeof(int) * ((size_t)H + 1); }

static size_t tc_layout(int H, int N, int d, int C, TcWs* out, void* ws) {
  Carve cv(ws);
  const int Cpad = round16(C), Cr = round128(C);
  TcWs w;
  w.xn = cv.take<float>((size_t)H * N);
  w.cb = cv.take<bf16>((size_t)H * Cr * d);
  w.table = cv.take<int2>((size_t)H * Cpad);
  w.centT = cv.take<float>((size_t)H * d * C);
  char* z = cv.take<char>(zeroed_bytes(H));
  w.bd = reinterpret_cast<Bounds*>(z);
  w.counts = z ? reinterpret_cast<int*>(z + sizeof(Bounds) * H) : nullptr;
  w.list2 = cv.take<int4>((size_t)H * N);
  w.list_full = cv.take<int>((size_t)H * N);
  w.part = segmented(d, C) ? cv.take<float>((size_t)3 * H * N) : nullptr;
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
  const int rpb = 8 * (256 / d);  // rows per block and pass: 8 warps x 32/(d/8)
  const unsigned grid = (unsigned)std::min<long long>((rows + rpb - 1) / rpb, 148LL * 16);
  if (d == 128) { k_row_norms<128><<<grid, 256, 0, st>>>(X, rows, xn); note_launch(); }
  else { k_row_norms<64><<<grid, 256, 0, st>>>(X, rows, xn); note_launch(); }
  return cudaGetLastError();
}

// Tiles per block: the count that minimises (waves of 148 blocks) x (tiles per
// block + a setup cost of about three tiles).
static int pick_tiles_per_cta(int H, int T) {
  int best = 1;
  long long best_cost = LLONG_MAX;
  for (int tpc = 4; tpc <= 64; ++tpc) {
    const long long ctas = (long long)H * ((T + tpc - 1) / tpc);
    const long long cost = ((ctas + 147) / 148) * (tpc + 3);
    if (cost < best_cost) { best_cost = cost; best = tpc; }
  }
  return std::min(best, std::max(1, T));
}

template <int D>
static cudaError_t assign_launch(const bf16* X, int H, int N, int C, const float* cent, int32_t* labels,
                                 const TcWs& w, cudaStream_t st) {
  const int Cpad = round16(C), Cr = round128(C);
  const int seg = segment_cols(D, C);
  if (seg < kChunk || (seg < Cpad && !w.part)) return cudaErrorInvalidValue;
  int nbits = 1;
  while ((1 << nbits) < Cpad) ++nbits;
  k_prep_centroids<D><<<dim3(Cr / 32, H), 256, 0, st>>>(cent, C, Cpad, Cr, w.cb, w.table, w.centT, w.bd);
  note_launch();
  CUtensorMap tmx, tmc;
  if (!tma_map_bf16_3d(&tmx, X, D, N, H, BM) || !tma_map_bf16_3d(&tmc, w.cb, D, Cr, H, 128))
    return cudaErrorInvalidValue;
  const int T = (N + BM - 1) / BM;
  const int tpc = pick_tiles_per_cta(H, T);
  for (int c_base = 0; c_base < Cpad; c_base += seg) {
    const int sp = std::min(seg, Cpad - c_base), sr = round128(sp);
    const int stages = pick_stages(D, sr, sp);
    const int pmode = (c_base > 0 ? 1 : 0) | (c_base + seg < Cpad ? 2 : 0);
    const int smem = layout(D, sr, sp, stages).total;
    cudaError_t e = cudaFuncSetAttribute(k_assign_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_assign_tc<D><<<dim3((T + tpc - 1) / tpc, H), kThreads, smem, st>>>(
        tmx, tmc, w.table, w.bd, w.xn, N, sp, sr, stages, tpc, nbits, labels, w.list2, w.list_full,
        w.counts, status_word(), Cpad, c_base, w.part, pmode);
    note_launch();
  }
  k_refine2<D><<<148 * 4, 256, 0, st>>>(X, cent, N, C, w.list2, w.counts, labels);
  note_launch();
  const int fthreads = C > kFullThreads ? kFullThreads : (C + 31) / 32 * 32;
  const int fgx = std::max(1, (148 * 8 + H - 1) / H);
  k_refine_full<D><<<dim3(fgx, H), fthreads, 0, st>>>(X, cent, w.centT, N, C, w.list_full, w.counts + 1,
                                                       labels);
  note_launch();
  return cudaGetLastError();
}

cudaError_t kmeans_assign_tc(const void* Xv, int H, int N, int d, int C, const float* cent,
                             int32_t* labels, void* ws, cudaStream_t st) {
  TcWs w;
  tc_layout(H, N, d, C, &w, ws);
  cudaError_t e = cudaMemsetAsync(w.bd, 0, zeroed_bytes(H), st);
  if (e != cudaSuccess) return e;
  const bf16* X = static_cast<const bf16*>(Xv);
  if (d == 128) return assign_launch<128>(X, H, N, C, cent, labels, w, st);
  return assign_launch<64>(X, H, N, C, cent, labels, w, st);
}

}  // namespace svg
