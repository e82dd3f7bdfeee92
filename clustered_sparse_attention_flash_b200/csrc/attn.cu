// Hybrid attention (SVG-EAR review, step (4); gist.science summary 2.A
// "lineare Kompensation"): for query i of cluster a,
//   o_i = [ sum_{c routed} sum_{j in c} e^{s q_i.k_j} v_j
//         + sum_{c compensated, |k_c|>0} |k_c| e^{s q_i.kbar_c} vbar_c ]
//       / [ the same sums without v ]
// evaluated as one online softmax over the routed keys followed by the
// centroid "keys" with logit bias log|k_c|; o_i goes to row perm_q[i].
//
// This file holds the CUDA-core kernel used for float32 inputs (and as the
// scaffold for bf16): 64 query rows per block, two threads per row.  The bf16
// tensor-core kernel lives in attn_tc.cu.
#include "common.cuh"
#include "internal.h"
#include "attn_tc.cuh"

namespace svg {

namespace {

constexpr int kBQ = 64;  // query rows per block of the CUDA-core kernel

// Tile table: per head, the (query cluster, first row) of every block; query
// tiles never straddle two clusters.
__global__ void k_tile_table(const int32_t* __restrict__ q_off, int Cq, int BQ, int tmax,
                             int2* __restrict__ tiles, int32_t* __restrict__ ntiles) {
  __shared__ int32_t wtot[32];
  __shared__ int32_t carry;
  const int h = blockIdx.x;
  const int32_t* off = q_off + (size_t)h * (Cq + 1);
  int2* tt = tiles + (size_t)h * tmax;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int a0 = 0; a0 < Cq; a0 += blockDim.x) {
    const int a = a0 + threadIdx.x;
    int n = 0, beg = 0;
    if (a < Cq) {
      beg = off[a];
      n = (off[a + 1] - beg + BQ - 1) / BQ;
    }
    int v = n;
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) wtot[w] = v;
    __syncthreads();
    if (w == 0) {
      int t = (lane < (int)(blockDim.x >> 5)) ? wtot[lane] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += u;
      }
      wtot[lane] = t;
    }
    __syncthreads();
    const int start = carry + v - n + (w > 0 ? wtot[w - 1] : 0);
    for (int t = 0; t < n; ++t) tt[start + t] = make_int2(a, beg + t * BQ);
    __syncthreads();
    if (threadIdx.x == 0) carry += wtot[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) ntiles[h] = carry;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) k_attn_simt(const T* __restrict__ Qp, const T* __restrict__ Kp,
                                                   const T* __restrict__ Vp, const int32_t* __restrict__ q_off,
                                                   const int32_t* __restrict__ k_off,
                                                   const int32_t* __restrict__ perm_q,
                                                   const float* __restrict__ Kbar, const float* __restrict__ Vbar,
                                                   const int32_t* __restrict__ sel, const int32_t* __restrict__ n_sel,
                                                   const int2* __restrict__ tiles, const int32_t* __restrict__ ntiles,
                                                   int tmax, int Nq, int Nk, int Cq, int Ck, float scale,
                                                   T* __restrict__ O) {
  constexpr int HALF = D / 2, KT = 32;
  __shared__ __align__(16) float ks[KT][D];
  __shared__ __align__(16) float vs[KT][D];
  __shared__ float bias[KT];
  __shared__ uint32_t routed_bits[kMaxCkBits / 32];
  const int h = blockIdx.y;
  if ((int)blockIdx.x >= ntiles[h]) return;
  const int2 tile = tiles[(size_t)h * tmax + blockIdx.x];
  const int a = tile.x;
  const int qend = q_off[(size_t)h * (Cq + 1) + a + 1];
  const int row = tile.y + (threadIdx.x >> 1);
  const int part = threadIdx.x & 1;
  const bool act = row < qend;
  float q[HALF], o[HALF];
  {
    const T* qr = Qp + ((size_t)h * Nq + (act ? row : tile.y)) * D + part * HALF;
#pragma unroll
    for (int t = 0; t < HALF; ++t) { q[t] = to_f(qr[t]) * scale; o[t] = 0.f; }
  }
  float m = -INFINITY, l = 0.f;
  const int32_t* koff = k_off + (size_t)h * (Ck + 1);
  const int ns = n_sel[(size_t)h * Cq + a];
  const int32_t* sl = sel + ((size_t)h * Cq + a) * Ck;
  for (int i = threadIdx.x; i < (Ck + 31) / 32; i += blockDim.x) routed_bits[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < ns; i += blockDim.x) atomicOr(&routed_bits[sl[i] >> 5], 1u << (sl[i] & 31));

  auto consume = [&](int nk, bool with_bias) {
    for (int r = 0; r < nk; ++r) {
      float s = 0.f;
#pragma unroll
      for (int t = 0; t < HALF; ++t) s = fmaf(q[t], ks[r][part * HALF + t], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      if (with_bias) s += bias[r];
      if (s == -INFINITY) continue;
      if (s > m) {
        const float rs = expf(m - s);
        l *= rs;
#pragma unroll
        for (int t = 0; t < HALF; ++t) o[t] *= rs;
        m = s;
      }
      const float p = expf(s - m);
      l += p;
#pragma unroll
      for (int t = 0; t < HALF; ++t) o[t] = fmaf(p, vs[r][part * HALF + t], o[t]);
    }
  };

  // exact keys of the routed clusters, in routing order
  const T* Kh = Kp + (size_t)h * Nk * D;
  const T* Vh = Vp + (size_t)h * Nk * D;
  for (int si = 0; si < ns; ++si) {
    const int c = sl[si];
    const int kb = koff[c], ke = koff[c + 1];
    for (int j0 = kb; j0 < ke; j0 += KT) {
      const int nk = min(KT, ke - j0);
      __syncthreads();
      for (int e = threadIdx.x; e < nk * D; e += blockDim.x) {
        const int r = e / D, t = e % D;
        ks[r][t] = to_f(Kh[(size_t)(j0 + r) * D + t]);
        vs[r][t] = to_f(Vh[(size_t)(j0 + r) * D + t]);
      }
      __syncthreads();
      consume(nk, false);
    }
  }
  // centroid compensation for every non-routed, non-empty key cluster
  const float* KBh = Kbar + (size_t)h * Ck * D;
  const float* VBh = Vbar + (size_t)h * Ck * D;
  for (int c0 = 0; c0 < Ck; c0 += KT) {
    const int nk = min(KT, Ck - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < nk * D; e += blockDim.x) {
      const int r = e / D, t = e % D;
      ks[r][t] = KBh[(size_t)(c0 + r) * D + t];
      vs[r][t] = VBh[(size_t)(c0 + r) * D + t];
    }
    for (int r = threadIdx.x; r < nk; r += blockDim.x) {
      const int c = c0 + r;
      const int n = koff[c + 1] - koff[c];
      const bool routed = (routed_bits[c >> 5] >> (c & 31)) & 1u;
      bias[r] = (n > 0 && !routed) ? logf((float)n) : -INFINITY;
    }
    __syncthreads();
    consume(nk, true);
  }
  if (act) {
    const float inv = 1.f / l;
    T* orow = O + ((size_t)h * Nq + perm_q[(size_t)h * Nq + row]) * D + part * HALF;
#pragma unroll
    for (int t = 0; t < HALF; ++t) orow[t] = from_f<T>(o[t] * inv);
  }
}

template <typename T, int D>
void launch_simt(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                 const int32_t* k_off, const int32_t* perm_q, const float* Kbar, const float* Vbar,
                 const int32_t* sel, const int32_t* n_sel, const int2* tiles, const int32_t* ntiles,
                 int tmax, int H, int Nq, int Nk, int Cq, int Ck, float scale, void* O, cudaStream_t st) {
  k_attn_simt<T, D><<<dim3(tmax, H), 2 * kBQ, 0, st>>>(
      static_cast<const T*>(Qp), static_cast<const T*>(Kp), static_cast<const T*>(Vp), q_off, k_off,
      perm_q, Kbar, Vbar, sel, n_sel, tiles, ntiles, tmax, Nq, Nk, Cq, Ck, scale, static_cast<T*>(O)); note_launch();
}

}  // namespace

size_t attn_ws_bytes(int H, int Nq, int Nk, int d, int Cq, int Ck) {
  Carve cv(nullptr);
  const int tmax = (Nq + kBQ - 1) / kBQ + Cq;
  cv.take<int2>((size_t)H * tmax);
  cv.take<int32_t>(H);
  cv.take<char>(attn_tc_ws_bytes(H, Nq, Nk, d, Cq, Ck));
  return cv.used();
}

cudaError_t attn_run(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                     const int32_t* k_off, const int32_t* perm_q, const float* Kbar,
                     const float* Vbar, const int32_t* sel, const int32_t* n_sel, int dtype,
                     int H, int Nq, int Nk, int d, int Cq, int Ck, float scale, void* O,
                     void* ws, cudaStream_t st) {
  Carve cv(ws);
  const int tmax = (Nq + kBQ - 1) / kBQ + Cq;
  int2* tiles = cv.take<int2>((size_t)H * tmax);
  int32_t* ntiles = cv.take<int32_t>(H);
  void* tcws = cv.take<char>(attn_tc_ws_bytes(H, Nq, Nk, d, Cq, Ck));
  if (dtype == DT_BF16 && attn_tc_supported(d, Ck))
    return attn_tc_run(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, H, Nq, Nk, d, Cq,
                       Ck, scale, O, tcws, st);
  k_tile_table<<<H, 1024, 0, st>>>(q_off, Cq, kBQ, tmax, tiles, ntiles); note_launch();
  if (dtype == DT_BF16) {
    if (d == 128) launch_simt<bf16, 128>(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, tiles, ntiles, tmax, H, Nq, Nk, Cq, Ck, scale, O, st);
    else launch_simt<bf16, 64>(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, tiles, ntiles, tmax, H, Nq, Nk, Cq, Ck, scale, O, st);
  } else {
    if (d == 128) launch_simt<float, 128>(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, tiles, ntiles, tmax, H, Nq, Nk, Cq, Ck, scale, O, st);
    else launch_simt<float, 64>(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, tiles, ntiles, tmax, H, Nq, Nk, Cq, Ck, scale, O, st);
  }
  return cudaGetLastError();
}

}  // namespace svg
