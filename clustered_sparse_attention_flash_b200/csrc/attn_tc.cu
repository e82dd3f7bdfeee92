// Tensor-core hybrid attention for bf16 (SVG-EAR review, step (4); gist.science
// summary 2.A): exact softmax attention over the keys of the routed key
// clusters and centroid compensation for every other non-empty key cluster,
// in one online softmax:
//   o_i = [ sum_{j routed} e^{s q_i.k_j} v_j + sum_{c comp} |k_c| e^{s q_i.kbar_c} vbar_c ]
//       / [ the same without v ],
// written to row perm_q[i] of the output.
//
// One block per 128-row query tile; tiles never straddle two query clusters,
// so all rows of a tile share one key stream:
//   * exact part: the rows of the routed clusters (routing order),
//     concatenated and cut into 128-key tiles (the last one masked),
//   * compensation part: all key centroids in 128-row tiles, logit bias
//     log2|k_c| (in base-2 units) or -inf when c is routed or empty.  The
//     float32 centroids enter as bf16 hi + lo pairs (two MMAs each for S and
//     for P.V), so their rounding stays near 2^-17 instead of 2^-9; such a
//     tile occupies both ring stages (hi, then lo).
// Warp roles (8 warps):
//   warp 0      tensor-memory allocation, MMA issue (one thread):
//               S_j = Q K_j^T into one of two S buffers, O += P_j V_j with P
//               read from tensor memory;
//   warps 1-3   producers: cp.async gathers of Q, K_j, V_j rows into the
//               128-byte-swizzled layout (two-stage ring), bias vectors;
//               named barriers 2 and 3 order them among themselves;
//   warps 4-7   softmax (thread = query row): row max, lazy rescale of O
//               when the max grows by more than 2^8, P = 2^(x - m) in bf16
//               into tensor memory, final O / l and the permuted store.
// Every decision that guards a warp-collective tensor-memory access is made
// warp-uniform, and every wait is time-bounded (device status word on expiry).
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O [256,384)
// P0 [384,448) P1 [448,512).
#include <algorithm>
#include <cmath>

#include "attn_tc.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace svg {

namespace {

constexpr int BQ = 128;        // query rows per tile
constexpr int BN = 128;        // keys per key tile
constexpr int kThreads = 256;
constexpr int kProducers = 96;
constexpr int kStages = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP0 = 384;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// bf16 hi/lo copies of the key / value centroids (x = hi + lo + O(2^-17 x);
// rows padded to a multiple of 128 with zeros) and log2 of the cluster sizes
// (-inf for empty or padding).
template <int D>
__global__ void k_prep_comp(const float* __restrict__ Kbar, const float* __restrict__ Vbar,
                            const int32_t* __restrict__ k_off, int Ck, int Ckpad, bf16* __restrict__ kh,
                            bf16* __restrict__ kl, bf16* __restrict__ vh, bf16* __restrict__ vl,
                            float* __restrict__ lc2) {
  const int h = blockIdx.y, c = blockIdx.x;
  const bool ok = c < Ck;
  for (int t = threadIdx.x; t < D; t += blockDim.x) {
    const size_t src = ((size_t)h * Ck + c) * D + t, dst = ((size_t)h * Ckpad + c) * D + t;
    const float k = ok ? Kbar[src] : 0.f, v = ok ? Vbar[src] : 0.f;
    const bf16 k1 = __float2bfloat16_rn(k), v1 = __float2bfloat16_rn(v);
    kh[dst] = k1;
    kl[dst] = __float2bfloat16_rn(k - __bfloat162float(k1));
    vh[dst] = v1;
    vl[dst] = __float2bfloat16_rn(v - __bfloat162float(v1));
  }
  if (threadIdx.x == 0) {
    int n = 0;
    if (ok) n = k_off[(size_t)h * (Ck + 1) + c + 1] - k_off[(size_t)h * (Ck + 1) + c];
    lc2[(size_t)h * Ckpad + c] = n > 0 ? log2f((float)n) : -INFINITY;
  }
}

// Per head: (query cluster, first row) of every 128-row tile.
__global__ void k_tile_table_tc(const int32_t* __restrict__ q_off, int Cq, int tmax,
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
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) wtot[w] = v;
    __syncthreads();
    if (w == 0) {
      int t = (lane < (int)(blockDim.x >> 5)) ? wtot[lane] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, t, o);
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

template <int D>
struct AttnSmem {
  static constexpr int kTile = BN * D * 2;  // one bf16 operand tile (128 rows)
  static constexpr int q_off = 0;
  static constexpr int k_off = q_off + kTile;
  static constexpr int v_off = k_off + kStages * kTile;
  static constexpr int idx_off = v_off + kStages * kTile;
  static constexpr int bias_off = idx_off + kStages * BN * 4;
  static constexpr int flag_off = bias_off + kStages * BN * 4;
  static constexpr int bits_off = flag_off + 64;
  static constexpr int bar_off = bits_off + kMaxCkBits / 8;
  static constexpr int total = bar_off + 32 * 8 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(const bf16* __restrict__ Qp, const bf16* __restrict__ Kp, const bf16* __restrict__ Vp,
              const int32_t* __restrict__ q_off, const int32_t* __restrict__ k_off,
              const int32_t* __restrict__ perm_q, const bf16* __restrict__ kb_hi,
              const bf16* __restrict__ kb_lo, const bf16* __restrict__ vb_hi, const bf16* __restrict__ vb_lo,
              const float* __restrict__ lc2, const int32_t* __restrict__ sel,
              const int32_t* __restrict__ n_sel, const int2* __restrict__ tiles,
              const int32_t* __restrict__ ntiles, int tmax, int Nq, int Nk, int Cq, int Ck, int Ckpad,
              float scale2, bf16* __restrict__ O, int* status) {
  using S = AttnSmem<D>;
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  const int h = blockIdx.y;
  if ((int)blockIdx.x >= ntiles[h]) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int* idx_s = reinterpret_cast<int*>(smem + S::idx_off);         // [stage][128] source rows
  float* bias_s = reinterpret_cast<float*>(smem + S::bias_off);   // [stage][128] log2 biases
  int* flag_s = reinterpret_cast<int*>(smem + S::flag_off);       // [stage]: 1 = apply bias
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + S::bits_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::bar_off);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_free = bars + 7;    // [2]
  uint64_t* p_full = bars + 9;    // [2]
  uint64_t* p_free = bars + 11;   // [2]
  uint64_t* done = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);

  const int2 tile = tiles[(size_t)h * tmax + blockIdx.x];
  const int a = tile.x, r0 = tile.y;
  const int qend = q_off[(size_t)h * (Cq + 1) + a + 1];
  const int ns = n_sel[(size_t)h * Cq + a];
  const int32_t* sl = sel + ((size_t)h * Cq + a) * Ck;
  const int32_t* koff = k_off + (size_t)h * (Ck + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // routed clusters of this query cluster as a bit set; total routed keys
  for (int i = threadIdx.x; i < (Ck + 31) / 32; i += blockDim.x) bits[i] = 0;
  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, kProducers);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(kv_full + i, kProducers);
      tc::mbar_init(kv_empty + i, 1);
      tc::mbar_init(s_full + i, 1);
      tc::mbar_init(s_free + i, 128);
      tc::mbar_init(p_full + i, 128);
      tc::mbar_init(p_free + i, 1);
    }
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  __syncthreads();
  long long lex_part = 0;
  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const int c = sl[i];
    atomicOr(&bits[c >> 5], 1u << (c & 31));
    lex_part += koff[c + 1] - koff[c];
  }
  // block-wide sum of routed keys (every thread needs the tile count)
  for (int o = 16; o > 0; o >>= 1) lex_part += __shfl_xor_sync(0xffffffffu, lex_part, o);
  __shared__ long long lex_w[8];
  if (lane == 0) lex_w[warp] = lex_part;
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  long long lex = 0;
  for (int i = 0; i < 8; ++i) lex += lex_w[i];
  const uint32_t tmem = *tmem_slot;
  const int n_ex = (int)((lex + BN - 1) / BN);
  const int n_cp = Ckpad / BN;
  const int ntile = n_ex + n_cp;
  // ring-stage sequence: an exact tile uses one stage, a compensation tile two
  auto ustart = [&](int j) { return j <= n_ex ? j : n_ex + 2 * (j - n_ex); };
  auto nparts = [&](int j) { return j < n_ex ? 1 : 2; };

  if (warp == 0) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t qa = tc::smem_u32(smem + S::q_off);
      const uint32_t id_s = tc::idesc_bf16(BQ, BN, false, false);
      const uint32_t id_o = tc::idesc_bf16(BQ, D, false, true);
      bool ok = tc::mbar_wait(q_full, 0, abort_flag, status);
      auto issue_s = [&](int j) -> bool {
        const int b = j & 1, u0 = ustart(j), np = nparts(j);
        if (!tc::mbar_wait(s_free + b, ((j >> 1) & 1) ^ 1, abort_flag, status)) return false;
        for (int p = 0; p < np; ++p) {
          const int u = u0 + p, st = u % kStages;
          if (!tc::mbar_wait(kv_full + st, (u / kStages) & 1, abort_flag, status)) return false;
          tc::tc_fence_after();
          const uint32_t ka = tc::smem_u32(smem + S::k_off + st * S::kTile);
          for (int k = 0; k < D / 16; ++k)
            tc::mma_ss(tmem + kColS0 + (uint32_t)b * BN, tc::desc_kmajor(qa, BQ * 128u, k),
                       tc::desc_kmajor(ka, BN * 128u, k), id_s, (p > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(s_full + b);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int b = j & 1, u0 = ustart(j), np = nparts(j);
        if (!tc::mbar_wait(p_full + b, (j >> 1) & 1, abort_flag, status)) return false;
        tc::tc_fence_after();
        for (int p = 0; p < np; ++p) {
          const int st = (u0 + p) % kStages;
          const uint32_t va = tc::smem_u32(smem + S::v_off + st * S::kTile);
          for (int k = 0; k < BN / 16; ++k)
            tc::mma_ts(tmem + kColO, tmem + kColP0 + (uint32_t)b * 64u + (uint32_t)k * 8u,
                       tc::desc_mnmajor(va, BN * 128u, k), id_o, (j > 0 || p > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(p_free + b);
        for (int p = 0; p < np; ++p) tc::mma_commit(kv_empty + (u0 + p) % kStages);
        return true;
      };
      if (ok && ntile > 0) ok = issue_s(0);
      for (int j = 0; ok && j < ntile; ++j) {
        // S_{j+1} goes ahead of P_j.V_j when its stages are already free; a
        // two-stage tile needs the stage P_j.V_j still reads
        const bool next = j + 1 < ntile;
        const bool early = next && nparts(j + 1) == 1;
        if (early && !issue_s(j + 1)) break;
        if (!issue_pv(j)) break;
        if (next && !early && !issue_s(j + 1)) break;
      }
      tc::mma_commit(done);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ producers
    const int pt = threadIdx.x - 32;
    const bf16* Qh = Qp + (size_t)h * Nq * D;
    {
      const uint32_t qa = tc::smem_u32(smem + S::q_off);
      for (int e = pt; e < BQ * CPR; e += kProducers) {
        const int r = e / CPR, c = e % CPR;
        const bool valid = r0 + r < Nq;
        tc::cp_async16(qa + tc::sw128_offset(r, c, BQ), Qh + (size_t)(valid ? r0 + r : 0) * D + c * 8,
                       valid ? 16u : 0u);
      }
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
      tc::mbar_arrive(q_full);
    }
    const bf16* Kh = Kp + (size_t)h * Nk * D;
    const bf16* Vh = Vp + (size_t)h * Nk * D;
    const float* LC = lc2 + (size_t)h * Ckpad;
    int ri = 0, ro = 0;  // cursor into the routed ranges (warp 1 only)
    for (int j = 0; j < ntile; ++j) {
      const bool exact = j < n_ex;
      const int u0 = ustart(j);
      for (int p = 0; p < nparts(j); ++p) {
        const int u = u0 + p, st = u % kStages;
        const bool got = tc::mbar_wait(kv_empty + st, ((u / kStages) & 1) ^ 1, abort_flag, status);
        if (!tc::bar_and(3, kProducers, got)) { j = ntile; break; }  // all producers leave together
        int* idx = idx_s + st * BN;
        float* bias = bias_s + st * BN;
        if (warp == 1) {
          if (exact) {
            int fill = 0;
            while (fill < BN && ri < ns) {
              const int c = sl[ri];
              const int cb = koff[c], clen = koff[c + 1] - cb;
              const int take = min(clen - ro, BN - fill);
              for (int i = lane; i < take; i += 32) idx[fill + i] = cb + ro + i;
              fill += take;
              ro += take;
              if (ro == clen) { ++ri; ro = 0; }
            }
            for (int i = fill + lane; i < BN; i += 32) idx[i] = -1;
            for (int i = lane; i < BN; i += 32) bias[i] = i < fill ? 0.f : -INFINITY;
            if (lane == 0) flag_s[st] = fill < BN ? 1 : 0;
          } else {
            const int c0 = (j - n_ex) * BN;
            for (int i = lane; i < BN; i += 32) {
              const int c = c0 + i;
              idx[i] = c;
              const bool routed = c < Ck && ((bits[c >> 5] >> (c & 31)) & 1u);
              bias[i] = routed ? -INFINITY : LC[c];
            }
            if (lane == 0) flag_s[st] = 1;
          }
        }
        asm volatile("bar.sync 2, 96;" ::: "memory");
        const uint32_t ka = tc::smem_u32(smem + S::k_off + st * S::kTile);
        const uint32_t va = tc::smem_u32(smem + S::v_off + st * S::kTile);
        const size_t cbase = (size_t)h * Ckpad * D;
        const bf16* ksrc = exact ? Kh : (p == 0 ? kb_hi : kb_lo) + cbase;
        const bf16* vsrc = exact ? Vh : (p == 0 ? vb_hi : vb_lo) + cbase;
        for (int e = pt; e < BN * CPR; e += kProducers) {
          const int r = e / CPR, c = e % CPR;
          const int row = idx[r];
          const uint32_t nb = row >= 0 ? 16u : 0u;
          const size_t off = (size_t)(row >= 0 ? row : 0) * D + c * 8;
          const uint32_t so = tc::sw128_offset(r, c, BN);
          tc::cp_async16(ka + so, ksrc + off, nb);
          tc::cp_async16(va + so, vsrc + off, nb);
        }
        tc::cp_async_wait_all();
        tc::fence_proxy_async();
        tc::mbar_arrive(kv_full + st);
      }
    }
    tc::cp_async_wait_all();
  } else {
    // -------------------------------------------------------------- softmax
    const int r = ((warp & 3) << 5) + lane;  // tile row == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < ntile; ++j) {
      const int u0 = ustart(j), st = u0 % kStages, b = j & 1;
      if (!tc::mbar_wait_warp(s_full + b, (j >> 1) & 1, abort_flag, status)) { ok = false; break; }
      tc::tc_fence_after();
      float x[BN];
      {
        uint32_t v[32];
#pragma unroll
        for (int q = 0; q < BN / 32; ++q) {
          tc::tmem_ld32(tmem + lane_base + kColS0 + (uint32_t)b * BN + (uint32_t)q * 32u, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) x[q * 32 + i] = __uint_as_float(v[i]) * scale2;
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(s_free + b);
      // bias / mask of this stage: acquire the producers' writes through the
      // stage's full barrier (its next phase needs this thread's P_j first)
      if (!tc::mbar_wait_warp(kv_full + st, (u0 / kStages) & 1, abort_flag, status)) { ok = false; break; }
      if (flag_s[st]) {
        const float* bias = bias_s + st * BN;
#pragma unroll
        for (int i = 0; i < BN; i += 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(bias + i);
          x[i] += b4.x; x[i + 1] += b4.y; x[i + 2] += b4.z; x[i + 3] += b4.w;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < BN; ++i) mx = fmaxf(mx, x[i]);
      // lazy rescale: a row whose maximum grew by more than 2^8 rescales O and
      // l.  The tensor-memory accesses are warp-collective, so the warp
      // rescales together (factor 1 for rows that do not need it).
      const bool grow = mx > m_used + 8.f;
      const bool has_o = j > 0 && m_used > -INFINITY;
      if (__any_sync(0xffffffffu, grow && has_o)) {
        const int pb = (j - 1) & 1;
        if (!tc::mbar_wait_warp(p_free + pb, ((j - 1) >> 1) & 1, abort_flag, status)) { ok = false; break; }
        tc::tc_fence_after();
        const float f = (grow && has_o) ? ex2(m_used - mx) : 1.f;
#pragma unroll
        for (int q = 0; q < D / 16; ++q) {
          uint32_t ov[16];
          tc::tmem_ld16(tmem + lane_base + kColO + (uint32_t)q * 16u, ov);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
          tc::tmem_st16(tmem + lane_base + kColO + (uint32_t)q * 16u, ov);
        }
        tc::tmem_st_wait();
        l *= f;
      }
      if (grow) m_used = mx;
      const float mref = m_used == -INFINITY ? 0.f : m_used;
      // P must not overwrite the buffer PV_{j-2} is still reading
      if (!tc::mbar_wait_warp(p_free + b, ((j >> 1) & 1) ^ 1, abort_flag, status)) { ok = false; break; }
      tc::tc_fence_after();
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < BN / 32; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(x[q * 32 + 2 * i] - mref), p1 = ex2(x[q * 32 + 2 * i + 1] - mref);
          rs += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
        tc::tmem_st16(tmem + lane_base + kColP0 + (uint32_t)b * 64u + (uint32_t)q * 16u, pk);
      }
      tc::tmem_st_wait();
      l += rs;
      tc::tc_fence_before();
      tc::mbar_arrive(p_full + b);
    }
    // epilogue: wait for the last PV, normalise, store through perm_q
    if (ok && ntile > 0) {
      const int jl = ntile - 1;
      ok = tc::mbar_wait_warp(p_free + (jl & 1), (jl >> 1) & 1, abort_flag, status);
    }
    if (ok && ntile > 0) {
      tc::tc_fence_after();
      const int row = r0 + r;
      const bool valid = row < qend;
      const float inv = 1.f / l;
      bf16* orow = O + ((size_t)h * Nq + (valid ? perm_q[(size_t)h * Nq + row] : 0)) * D;
#pragma unroll
      for (int q = 0; q < D / 16; ++q) {
        uint32_t ov[16];
        tc::tmem_ld16(tmem + lane_base + kColO + (uint32_t)q * 16u, ov);
        tc::tmem_ld_wait();
        uint4 w0, w1;
        w0.x = pack_bf16(__uint_as_float(ov[0]) * inv, __uint_as_float(ov[1]) * inv);
        w0.y = pack_bf16(__uint_as_float(ov[2]) * inv, __uint_as_float(ov[3]) * inv);
        w0.z = pack_bf16(__uint_as_float(ov[4]) * inv, __uint_as_float(ov[5]) * inv);
        w0.w = pack_bf16(__uint_as_float(ov[6]) * inv, __uint_as_float(ov[7]) * inv);
        w1.x = pack_bf16(__uint_as_float(ov[8]) * inv, __uint_as_float(ov[9]) * inv);
        w1.y = pack_bf16(__uint_as_float(ov[10]) * inv, __uint_as_float(ov[11]) * inv);
        w1.z = pack_bf16(__uint_as_float(ov[12]) * inv, __uint_as_float(ov[13]) * inv);
        w1.w = pack_bf16(__uint_as_float(ov[14]) * inv, __uint_as_float(ov[15]) * inv);
        if (valid) {
          reinterpret_cast<uint4*>(orow + q * 16)[0] = w0;
          reinterpret_cast<uint4*>(orow + q * 16)[1] = w1;
        }
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

int round128(int x) { return (x + 127) / 128 * 128; }

struct AttnWs {
  bf16 *kh, *kl, *vh, *vl;
  float* lc2;
  int2* tiles;
  int32_t* ntiles;
};

size_t attn_layout(int H, int Nq, int d, int Cq, int Ck, AttnWs* out, void* ws) {
  Carve cv(ws);
  const int Ckpad = round128(Ck);
  const int tmax = (Nq + BQ - 1) / BQ + Cq;
  AttnWs w;
  w.kh = cv.take<bf16>((size_t)H * Ckpad * d);
  w.kl = cv.take<bf16>((size_t)H * Ckpad * d);
  w.vh = cv.take<bf16>((size_t)H * Ckpad * d);
  w.vl = cv.take<bf16>((size_t)H * Ckpad * d);
  w.lc2 = cv.take<float>((size_t)H * Ckpad);
  w.tiles = cv.take<int2>((size_t)H * tmax);
  w.ntiles = cv.take<int32_t>(H);
  if (out) *out = w;
  return cv.used();
}

template <int D>
cudaError_t launch(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off, const int32_t* k_off,
                   const int32_t* perm_q, const float* Kbar, const float* Vbar, const int32_t* sel,
                   const int32_t* n_sel, int H, int Nq, int Nk, int Cq, int Ck, float scale, void* O,
                   void* ws, cudaStream_t st) {
  AttnWs w;
  attn_layout(H, Nq, D, Cq, Ck, &w, ws);
  const int Ckpad = round128(Ck);
  const int tmax = (Nq + BQ - 1) / BQ + Cq;
  k_prep_comp<D><<<dim3(Ckpad, H), 64, 0, st>>>(Kbar, Vbar, k_off, Ck, Ckpad, w.kh, w.kl, w.vh, w.vl, w.lc2);
  note_launch();
  k_tile_table_tc<<<H, 1024, 0, st>>>(q_off, Cq, tmax, w.tiles, w.ntiles); note_launch();
  const int smem = AttnSmem<D>::total;
  cudaError_t e = cudaFuncSetAttribute(k_attn_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k_attn_tc<D><<<dim3(tmax, H), kThreads, smem, st>>>(
      static_cast<const bf16*>(Qp), static_cast<const bf16*>(Kp), static_cast<const bf16*>(Vp), q_off, k_off,
      perm_q, w.kh, w.kl, w.vh, w.vl, w.lc2, sel, n_sel, w.tiles, w.ntiles, tmax, Nq, Nk, Cq, Ck, Ckpad, scale * kLog2e,
      static_cast<bf16*>(O), status_word());
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(int d, int Ck) { return (d == 64 || d == 128) && Ck <= kMaxCkBits; }

size_t attn_tc_ws_bytes(int H, int Nq, int d, int Cq, int Ck) {
  if (!attn_tc_supported(d, Ck)) return 0;
  return attn_layout(H, Nq, d, Cq, Ck, nullptr, nullptr);
}

cudaError_t attn_tc_run(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                        const int32_t* k_off, const int32_t* perm_q, const float* Kbar,
                        const float* Vbar, const int32_t* sel, const int32_t* n_sel, int H, int Nq,
                        int Nk, int d, int Cq, int Ck, float scale, void* O, void* ws,
                        cudaStream_t st) {
  if (d == 128)
    return launch<128>(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, H, Nq, Nk, Cq, Ck, scale, O, ws, st);
  return launch<64>(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, H, Nq, Nk, Cq, Ck, scale, O, ws, st);
}

}  // namespace svg
