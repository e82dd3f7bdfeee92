// Tensor-core hybrid attention for bf16 (SVG-EAR review, step (4); gist.science
// summary 2.A): exact softmax attention over the keys of the routed key
// clusters and centroid compensation for every other non-empty key cluster,
// in one online softmax:
//   o_i = [ sum_{j routed} e^{s q_i.k_j} v_j + sum_{c comp} |k_c| e^{s q_i.kbar_c} vbar_c ]
//       / [ the same without v ],
// written to row perm_q[i] of the output.
//
// One block per pair of 128-row query tiles of one query cluster (256
// consecutive rows of the cluster; tiles never straddle clusters, so both
// tiles share one key stream and every key / value stage is used by both):
//   * exact part: the rows of the routed clusters (routing order),
//     concatenated and cut into 128-key tiles (the last one masked),
//   * compensation part: all key centroids in 128-row tiles, logit bias
//     log2|k_c| (in base-2 units) or -inf when c is routed or empty.  The
//     float32 centroids enter as bf16 hi + lo pairs (two MMAs each for S and
//     for P.V), so their rounding stays near 2^-17 instead of 2^-9; such a
//     tile occupies two ring stages (hi, then lo).
// Keys and values are staged in an "8-row group" layout (each key cluster
// padded to a multiple of 8 rows, each group of 8 rows stored as
// [16-byte chunk][row]), which is directly a no-swizzle UMMA operand (K-major
// for K, MN-major for V); a stage is one or a few contiguous runs, each moved
// by a single cp.async.bulk.  K and V each have a two-slot ring: a K slot is
// free once S of its stage is computed for both query tiles, a V slot once
// P.V is done for both tiles.  The stage's bias vector (padding rows and
// routed centroids masked, log2|k_c| on compensated centroids) has a
// four-slot ring of its own, freed by the softmax warps once they have read
// it, so keys for later stages load while the softmax of this one runs, and a
// softmax stage never waits for the values.  Sharing each stage between two query
// tiles halves the key / value traffic from L2 per FLOP, which is what bounds
// a one-tile block.
// Warp roles (12 warps):
//   warp 0      tensor-memory allocation and the MMA issue loop (run by the
//               whole warp, one elected lane issues) in the order
//               P.V_0(j), S_0(j+1), P.V_1(j), S_1(j+1): while the tensor core
//               works for one query tile the other tile's softmax runs;
//   warps 1-3   load the two query tiles; warps 1 and 2 then produce the
//               even and the odd stages (bulk copies issued by one lane, bias
//               vectors by the warp);
//   warps 4-7   softmax of query tile 0, warps 8-11 of query tile 1 (thread =
//               query row, all 128 keys of each stage): running maximum, row
//               sum, lazy rescale of the tile's accumulator O[t] when the
//               maximum grows by more than 2^8, P = 2^(x - m) in bf16 over the
//               S columns of the tile; most routed stages take a speculative
//               pass against the running maximum with no maximum pass
//               (accepted when no term can exceed 2^16); at the end O / l is
//               stored through perm_q.
// Tensor memory (512 columns): S[t] [128 t, 128 t + 128), O[t]
// [256 + d t, 256 + d t + d); P[t] lives in the first 64 columns of S[t].
// Every decision that guards a warp-collective tensor-memory access is made
// warp-uniform, and every wait is time-bounded (device status word on expiry).
#include <algorithm>
#include <cmath>

#include "attn_tc.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace svg {

namespace {

constexpr int BQ = 128;        // rows per query tile (two tiles per block)
constexpr int BN = 128;        // keys per ring stage
constexpr int kThreads = 384;
constexpr int kProducers = 96;
constexpr int kKSlots = 2;     // K ring
constexpr int kBSlots = 4;     // bias ring
constexpr int kVSlots = 2;     // V ring
constexpr int kUnitRows = 2 * BQ;  // query rows of one block
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr int kMaxRanges = 512;  // routed clusters staged in shared memory
constexpr int kRegsLow = 48;     // MMA / producer warpgroup after the split
constexpr int kRegsHigh = 224;   // each softmax warpgroup after the split
// the split fits a launch of 168 registers per thread (checked at launch)
static_assert(4 * 32 * kRegsLow + 8 * 32 * kRegsHigh <= kThreads * 168, "register split");

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed pairs of float32 (sm_100 two-wide FMA pipe): one instruction
// applies the same operation to both halves, rounded as the scalar one.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ float f2_lo(uint64_t x) { return __uint_as_float((uint32_t)x); }
__device__ __forceinline__ float f2_hi(uint64_t x) { return __uint_as_float((uint32_t)(x >> 32)); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Byte offset of (row, 16-byte chunk) in the 8-row group layout.
template <int D>
__host__ __device__ __forceinline__ size_t g8_offset(size_t row, int chunk) {
  return (row >> 3) * (size_t)(8 * D * 2) + (size_t)chunk * 128u + (row & 7) * 16u;
}

// bf16 hi/lo copies of the key / value centroids (x = hi + lo + O(2^-17 x)),
// in the 8-row group layout with rows padded to a multiple of the stage size
// (zeros), and log2 of the cluster sizes (-inf for empty or padding).
template <int D>
__global__ void k_prep_comp(const float* __restrict__ Kbar, const float* __restrict__ Vbar,
                            const int32_t* __restrict__ k_off, int Ck, int Ckpad, uint8_t* __restrict__ kh,
                            uint8_t* __restrict__ kl, uint8_t* __restrict__ vh, uint8_t* __restrict__ vl,
                            float* __restrict__ lc2) {
  const int h = blockIdx.y, c = blockIdx.x;
  const bool ok = c < Ck;
  const size_t hb = (size_t)h * Ckpad * D * 2;
  for (int t = threadIdx.x; t < D; t += blockDim.x) {
    const size_t src = ((size_t)h * Ck + c) * D + t;
    const size_t dst = hb + g8_offset<D>(c, t >> 3) + (t & 7) * 2;
    const float k = ok ? Kbar[src] : 0.f, v = ok ? Vbar[src] : 0.f;
    const bf16 k1 = __float2bfloat16_rn(k), v1 = __float2bfloat16_rn(v);
    *reinterpret_cast<bf16*>(kh + dst) = k1;
    *reinterpret_cast<bf16*>(kl + dst) = __float2bfloat16_rn(k - __bfloat162float(k1));
    *reinterpret_cast<bf16*>(vh + dst) = v1;
    *reinterpret_cast<bf16*>(vl + dst) = __float2bfloat16_rn(v - __bfloat162float(v1));
  }
  if (threadIdx.x == 0) {
    int n = 0;
    if (ok) n = k_off[(size_t)h * (Ck + 1) + c + 1] - k_off[(size_t)h * (Ck + 1) + c];
    lc2[(size_t)h * Ckpad + c] = n > 0 ? log2f((float)n) : -INFINITY;
  }
}

// poff[h][c]: first padded row of key cluster c (sizes rounded up to 8).
__global__ void k_pad_offsets(const int32_t* __restrict__ k_off, int Ck, int32_t* __restrict__ poff) {
  __shared__ int32_t wtot[32];
  __shared__ int32_t carry;
  const int h = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int32_t* off = k_off + (size_t)h * (Ck + 1);
  int32_t* po = poff + (size_t)h * (Ck + 1);
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int c0 = 0; c0 < Ck; c0 += blockDim.x) {
    const int c = c0 + threadIdx.x;
    const int n = c < Ck ? ((off[c + 1] - off[c] + 7) & ~7) : 0;
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
    if (c < Ck) po[c] = carry + v - n + (w > 0 ? wtot[w - 1] : 0);
    __syncthreads();
    if (threadIdx.x == 0) carry += wtot[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) po[Ck] = carry;
}

// Key / value rows of cluster c (row-major, cluster order) into the padded
// 8-row group layout; padding rows are zero.
template <int D>
__global__ void k_pack(const bf16* __restrict__ Kp, const bf16* __restrict__ Vp, const int32_t* __restrict__ k_off,
                       const int32_t* __restrict__ poff, int Nk, int Ck, size_t npad, uint8_t* __restrict__ kpk,
                       uint8_t* __restrict__ vpk) {
  constexpr int CPR = D / 8;
  const int h = blockIdx.y, c = blockIdx.x;
  const int beg = k_off[(size_t)h * (Ck + 1) + c], len = k_off[(size_t)h * (Ck + 1) + c + 1] - beg;
  const int pbeg = poff[(size_t)h * (Ck + 1) + c], plen = (len + 7) & ~7;
  const size_t hb = (size_t)h * npad * D * 2;
  const uint4* ks = reinterpret_cast<const uint4*>(Kp + ((size_t)h * Nk + beg) * D);
  const uint4* vs = reinterpret_cast<const uint4*>(Vp + ((size_t)h * Nk + beg) * D);
  for (int e = threadIdx.x; e < plen * CPR; e += blockDim.x) {
    const int r = e / CPR, ch = e % CPR;
    const uint4 z = make_uint4(0, 0, 0, 0);
    const uint4 kv = r < len ? ks[(size_t)r * CPR + ch] : z;
    const uint4 vv = r < len ? vs[(size_t)r * CPR + ch] : z;
    const size_t o = hb + g8_offset<D>((size_t)(pbeg + r), ch);
    *reinterpret_cast<uint4*>(kpk + o) = kv;
    *reinterpret_cast<uint4*>(vpk + o) = vv;
  }
}

// Per head: (query cluster, first row) of every 128-row query tile.
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
      n = (off[a + 1] - beg + kUnitRows - 1) / kUnitRows;
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
    for (int t = 0; t < n; ++t) tt[start + t] = make_int2(a, beg + t * kUnitRows);
    __syncthreads();
    if (threadIdx.x == 0) carry += wtot[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) ntiles[h] = carry;
}

template <int D>
struct AttnSmem {
  static constexpr int kQTile = BQ * D * 2;   // one 128-row bf16 query tile
  static constexpr int kKTile = BN * D * 2;   // one 128-row bf16 key (or value) tile
  static constexpr int q_off = 0;                                    // [2] query tiles
  static constexpr int k_off = q_off + 2 * kQTile;                   // [kKSlots] key tiles
  static constexpr int v_off = k_off + kKSlots * kKTile;             // [kVSlots] value tiles
  static constexpr int bias_off = v_off + kVSlots * kKTile;          // [kBSlots][BN] log2 biases
  static constexpr int nv_off = bias_off + kBSlots * BN * 4;         // [kBSlots] valid keys of the stage
  static constexpr int bits_off = nv_off + 16;
  static constexpr int rng_off = bits_off + kMaxCkBits / 8;          // [3][kMaxRanges] start, prefix, len
  static constexpr int pc_off = rng_off + 3 * kMaxRanges * 4 + 16;   // [producer warp][32] piece lists
  static constexpr int bar_off = pc_off + 2 * 32 * 16;
  // at least 120 KB, so that one block (and one 512-column tensor-memory
  // allocation) lives on an SM
  static constexpr int total = bar_off + 32 * 8 + 1024 > 120 * 1024 ? bar_off + 32 * 8 + 1024 : 120 * 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(const bf16* __restrict__ Qp, const uint8_t* __restrict__ kpk, const uint8_t* __restrict__ vpk,
              size_t npad, const int32_t* __restrict__ q_off, const int32_t* __restrict__ k_off,
              const int32_t* __restrict__ poff, const int32_t* __restrict__ perm_q,
              const uint8_t* __restrict__ kb_hi, const uint8_t* __restrict__ kb_lo,
              const uint8_t* __restrict__ vb_hi, const uint8_t* __restrict__ vb_lo,
              const float* __restrict__ lc2, const int32_t* __restrict__ sel,
              const int32_t* __restrict__ n_sel, const int2* __restrict__ tiles,
              const int32_t* __restrict__ ntiles, int tmax, int Nq, int Nk, int Cq, int Ck, int Ckpad,
              float scale2, bf16* __restrict__ O, int* status) {
  using S = AttnSmem<D>;
  constexpr int CPR = D / 8;              // 16-byte chunks per row
  constexpr uint32_t kGroup = 8 * D * 2;  // bytes of one 8-row group
  constexpr int kMaxPieces = 32;          // runs per stage (one per lane)
  const int h = blockIdx.y;
  if ((int)blockIdx.x >= ntiles[h]) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + S::bias_off);
  int* nv_s = reinterpret_cast<int*>(smem + S::nv_off);
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + S::bits_off);
  int* rng_start = reinterpret_cast<int*>(smem + S::rng_off);  // first padded row of routed range i
  int* rng_cum = rng_start + kMaxRanges;                        // padded rows in ranges [0, i)
  int* rng_len = rng_cum + kMaxRanges + 4;                      // keys in range i
  int4* pieces = reinterpret_cast<int4*>(smem + S::pc_off);     // stage row group, global row, groups, valid
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::bar_off);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;     // [kKSlots]
  uint64_t* k_empty = bars + 4;    // [kKSlots]
  uint64_t* v_full = bars + 7;     // [kVSlots]
  uint64_t* v_empty = bars + 9;    // [kVSlots]
  uint64_t* s_full = bars + 11;    // [2 query tiles]
  uint64_t* p_full = bars + 13;    // [2 query tiles]
  uint64_t* o_done = bars + 15;    // [2 query tiles]
  uint64_t* done = bars + 18;
  uint64_t* b_full = bars + 19;    // [kBSlots]
  uint64_t* b_empty = bars + 23;   // [kBSlots]: read by one lane of every softmax warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 27);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 28);

  const int2 unit = tiles[(size_t)h * tmax + blockIdx.x];
  const int a = unit.x, r0 = unit.y;
  const int qend = q_off[(size_t)h * (Cq + 1) + a + 1];
  const int nq = qend - r0 > BQ ? 2 : 1;  // query tiles of this block with rows
  const int ns = n_sel[(size_t)h * Cq + a];
  const int32_t* sl = sel + ((size_t)h * Cq + a) * Ck;
  const int32_t* koff = k_off + (size_t)h * (Ck + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // routed clusters of this query cluster: bit set, ranges, total keys
  for (int i = threadIdx.x; i < (Ck + 31) / 32; i += blockDim.x) bits[i] = 0;
  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, kProducers);
    for (int i = 0; i < kKSlots; ++i) {
      tc::mbar_init(k_full + i, 1);   // one arrival carrying the stage's byte count
      tc::mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < kVSlots; ++i) {
      tc::mbar_init(v_full + i, 1);
      tc::mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(s_full + i, 1);
      tc::mbar_init(p_full + i, 128);
      tc::mbar_init(o_done + i, 1);
    }
    tc::mbar_init(done, 1);
    for (int i = 0; i < kBSlots; ++i) {
      tc::mbar_init(b_full + i, 1);
      tc::mbar_init(b_empty + i, 4 * nq);
    }
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  __syncthreads();
  long long lex_part = 0;
  const int32_t* pof = poff + (size_t)h * (Ck + 1);
  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const int c = sl[i];
    atomicOr(&bits[c >> 5], 1u << (c & 31));
    const int len = koff[c + 1] - koff[c];
    lex_part += (len + 7) & ~7;  // padded stream length
    if (i < kMaxRanges) { rng_start[i] = pof[c]; rng_cum[i + 1] = (len + 7) & ~7; rng_len[i] = len; }
  }
  for (int o = 16; o > 0; o >>= 1) lex_part += __shfl_xor_sync(0xffffffffu, lex_part, o);
  __shared__ long long lex_w[kThreads / 32];
  if (lane == 0) lex_w[warp] = lex_part;
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  long long lex = 0;
  for (int i = 0; i < kThreads / 32; ++i) lex += lex_w[i];
  // prefix of the staged range lengths (warp 1; read only by the producers,
  // which meet warp 1 at named barrier 2 before using it)
  const int nr = min(ns, kMaxRanges);
  if (warp == 1) {
    int carry = 0;
    for (int i0 = 0; i0 < nr; i0 += 32) {
      const int i = i0 + lane;
      int v = i < nr ? rng_cum[i + 1] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      if (i < nr) rng_cum[i + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) rng_cum[0] = 0;
  }
  const uint32_t tmem = *tmem_slot;
  const int n_ex = (int)((lex + BN - 1) / BN);
  const int n_cp = Ckpad / BN;
  const int ntile = n_ex + n_cp;
  // ring-stage sequence: an exact tile uses one stage, a compensation tile two
  auto ustart = [&](int j) { return j <= n_ex ? j : n_ex + 2 * (j - n_ex); };
  auto nparts = [&](int j) { return j < n_ex ? 1 : 2; };

  // Register split between the warpgroups: the MMA / producer warpgroup
  // gives registers back, the two softmax warpgroups take them (one S row of
  // 128 values stays in registers).  4 warps x 32 x kRegsLow + 8 warps x 32 x
  // kRegsHigh must not exceed the block's registers at launch (384 threads
  // x the compiled count, checked on the host before the first launch).
  if (warp < 4) tc::setmaxnreg_dec<kRegsLow>();
  else tc::setmaxnreg_inc<kRegsHigh>();

  if (warp == 0) {
    // ------------------------------------------------------------------ MMA
    // The whole warp runs the issue loop, so the loop control and the
    // descriptor arithmetic are warp-uniform; one elected lane issues each
    // tcgen05.mma and commit.  Every wait is made warp-uniform.
    const bool leader = tc::elect_one();
    const uint32_t id_s = tc::idesc_bf16(BQ, BN, false, false);
    const uint32_t id_o = tc::idesc_bf16(BQ, D, false, true);
    // descriptors are built once; a K step only moves the start-address
    // field (address >> 4): +2 per 32 B inside a swizzled row, +1024 per
    // 16 KB region of Q, +16 per 256 B of a K tile, +2*kGroup/16 for V
    const uint64_t qd0 = tc::desc_kmajor(tc::smem_u32(smem + S::q_off), BQ * 128u, 0);
    const uint64_t kd0 = tc::desc_kmajor_g8(tc::smem_u32(smem + S::k_off), kGroup, 0);
    const uint64_t vd0 = tc::desc_mnmajor_g8(tc::smem_u32(smem + S::v_off), kGroup, 0);
    constexpr uint64_t kStageStep = (uint64_t)(S::kKTile >> 4);
    constexpr uint64_t kQStep = (uint64_t)(S::kQTile >> 4);
    bool ok = tc::mbar_wait_warp(q_full, 0, abort_flag, status);
    // S[t] = Q_t K_j^T (all parts of stage j); S[t] was last read as P[t]
    // by P.V_t(j - 1), issued before
    auto issue_s = [&](int t, int j) {
      const int u0 = ustart(j), np = nparts(j);
      const uint32_t scol = tmem + kColS + (uint32_t)(t * 128);
      const uint64_t qd = qd0 + (uint64_t)t * kQStep;
      for (int p = 0; p < np; ++p) {
        const uint64_t kd = kd0 + (uint64_t)((u0 + p) % kKSlots) * kStageStep;
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            tc::mma_ss(scol, qd + (uint64_t)((k >> 2) * 1024 + (k & 3) * 2), kd + (uint64_t)k * 16u, id_s,
                       (p > 0 || k > 0) ? 1u : 0u);
        }
      }
      if (leader) tc::mma_commit(s_full + t);
      __syncwarp();
    };
    auto wait_k = [&](int j) -> bool {
      const int u0 = ustart(j), np = nparts(j);
      for (int p = 0; p < np; ++p)
        if (!tc::mbar_wait_warp(k_full + (u0 + p) % kKSlots, ((u0 + p) / kKSlots) & 1, abort_flag, status))
          return false;
      tc::tc_fence_after();
      return true;
    };
    auto commit_slots = [&](uint64_t* ring, int nslots, int j) {
      if (leader)
        for (int p = 0; p < nparts(j); ++p) tc::mma_commit(ring + (ustart(j) + p) % nslots);
      __syncwarp();
    };
    if (ok && ntile > 0) {
      ok = wait_k(0);
      if (ok) {
        for (int t = 0; t < nq; ++t) issue_s(t, 0);
        commit_slots(k_empty, kKSlots, 0);
      }
    }
    for (int j = 0; ok && j < ntile; ++j) {
      const int u0 = ustart(j), np = nparts(j);
      for (int p = 0; ok && p < np; ++p)
        ok = tc::mbar_wait_warp(v_full + (u0 + p) % kVSlots, ((u0 + p) / kVSlots) & 1, abort_flag, status);
      for (int t = 0; ok && t < nq; ++t) {
        // O[t] += P[t] V_j once the softmax of tile t has written P[t]
        if (!tc::mbar_wait_warp(p_full + t, j & 1, abort_flag, status)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t pcol = tmem + kColS + (uint32_t)(t * 128);
        const uint32_t ocol = tmem + kColO + (uint32_t)(t * D);
        for (int p = 0; p < np; ++p) {
          const uint64_t vd = vd0 + (uint64_t)((u0 + p) % kVSlots) * kStageStep;
          if (leader) {
#pragma unroll
            for (int k = 0; k < BN / 16; ++k)
              tc::mma_ts(ocol, pcol + (uint32_t)k * 8u, vd + (uint64_t)k * (2u * kGroup >> 4), id_o,
                         (j > 0 || p > 0 || k > 0) ? 1u : 0u);
          }
        }
        if (leader) tc::mma_commit(o_done + t);
        __syncwarp();
        if (t == nq - 1) commit_slots(v_empty, kVSlots, j);
        // then S of the next stage for the same tile
        if (j + 1 < ntile) {
          if (t == 0 && !wait_k(j + 1)) { ok = false; break; }
          issue_s(t, j + 1);
          if (t == nq - 1) commit_slots(k_empty, kKSlots, j + 1);
        }
      }
    }
    if (leader) tc::mma_commit(done);
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ producers
    const int pt = threadIdx.x - 32;
    {
      const bf16* Qh = Qp + (size_t)h * Nq * D;
      const uint32_t qa = tc::smem_u32(smem + S::q_off);
      // both query tiles (rows past the cluster's end are zero)
      for (int e = pt; e < 2 * BQ * CPR; e += kProducers) {
        const int r = e / CPR, c = e % CPR, row = r0 + r;
        const bool valid = row < qend;
        tc::cp_async16(qa + (uint32_t)(r / BQ) * (uint32_t)S::kQTile + tc::sw128_offset(r % BQ, c, BQ),
                       Qh + (size_t)(valid ? row : 0) * D + c * 8, valid ? 16u : 0u);
      }
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
      tc::mbar_arrive(q_full);
    }
    asm volatile("bar.sync 2, 96;" ::: "memory");  // range prefix ready
    // Pieces of the padded routed stream in [pos0, pos0 + BN): one lane per
    // staged range from the first one that ends after pos0 (a routed range
    // holds at least 8 padded rows, so the window meets at most 16 of them).
    // A piece that would leave the stage tile or the packed rows gets zero
    // groups (status word) and is neither copied nor unmasked.  Returns the
    // piece count; tail = rows of the window the stream covers.
    auto make_pieces = [&](int pos0, int4* pcs, int& tail, uint32_t& bytes) -> int {
      const int end = pos0 + BN;
      int npc = 0;
      if (ns <= kMaxRanges) {
        int ri = ns;
        for (int base = 0; base < ns; base += 32) {
          const int i = base + lane;
          const unsigned m = __ballot_sync(0xffffffffu, i < ns && rng_cum[i + 1] > pos0);
          if (m) { ri = base + __ffs(m) - 1; break; }
        }
        const int ci = ri + lane;
        int lo = 0, hi = 0, cs = 0;
        if (ci < ns) {
          cs = rng_cum[ci];
          lo = max(cs, pos0);
          hi = min(rng_cum[ci + 1], end);
        }
        const bool has = hi > lo;
        const unsigned hm = __ballot_sync(0xffffffffu, has);
        int z = 0;
        if (has) {
          const int off = lo - cs;
          int4 pc = make_int4((lo - pos0) >> 3, rng_start[ci] + off, (hi - lo) >> 3,
                              max(0, min(rng_len[ci] - off, hi - lo)));
          const bool good = pc.x >= 0 && pc.z > 0 && pc.x + pc.z <= BN / 8 && pc.y >= 0 &&
                            (size_t)pc.y + (size_t)pc.z * 8 <= npad;
          if (!good) { set_status(status, ST_BOUNDS); pc.z = 0; pc.w = 0; }
          z = pc.z;
          pcs[__popc(hm & ((1u << lane) - 1u))] = pc;
        }
        npc = __popc(hm);
        tail = __reduce_max_sync(0xffffffffu, has ? hi - pos0 : 0);
        // the window must be covered up to the stream end (status word if not)
        if (lane == 0 && (long long)tail < min((long long)BN, lex - pos0)) set_status(status, ST_BOUNDS);
        bytes = (uint32_t)__reduce_add_sync(0xffffffffu, z) * kGroup;
      } else {
        // more routed clusters than staged ranges: walk the selection list
        int t = 0, nb = 0;
        if (lane == 0) {
          int cum = 0, pos = pos0;
          for (int ri = 0; pos < end && ri < ns && npc < kMaxPieces; ++ri) {
            const int c = sl[ri];
            const int pst = pof[c], len = koff[c + 1] - koff[c], plen = (len + 7) & ~7;
            if (cum + plen <= pos) { cum += plen; continue; }
            const int off = pos - cum, take = min(plen - off, end - pos);
            int4 pc = make_int4((pos - pos0) >> 3, pst + off, take >> 3, max(0, min(len - off, take)));
            const bool good = pc.x >= 0 && pc.z > 0 && pc.x + pc.z <= BN / 8 && pc.y >= 0 &&
                              (size_t)pc.y + (size_t)pc.z * 8 <= npad;
            if (!good) { set_status(status, ST_BOUNDS); pc.z = 0; pc.w = 0; }
            nb += pc.z;
            pcs[npc++] = pc;
            pos += take;
            cum += plen;
          }
          t = pos - pos0;
        }
        // the window must be covered up to the stream end (status word if not)
        if (lane == 0 && (long long)t < min((long long)BN, lex - pos0)) set_status(status, ST_BOUNDS);
        npc = __shfl_sync(0xffffffffu, npc, 0);
        tail = __shfl_sync(0xffffffffu, t, 0);
        bytes = (uint32_t)__shfl_sync(0xffffffffu, nb, 0) * kGroup;
      }
      __syncwarp();
      return npc;
    };
    // warp 1 produces the even stages, warp 2 the odd ones (warp 3 only helps
    // with the query tile): keys once the K slot is free, the stage's bias
    // once its bias slot is, then values once the V slot is.  Each warp always
    // fills the same K and V slot and its own two bias slots, and it waits on
    // a slot only for the stage it filled there last, so no wait on a ring
    // barrier can run a phase ahead.
    if (warp == 1 || warp == 2) {
      const int pw = warp - 1;
      int4* pcs = pieces + pw * kMaxPieces;  // this warp's piece list
      const uint8_t* Kh = kpk + (size_t)h * npad * D * 2;
      const uint8_t* Vh = vpk + (size_t)h * npad * D * 2;
      const float* LC = lc2 + (size_t)h * Ckpad;
      const size_t cbase = (size_t)h * Ckpad * D * 2;
      const int nstage = ustart(ntile);  // total ring stages of the stream
      const unsigned rot = n_ex > 0 ? (blockIdx.x * 2654435761u + h * 40503u) % (unsigned)n_ex : 0u;
      for (int u = pw; u < nstage; u += 2) {
        const int sk = u % kKSlots, st = u % kVSlots;
        const bool exact = u < n_ex;
        int j = exact ? u : n_ex + (u - n_ex) / 2;
        const int p = exact ? 0 : (u - n_ex) & 1;
        // blocks start their walk over the routed keys at different tiles (the
        // softmax does not depend on the order), so that the blocks of a head
        // do not all read the same popular clusters at the same time
        if (exact) j = (int)(((unsigned)j + rot) % (unsigned)n_ex);
        uint8_t* ktile = smem + S::k_off + sk * S::kKTile;
        uint8_t* vtile = smem + S::v_off + st * S::kKTile;
        int npc = 0, tail = BN;
        uint32_t bytes = 0;
        // ---- keys
        if (!tc::mbar_wait_warp(k_empty + sk, ((u / kKSlots) & 1) ^ 1, abort_flag, status)) break;
        if (exact) {
          npc = make_pieces(j * BN, pcs, tail, bytes);
          // zero the rows past the stream end so the MMAs see finite values
          if (tail < BN) {
            uint4* zr = reinterpret_cast<uint4*>(ktile) + (tail >> 3) * (kGroup / 16);
            const int nz = ((BN - tail) >> 3) * (int)(kGroup / 16);
            for (int i = lane; i < nz; i += 32) zr[i] = make_uint4(0, 0, 0, 0);
            tc::fence_proxy_async();
          }
          __syncwarp();
          if (lane == 0) {
            tc::mbar_arrive_expect_tx(k_full + sk, bytes);
            for (int q = 0; q < npc; ++q) {
              const int4 pc = pcs[q];
              if (pc.z > 0)
                tc::bulk_g2s(tc::smem_u32(ktile) + (uint32_t)pc.x * kGroup, Kh + (size_t)(pc.y >> 3) * kGroup,
                             (uint32_t)pc.z * kGroup, k_full + sk);
            }
          }
        } else if (lane == 0) {
          const uint32_t n = (uint32_t)(BN / 8) * kGroup;
          const size_t go = cbase + (size_t)(((j - n_ex) * BN) >> 3) * kGroup;
          tc::mbar_arrive_expect_tx(k_full + sk, n);
          tc::bulk_g2s(tc::smem_u32(ktile), (p == 0 ? kb_hi : kb_lo) + go, n, k_full + sk);
        }
        __syncwarp();
        // ---- bias and mask (every ring stage passes through the bias ring;
        // a compensation tile's bias rides with its first, hi, part)
        const int sb = u % kBSlots;
        if (!tc::mbar_wait_warp(b_empty + sb, ((u / kBSlots) & 1) ^ 1, abort_flag, status)) break;
        float* bias = bias_s + sb * BN;
        if (exact) {
          // valid keys 0, padding and the stream tail -inf
          for (int i = lane; i < BN; i += 32) bias[i] = -INFINITY;
          __syncwarp();
          int nvalid = 0;
          for (int q = 0; q < npc; ++q) {
            const int4 pc = pcs[q];
            for (int i = lane; i < pc.w; i += 32) bias[pc.x * 8 + i] = 0.f;
            nvalid += pc.w;
          }
          if (lane == 0) nv_s[sb] = nvalid;
        } else if (p == 0) {
          const int c0 = (j - n_ex) * BN;
          for (int i = lane; i < BN; i += 32) {
            const int c = c0 + i;
            const bool routed = c < Ck && ((bits[c >> 5] >> (c & 31)) & 1u);
            bias[i] = routed ? -INFINITY : LC[c];
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(b_full + sb);
        // ---- values
        if (!tc::mbar_wait_warp(v_empty + st, ((u / kVSlots) & 1) ^ 1, abort_flag, status)) break;
        if (exact) {
          if (tail < BN) {
            uint4* zr = reinterpret_cast<uint4*>(vtile) + (tail >> 3) * (kGroup / 16);
            const int nz = ((BN - tail) >> 3) * (int)(kGroup / 16);
            for (int i = lane; i < nz; i += 32) zr[i] = make_uint4(0, 0, 0, 0);
            tc::fence_proxy_async();
          }
          __syncwarp();
          if (lane == 0) {
            tc::mbar_arrive_expect_tx(v_full + st, bytes);
            for (int q = 0; q < npc; ++q) {
              const int4 pc = pcs[q];
              if (pc.z > 0)
                tc::bulk_g2s(tc::smem_u32(vtile) + (uint32_t)pc.x * kGroup, Vh + (size_t)(pc.y >> 3) * kGroup,
                             (uint32_t)pc.z * kGroup, v_full + st);
            }
          }
        } else if (lane == 0) {
          const uint32_t n = (uint32_t)(BN / 8) * kGroup;
          const size_t go = cbase + (size_t)(((j - n_ex) * BN) >> 3) * kGroup;
          tc::mbar_arrive_expect_tx(v_full + st, n);
          tc::bulk_g2s(tc::smem_u32(vtile), (p == 0 ? vb_hi : vb_lo) + go, n, v_full + st);
        }
        __syncwarp();
      }
    }
  } else if (warp < 8 || nq == 2) {
    // -------------------------------------------------------------- softmax
    // group t (warps 4-7: t = 0, warps 8-11: t = 1) owns query tile t: S[t],
    // its running maximum m, row sum l and accumulator O[t], over every stage.
    const int t = (warp - 4) >> 2;
    const int r = ((warp & 3) << 5) + lane;   // tile row == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;
    const uint32_t scol = kColS + (uint32_t)(t * 128);
    const uint32_t ocol = kColO + (uint32_t)(t * D);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < ntile; ++j) {
      const int u0 = ustart(j), sb = u0 % kBSlots;
      if (!tc::mbar_wait_warp(s_full + t, j & 1, abort_flag, status)) { ok = false; break; }
      // bias / mask of this stage (its next phase needs this warp's arrival
      // on the slot's empty barrier, so the parity cannot run ahead)
      if (!tc::mbar_wait_warp(b_full + sb, (u0 / kBSlots) & 1, abort_flag, status)) { ok = false; break; }
      tc::tc_fence_after();
      const float* bias = bias_s + sb * BN;
      // the stage's 128 logits of this row, read once: x = s*log2e * S + bias
      uint32_t v[128];
      tc::tmem_ld32(tmem + lane_base + scol, *reinterpret_cast<uint32_t(*)[32]>(v));
      tc::tmem_ld32(tmem + lane_base + scol + 32u, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tc::tmem_ld32(tmem + lane_base + scol + 64u, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
      tc::tmem_ld32(tmem + lane_base + scol + 96u, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
      tc::tmem_ld_wait();
      // Routed stage of rows whose running maximum is already a non-negative
      // real logit: the exponentials are taken against it straight away (the
      // padding keys' share 2^(0 - m) <= 1 comes off the row sum, as on the
      // fast path below), without a maximum pass.  The stage is accepted when
      // every row's sum of the 128 terms is at most 2^16: then no term exceeds
      // 2^16, which bf16 P and the float32 accumulators carry without loss
      // (the reference maximum only has to keep the terms finite; the result
      // does not depend on it).  P stays in registers until then, so S[t] is
      // still intact when a row's sum is larger (its maximum grew by more than
      // 2^9 at least, rare once a row has seen a few stages): S is reloaded and
      // the stage takes the path below, which finds the maximum and rescales,
      // on the raw formula (every reference maximum is >= 0) and without
      // touching the released bias slot again.
      bool spec_failed = false;
      int npad_spec = 0;
      if (j < n_ex && __all_sync(0xffffffffu, m_used >= 0.f)) {
        npad_spec = BN - nv_s[sb];
        const uint64_t negm = f2(-m_used, -m_used);
        const uint64_t sc2 = f2(scale2, scale2);
        uint32_t pk[64];
        uint64_t r2[2] = {0ull, 0ull};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const uint64_t x = f2_fma(f2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), sc2, negm);
          const float p0 = ex2(f2_lo(x)), p1 = ex2(f2_hi(x));
          r2[i & 1] = f2_add(r2[i & 1], f2(p0, p1));
          pk[i] = pack_bf16(p0, p1);
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(b_empty + sb);
        const uint64_t rs = f2_add(r2[0], r2[1]);
        const float tot = f2_lo(rs) + f2_hi(rs);
        if (__all_sync(0xffffffffu, tot <= 65536.f)) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tc::tmem_st16(tmem + lane_base + scol + (uint32_t)(q * 16),
                          *reinterpret_cast<const uint32_t(*)[16]>(pk + 16 * q));
          tc::tmem_st_wait();
          l += tot - (float)npad_spec * ex2(-m_used);
          tc::tc_fence_before();
          tc::mbar_arrive(p_full + t);
          continue;
        }
        spec_failed = true;
        tc::tmem_ld32(tmem + lane_base + scol, *reinterpret_cast<uint32_t(*)[32]>(v));
        tc::tmem_ld32(tmem + lane_base + scol + 32u, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tc::tmem_ld32(tmem + lane_base + scol + 64u, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
        tc::tmem_ld32(tmem + lane_base + scol + 96u, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
        tc::tmem_ld_wait();
      }
      // Routed stage, fast path: padding and tail keys have zero key rows, so
      // their logits are exactly 0 and their value rows are 0.  When the raw
      // maximum of the stage is positive it is a real key's, the scale and
      // the row maximum are applied in one FMA in the exponential pass, and
      // the padding's known share is taken off the row sum.  Otherwise (and
      // for compensation stages) x = s * scale2 + bias with the stage's bias.
      const uint64_t sc2 = f2(scale2, scale2);
      float mx;
      bool raw = false;
      {
        float m8[8];
        if (j < n_ex) {
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
#pragma unroll
          for (int i = 0; i < 128; i += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              m8[k] = tc::fmax3(m8[k], __uint_as_float(v[i + 2 * k]), __uint_as_float(v[i + 2 * k + 1]));
          const float mr = fmaxf(tc::fmax3(m8[0], m8[1], m8[2]), tc::fmax3(tc::fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
          raw = spec_failed || __all_sync(0xffffffffu, mr > 0.f);
          mx = mr * scale2;
        }
        if (!raw) {
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
#pragma unroll
          for (int i = 0; i < 128; i += 16) {
            const float4 b0 = *reinterpret_cast<const float4*>(bias + i);
            const float4 b1 = *reinterpret_cast<const float4*>(bias + i + 4);
            const float4 b2 = *reinterpret_cast<const float4*>(bias + i + 8);
            const float4 b3 = *reinterpret_cast<const float4*>(bias + i + 12);
            const float bb[16] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w,
                                  b2.x, b2.y, b2.z, b2.w, b3.x, b3.y, b3.z, b3.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              // x = s * scale2 + bias for two keys per instruction
              const uint64_t x = f2_fma(f2(__uint_as_float(v[i + 2 * k]), __uint_as_float(v[i + 2 * k + 1])), sc2,
                                        f2(bb[2 * k], bb[2 * k + 1]));
              v[i + 2 * k] = __float_as_uint(f2_lo(x));
              v[i + 2 * k + 1] = __float_as_uint(f2_hi(x));
              m8[k] = tc::fmax3(m8[k], f2_lo(x), f2_hi(x));
            }
          }
          mx = fmaxf(tc::fmax3(m8[0], m8[1], m8[2]), tc::fmax3(tc::fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
        }
      }
      const int npad = spec_failed ? npad_spec : raw ? BN - nv_s[sb] : 0;
      // the bias is read: release the stage's bias slot(s) on this warp's
      // behalf (a failed speculative stage released its slot already)
      __syncwarp();
      if (lane == 0 && !spec_failed)
        for (int q = 0; q < nparts(j); ++q) tc::mbar_arrive(b_empty + (u0 + q) % kBSlots);
      // lazy rescale: a row whose maximum grew by more than 2^8 rescales O[t]
      // and l.  The tensor-memory accesses are warp-collective, so the warp
      // rescales together (factor 1 for rows that do not need it).  O[t] is
      // complete up to P.V_t(j - 1): S[t] of this stage was issued after it.
      const bool grow = mx > m_used + 8.f;
      const bool has_o = j >= 1 && m_used > -INFINITY;
      if (__any_sync(0xffffffffu, grow && has_o)) {
        if (!tc::mbar_wait_warp(o_done + t, (j - 1) & 1, abort_flag, status)) { ok = false; break; }
        tc::tc_fence_after();
        const float f = (grow && has_o) ? ex2(m_used - mx) : 1.f;
#pragma unroll
        for (int q = 0; q < D / 16; ++q) {
          uint32_t ov[16];
          tc::tmem_ld16(tmem + lane_base + ocol + (uint32_t)q * 16u, ov);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
          tc::tmem_st16(tmem + lane_base + ocol + (uint32_t)q * 16u, ov);
        }
        tc::tmem_st_wait();
        l *= f;
      }
      if (grow) m_used = mx;
      const float mref = m_used == -INFINITY ? 0.f : m_used;
      // P = 2^(x - m) in bf16 over the first 64 columns of S[t] (keys 2c and
      // 2c + 1 in column c; every S value of the row is already in registers);
      // x - m (fast path: s * scale2 - m) for two keys per instruction, row
      // sums in four packed pairs
      // (fallback: the stored x times 1 minus m, which is x - m exactly)
      const uint64_t negm = f2(-mref, -mref);
      const uint64_t mul2 = raw ? sc2 : f2(1.f, 1.f);
      uint64_t r4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = q * 32 + 2 * i;
          const uint64_t x = f2_fma(f2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), mul2, negm);
          const float p0 = ex2(f2_lo(x)), p1 = ex2(f2_hi(x));
          r4[i & 3] = f2_add(r4[i & 3], f2(p0, p1));
          pk[i] = pack_bf16(p0, p1);
        }
        tc::tmem_st16(tmem + lane_base + scol + (uint32_t)(q * 16), pk);
      }
      tc::tmem_st_wait();
      {
        const uint64_t r2 = f2_add(f2_add(r4[0], r4[1]), f2_add(r4[2], r4[3]));
        // the padding keys (fast path) each added 2^(0 - m)
        l += (f2_lo(r2) + f2_hi(r2)) - (float)npad * ex2(-mref);
      }
      tc::tc_fence_before();
      tc::mbar_arrive(p_full + t);
    }
    // epilogue: the last P.V into O[t], then O / l stored via perm_q
    if (ok && ntile > 0) ok = tc::mbar_wait_warp(o_done + t, (ntile - 1) & 1, abort_flag, status);
    if (ok) {
      tc::tc_fence_after();
      // a row that saw no key (every logit masked) stores zeros
      const bool have = m_used > -INFINITY && l > 0.f;
      const float inv = have ? 1.f / l : 0.f;
      const int row = r0 + t * BQ + r;
      const bool valid = row < qend;
      bf16* orow = O + ((size_t)h * Nq + (valid ? perm_q[(size_t)h * Nq + row] : 0)) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tc::tmem_ld32(tmem + lane_base + ocol + (uint32_t)(q * 32), o);
        tc::tmem_ld_wait();
        uint4 w4[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w4);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wp[i] = have ? pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv) : 0u;
        if (valid) {
#pragma unroll
          for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(orow + q * 32)[i] = w4[i];
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

int round_stage(int x) { return (x + BN - 1) / BN * BN; }

// Events the next launch records around the attention kernel alone (set by
// the forward when the caller asked for stage timings; per host thread).
thread_local cudaEvent_t t_kernel_ev[2] = {nullptr, nullptr};
thread_local bool t_kernel_ev_used = false;

struct AttnWs {
  uint8_t *kh, *kl, *vh, *vl, *kpk, *vpk;
  int32_t* poff;
  float* lc2;
  int2* tiles;
  int32_t* ntiles;
  size_t npad;
};

size_t attn_layout(int H, int Nq, int Nk, int d, int Cq, int Ck, AttnWs* out, void* ws) {
  Carve cv(ws);
  const int Ckpad = round_stage(Ck);
  const int tmax = (Nq + kUnitRows - 1) / kUnitRows + Cq;
  AttnWs w;
  w.npad = (size_t)Nk + 8 * (size_t)Ck;  // rows after padding every cluster to 8
  w.kh = cv.take<uint8_t>((size_t)H * Ckpad * d * 2);
  w.kl = cv.take<uint8_t>((size_t)H * Ckpad * d * 2);
  w.vh = cv.take<uint8_t>((size_t)H * Ckpad * d * 2);
  w.vl = cv.take<uint8_t>((size_t)H * Ckpad * d * 2);
  w.kpk = cv.take<uint8_t>((size_t)H * w.npad * d * 2);
  w.vpk = cv.take<uint8_t>((size_t)H * w.npad * d * 2);
  w.poff = cv.take<int32_t>((size_t)H * (Ck + 1));
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
  attn_layout(H, Nq, Nk, D, Cq, Ck, &w, ws);
  const int Ckpad = round_stage(Ck);
  const int tmax = (Nq + kUnitRows - 1) / kUnitRows + Cq;
  k_prep_comp<D><<<dim3(Ckpad, H), 64, 0, st>>>(Kbar, Vbar, k_off, Ck, Ckpad, w.kh, w.kl, w.vh, w.vl, w.lc2);
  note_launch();
  k_pad_offsets<<<H, 1024, 0, st>>>(k_off, Ck, w.poff); note_launch();
  k_pack<D><<<dim3(Ck, H), 256, 0, st>>>(static_cast<const bf16*>(Kp), static_cast<const bf16*>(Vp), k_off, w.poff,
                                         Nk, Ck, w.npad, w.kpk, w.vpk);
  note_launch();
  k_tile_table_tc<<<H, 1024, 0, st>>>(q_off, Cq, tmax, w.tiles, w.ntiles); note_launch();
  const int smem = AttnSmem<D>::total;
  cudaError_t e = cudaFuncSetAttribute(k_attn_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // the softmax warpgroups' register increase waits for the pool the block
  // was launched with: refuse a build whose launch count cannot cover it
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, k_attn_tc<D>);
  if (e != cudaSuccess) return e;
  if ((long long)fa.numRegs * kThreads < 4LL * 32 * kRegsLow + 8LL * 32 * kRegsHigh) return cudaErrorInvalidValue;
  const bool timed = t_kernel_ev[0] != nullptr;
  if (timed) cudaEventRecord(t_kernel_ev[0], st);
  k_attn_tc<D><<<dim3(tmax, H), kThreads, smem, st>>>(
      static_cast<const bf16*>(Qp), w.kpk, w.vpk, w.npad, q_off, k_off, w.poff, perm_q, w.kh, w.kl, w.vh, w.vl,
      w.lc2, sel, n_sel, w.tiles, w.ntiles, tmax, Nq, Nk, Cq, Ck, Ckpad, scale * kLog2e,
      static_cast<bf16*>(O), status_word());
  note_launch();
  if (timed) {
    cudaEventRecord(t_kernel_ev[1], st);
    t_kernel_ev[0] = t_kernel_ev[1] = nullptr;
    t_kernel_ev_used = true;
  }
  return cudaGetLastError();
}

}  // namespace

void attn_tc_time_next_kernel(cudaEvent_t begin, cudaEvent_t end) {
  t_kernel_ev[0] = begin;
  t_kernel_ev[1] = end;
  t_kernel_ev_used = false;
}

bool attn_tc_kernel_was_timed() { return t_kernel_ev_used; }

bool attn_tc_supported(int d, int Ck) { return (d == 64 || d == 128) && Ck <= kMaxCkBits; }

size_t attn_tc_ws_bytes(int H, int Nq, int Nk, int d, int Cq, int Ck) {
  if (!attn_tc_supported(d, Ck)) return 0;
  return attn_layout(H, Nq, Nk, d, Cq, Ck, nullptr, nullptr);
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
