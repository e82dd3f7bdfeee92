// Value-aware block error on the tensor cores (SVG-EAR review, step (2);
// gist.science summary 2.B, "lightweight probe", O(C_q N_k d)).
//
// With w = -expm1(u), u = s qbar_a.k_j - L[a][c] (L = s qbar_a.kbar_c) and
// A = e^{L[a][c] - M_a}, the block error of the review's step (2) is
//   E[a][c] = A^2 / |k_c| * sum_{j in c} (s1_j + 2 w s2_j + w^2 s3_j)
// (the same algebra as the CUDA-core kernel in block_error.cu).  The dot
// products s qbar_a.k_j come from tcgen05 MMAs: A operand = s*qbar split into
// bf16 hi + lo (query clusters on the 128 TMEM lanes; the residual of the
// split is below 2^-18 |s qbar| per component), B operand = 256 permuted keys
// (exact in bf16), fp32 accumulators in tensor memory.
//
// A block owns whole key clusters (the clusters whose first key falls in its
// share of the head's keys), so every E[a][c] is one thread's sum in a fixed
// order.  Warp 0 allocates tensor memory and issues MMAs, warp 1 issues the
// TMA copies of the key tiles and stages the per-key scalars, and the
// remaining warps are kBeGroups epilogue warpgroups (one TMEM lane = one query
// cluster): group g owns the key clusters c with c % kBeGroups == g and reads
// only the 32-key chunks of each tile that hold its clusters' keys, so a
// cluster is still summed by one thread in key order.
// For the value-agnostic ablation the staged scalars are (0, 0, 1), so each
// key adds w^2 = (A - B_j)^2 / A^2.
#include <cuda.h>

#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace svg {

namespace {

constexpr int kBeGroups = 3;                    // epilogue warpgroups (clusters round-robin)
constexpr int kBeThreads = 64 + 128 * kBeGroups;
constexpr int kBeKeys = 256;    // keys per tile (MMA N)
constexpr int kBeStages = 2;
constexpr int kBeRows = 128;    // query-cluster rows of the A operand (MMA M)
constexpr int kBeSmemLimit = 232448;

// s*qbar split into bf16 hi and lo parts, rows padded to 128 with zeros:
// out [H][2][128][D] (part 0 = hi, part 1 = lo).
template <int D>
__global__ void __launch_bounds__(256) k_prep_qhl(const float* __restrict__ Qbar, int Cq, float scale,
                                                  bf16* __restrict__ out) {
  const int h = blockIdx.x;
  for (int e = threadIdx.x; e < kBeRows * D; e += blockDim.x) {
    const int r = e / D, t = e % D;
    const float q = r < Cq ? Qbar[((size_t)h * Cq + r) * D + t] * scale : 0.f;
    const bf16 hi = __float2bfloat16_rn(q);
    const bf16 lo = __float2bfloat16_rn(q - __bfloat162float(hi));
    out[(((size_t)h * 2 + 0) * kBeRows + r) * D + t] = hi;
    out[(((size_t)h * 2 + 1) * kBeRows + r) * D + t] = lo;
  }
}

// -expm1(u): for |u| < 1/4 the Taylor series of e^u - 1 to the u^7 term
// (the first omitted term is u^8/8!, a relative 2e-9 of e^u - 1); otherwise
// 1 - e^u through the fast exponential, whose relative error is a few 1e-7
// of e^u while |e^u - 1| >= 0.22 there.
__device__ __forceinline__ float neg_expm1(float u) {
  float p = 1.f / 5040.f;
  p = fmaf(p, u, 1.f / 720.f);
  p = fmaf(p, u, 1.f / 120.f);
  p = fmaf(p, u, 1.f / 24.f);
  p = fmaf(p, u, 1.f / 6.f);
  p = fmaf(p, u, 0.5f);
  p = fmaf(p, u, 1.f);
  const float small = -(p * u);
  const float large = 1.f - __expf(u);
  return fabsf(u) < 0.25f ? small : large;
}

struct BeLay {
  int q, k, sc, bars, total;
};
__host__ __device__ inline BeLay be_layout(int D) {
  BeLay l;
  l.q = 0;                                        // hi then lo: 2 x 128 rows x D bf16
  l.k = l.q + 2 * kBeRows * D * 2;                // stages of 256 keys x D bf16
  l.sc = l.k + kBeStages * kBeKeys * D * 2;       // stages of 256 x {s1, s2, s3, 0}
  l.bars = l.sc + kBeStages * kBeKeys * 16;
  l.total = l.bars + 16 * 8 + 1024;
  return l;
}

// First cluster c in [0, Ck] whose first key index off[c] satisfies
// off[c] * G >= g * Nk (clusters are assigned to blocks by their first key).
__device__ __forceinline__ int first_cluster(const int32_t* off, int Ck, long long g, long long G, long long Nk) {
  int lo = 0, hi = Ck;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((long long)off[mid] * G >= g * Nk) hi = mid; else lo = mid + 1;
  }
  return lo;
}

template <int D>
__global__ void __launch_bounds__(kBeThreads, 1)
    k_block_error_tc(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const int32_t* __restrict__ k_off, const float* __restrict__ ks,
                     const float* __restrict__ L, const float* __restrict__ M, int H, int Nk, int Cq, int Ck,
                     int value_agnostic, float* __restrict__ E, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const BeLay Ly = be_layout(D);
  uint8_t* q_s = smem + Ly.q;
  uint8_t* k_s = smem + Ly.k;
  float4* sc_s = reinterpret_cast<float4*>(smem + Ly.sc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* q_full = bars;
  uint64_t* full = bars + 1;                 // [kBeStages]
  uint64_t* empty = bars + 1 + kBeStages;    // [kBeStages]
  uint64_t* acc_full = bars + 5;             // [2]
  uint64_t* acc_empty = bars + 7;            // [2]
  uint64_t* done = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 11);
  constexpr int kQPart = kBeRows * D * 2;    // bytes of hi (or lo)
  constexpr int kKStage = kBeKeys * D * 2;

  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* off = k_off + (size_t)h * (Ck + 1);
  const int c_lo = first_cluster(off, Ck, blockIdx.x, gridDim.x, Nk);
  // the last block also takes the empty clusters that start at Nk
  const int c_hi = blockIdx.x + 1 == gridDim.x ? Ck : first_cluster(off, Ck, (long long)blockIdx.x + 1, gridDim.x, Nk);
  const int kb = off[c_lo], ke = off[c_hi];
  const int ntiles = (ke - kb + kBeKeys - 1) / kBeKeys;

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int i = 0; i < kBeStages; ++i) {
      tc::mbar_init(full + i, 2);    // TMA arrival with bytes + the scalars' arrival
      tc::mbar_init(empty + i, 1 + 4 * kBeGroups);   // MMA commit + every epilogue warp
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(acc_full + i, 1);
      tc::mbar_init(acc_empty + i, 4 * kBeGroups);
    }
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
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
    if (ntiles > 0) {
      bool ok = tc::mbar_wait_warp(q_full, 0, abort_flag, status);
      const uint32_t qa = tc::smem_u32(q_s);
      const uint32_t id = tc::idesc_bf16(kBeRows, kBeKeys, false, false);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int s = t % kBeStages, buf = t & 1;
        ok = tc::mbar_wait_warp(full + s, (t / kBeStages) & 1, abort_flag, status);
        if (ok) ok = tc::mbar_wait_warp(acc_empty + buf, ((t >> 1) & 1) ^ 1, abort_flag, status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t ka = tc::smem_u32(k_s + s * kKStage);
        const uint32_t d_t = tmem + (uint32_t)(buf * kBeKeys);
        if (leader) {
#pragma unroll
          for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int k16 = 0; k16 < D / 16; ++k16) {
              const uint64_t a = tc::desc_kmajor(qa + (uint32_t)(part * kQPart), kBeRows * 128u, k16);
              const uint64_t b = tc::desc_kmajor(ka, kBeKeys * 128u, k16);
              tc::mma_ss(d_t, a, b, id, (part | k16) ? 1u : 0u);
            }
          tc::mma_commit(acc_full + buf);
          tc::mma_commit(empty + s);
        }
        __syncwarp();
      }
    }
    if (leader) tc::mma_commit(done);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- TMA copies and key scalars
    if (ntiles > 0) {
      if (lane == 0) {
        tc::tma_prefetch_map(&tmq);
        tc::tma_prefetch_map(&tmk);
        const uint32_t qa = tc::smem_u32(q_s);
        tc::mbar_arrive_expect_tx(q_full, (uint32_t)(2 * kQPart));
        for (int part = 0; part < 2; ++part)
          for (int kh = 0; kh < D / 64; ++kh)
            tc::tma_load_3d(qa + (uint32_t)(part * kQPart + kh * kBeRows * 128), &tmq, kh * 64,
                            part * kBeRows, h, q_full);
      }
      const size_t plane = (size_t)H * Nk;
      const float* ks1 = value_agnostic ? nullptr : ks + (size_t)h * Nk;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % kBeStages;
        const int j0 = kb + t * kBeKeys;
        // the tile's per-key scalars go to registers first (all loads in
        // flight together, before the wait for the stage)
        float4 vv[kBeKeys / 32];
#pragma unroll
        for (int u = 0; u < kBeKeys / 32; ++u) {
          const int j = j0 + u * 32 + lane;
          vv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (j < ke)
            vv[u] = ks1 ? make_float4(ks1[j], ks1[plane + j], ks1[2 * plane + j], 0.f) : make_float4(0.f, 0.f, 1.f, 0.f);
        }
        const bool ok = tc::mbar_wait_warp(empty + s, ((t / kBeStages) & 1) ^ 1, abort_flag, status);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t ka = tc::smem_u32(k_s + s * kKStage);
          tc::mbar_arrive_expect_tx(full + s, (uint32_t)kKStage);
          for (int kh = 0; kh < D / 64; ++kh)
            tc::tma_load_3d(ka + (uint32_t)(kh * kBeKeys * 128), &tmk, kh * 64, j0, h, full + s);
        }
        float4* sc = sc_s + s * kBeKeys;
#pragma unroll
        for (int u = 0; u < kBeKeys / 32; ++u) sc[u * 32 + lane] = vv[u];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(full + s);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int grp = (warp - 2) >> 2;     // epilogue group: owns clusters c % kBeGroups == grp
    const int quarter = warp & 3;
    const int a = quarter * 32 + lane;   // query cluster == TMEM lane
    const bool act = a < Cq;
    const float Ma = act ? M[(size_t)h * Cq + a] : 0.f;
    const float* La = L + ((size_t)h * Cq + (act ? a : 0)) * Ck;
    float* Ea = E + ((size_t)h * Cq + (act ? a : 0)) * Ck;
    // the group's first cluster at or after c_lo
    int c = c_lo + ((grp - c_lo % kBeGroups) + kBeGroups) % kBeGroups;
    int cbeg = 0, cend = 0, csize = 1;
    float Lc = 0.f;
    double acc = 0.0;
    // moves c to this group's next non-empty cluster (empty ones get E = 0)
    auto enter = [&]() {
      while (c < c_hi && off[c + 1] == off[c]) {
        if (act) Ea[c] = 0.f;
        c += kBeGroups;
      }
      if (c < c_hi) {
        cbeg = off[c];
        cend = off[c + 1];
        csize = cend - cbeg;
        Lc = La[c];
        acc = 0.0;
      }
    };
    auto flush = [&]() {
      if (act) {
        const float A = expf(Lc - Ma);
        Ea[c] = (float)((double)(A * A) * acc / (double)csize);
      }
      c += kBeGroups;
      enter();
    };
    enter();
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      const int s = t % kBeStages, buf = t & 1;
      // the stage's scalars (full) and the tile's accumulators (acc_full)
      ok = tc::mbar_wait_warp(full + s, (t / kBeStages) & 1, abort_flag, status) &&
           tc::mbar_wait_warp(acc_full + buf, (t >> 1) & 1, abort_flag, status);
      if (!ok) break;
      tc::tc_fence_after();
      const float4* sc = sc_s + s * kBeKeys;
      const int j0 = kb + t * kBeKeys;
      const int nk = min(kBeKeys, ke - j0);
      const uint32_t base = tc::taddr(tmem, (uint32_t)(quarter * 32), (uint32_t)(buf * kBeKeys));
      for (int q0 = 0; q0 < nk; q0 += 32) {
        const int k0 = j0 + q0, k1 = j0 + min(q0 + 32, nk);
        // skip chunks that hold none of this group's keys (block-uniform)
        if (!(c < c_hi && cbeg < k1)) continue;
        uint32_t v[32];
        tc::tmem_ld32(base + (uint32_t)q0, v);
        tc::tmem_ld_wait();
        if (cbeg <= k0 && k0 + 32 <= cend && k1 == k0 + 32) {
          // all 32 keys inside the current cluster (the common case): the
          // terms are independent, with no branch between them
          float t8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float4 e = sc[q0 + i];
            const float w = neg_expm1(__uint_as_float(v[i]) - Lc);
            t8[i & 7] += fmaxf(fmaf(w, fmaf(w, e.z, 2.f * e.y), e.x), 0.f);
          }
          acc += (double)(((t8[0] + t8[1]) + (t8[2] + t8[3])) + ((t8[4] + t8[5]) + (t8[6] + t8[7])));
          if (cend == k1) flush();
          continue;
        }
        // cluster boundaries inside the chunk: one segment of the current
        // cluster at a time (keys of other groups' clusters are passed over;
        // every decision is block-uniform), its keys summed in order by a
        // predicated pass over the chunk, so the flush is emitted once
        int i0 = 0;
        const int iend = k1 - k0;
        while (i0 < iend && c < c_hi) {
          if (k0 + i0 < cbeg) {            // another group's cluster
            i0 = min(cbeg - k0, iend);
            continue;
          }
          const int i1 = min(cend - k0, iend);
          float part = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (i >= i0 && i < i1) {
              const float4 e = sc[q0 + i];
              const float w = neg_expm1(__uint_as_float(v[i]) - Lc);
              part += fmaxf(fmaf(w, fmaf(w, e.z, 2.f * e.y), e.x), 0.f);
            }
          }
          acc += (double)part;
          i0 = i1;
          if (k0 + i1 == cend) flush();    // the cluster ends in this chunk
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(acc_empty + buf);
        tc::mbar_arrive(empty + s);
      }
    }
    // trailing empty clusters of this group (every non-empty one was flushed
    // when its last key was summed)
    if (ok) enter();
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

bool block_error_tc_shape_ok(int dtype, int d, int Cq) {
  return dtype == DT_BF16 && (d == 64 || d == 128) && Cq >= 1 && Cq <= kBeRows &&
         be_layout(d).total <= kBeSmemLimit;
}

bool block_error_tc_supported(int dtype, int d, int Cq, int Nk) {
  return block_error_tc_shape_ok(dtype, d, Cq) && Nk >= kBeKeys && tma_available();
}

size_t block_error_tc_ws_bytes(int H, int d) { return (size_t)H * 2 * kBeRows * d * sizeof(bf16); }

// Blocks per head: the count that minimises (waves of 148 blocks) x (key
// tiles per block + a setup cost of about two tiles).
static int pick_blocks_per_head(int H, int Nk) {
  const int tiles = (Nk + kBeKeys - 1) / kBeKeys;
  int best = 1;
  long long best_cost = -1;
  for (int G = 1; G <= tiles; ++G) {
    const long long waves = ((long long)H * G + 147) / 148;
    const long long cost = waves * ((tiles + G - 1) / G + 2);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = G; }
  }
  return best;
}

template <int D>
static cudaError_t be_launch(const float* Qbar, const bf16* Kp, const int32_t* k_off, const float* ks,
                             const float* L, const float* M, int H, int Nk, int Cq, int Ck, float scale,
                             float* E, bf16* qhl, cudaStream_t st, int vagn) {
  k_prep_qhl<D><<<H, 256, 0, st>>>(Qbar, Cq, scale, qhl);
  note_launch();
  CUtensorMap tmq, tmk;
  if (!tma_map_bf16_3d(&tmq, qhl, D, 2 * kBeRows, H, kBeRows) || !tma_map_bf16_3d(&tmk, Kp, D, Nk, H, kBeKeys))
    return cudaErrorInvalidValue;
  const int smem = be_layout(D).total;
  cudaError_t e = cudaFuncSetAttribute(k_block_error_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int G = pick_blocks_per_head(H, Nk);
  k_block_error_tc<D><<<dim3(G, H), kBeThreads, smem, st>>>(tmq, tmk, k_off, ks, L, M, H, Nk, Cq, Ck, vagn,
                                                             E, status_word());
  note_launch();
  return cudaGetLastError();
}

cudaError_t block_error_tc_run(const float* Qbar, const void* Kp, const int32_t* k_off, const float* ks,
                               const float* L, const float* M, int H, int Nk, int d, int Cq, int Ck,
                               float scale, float* E, void* ws, cudaStream_t st, bool value_agnostic) {
  if ((reinterpret_cast<uintptr_t>(Kp) & 15u) || (reinterpret_cast<uintptr_t>(ws) & 15u))
    return cudaErrorInvalidValue;
  const bf16* kp = static_cast<const bf16*>(Kp);
  bf16* qhl = static_cast<bf16*>(ws);
  if (d == 128) return be_launch<128>(Qbar, kp, k_off, ks, L, M, H, Nk, Cq, Ck, scale, E, qhl, st, value_agnostic ? 1 : 0);
  return be_launch<64>(Qbar, kp, k_off, ks, L, M, H, Nk, Cq, Ck, scale, E, qhl, st, value_agnostic ? 1 : 0);
}

}  // namespace svg
