// Stable counting sort of cluster labels: histogram per chunk, one exclusive
// scan per head over (cluster, chunk), then an order-preserving scatter.
// Used by the k-means update (cluster membership lists) and by the token
// reordering that makes every cluster contiguous (SVG-EAR review, step (1)).
#include "common.cuh"
#include "internal.h"

namespace svg {

namespace {

__global__ void k_chunk_hist(const int32_t* __restrict__ labels, int N, int C, int nchunk,
                             int32_t* __restrict__ bh, int* status) {
  extern __shared__ int32_t hist[];
  const int h = blockIdx.y, chunk = blockIdx.x;
  for (int c = threadIdx.x; c < C; c += blockDim.x) hist[c] = 0;
  __syncthreads();
  const int32_t* lab = labels + (size_t)h * N;
  const int beg = chunk * kSortChunk, end = min(N, beg + kSortChunk);
  for (int i = beg + threadIdx.x; i < end; i += blockDim.x) {
    int l = lab[i];
    if ((unsigned)l < (unsigned)C) atomicAdd(&hist[l], 1);
    else set_status(status, ST_BOUNDS);
  }
  __syncthreads();
  int32_t* out = bh + (size_t)h * C * nchunk + chunk;
  for (int c = threadIdx.x; c < C; c += blockDim.x) out[(size_t)c * nchunk] = hist[c];
}

// One block per head: exclusive scan over the head's C*nchunk entries, in
// tiles of 4 consecutive entries per thread (coalesced) with a running carry.
__global__ void __launch_bounds__(1024) k_scan(int32_t* __restrict__ bh, int C, int nchunk, int N,
                                               int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  __shared__ int32_t warp_tot[32];
  const int h = blockIdx.x;
  const long long M = (long long)C * nchunk;
  int32_t* a = bh + (size_t)h * M;
  const int T = blockDim.x, nw = T >> 5;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int32_t carry = 0;
  for (long long t0 = 0; t0 < M; t0 += 4LL * T) {
    const long long i0 = t0 + 4LL * threadIdx.x;
    int32_t x[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = (i0 + k < M) ? a[i0 + k] : 0;
    const int32_t s = x[0] + x[1] + x[2] + x[3];
    int32_t v = s;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[w] = v;
    __syncthreads();
    if (w == 0) {
      int32_t t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += u;
      }
      warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    int32_t run = carry + v - s + (w > 0 ? warp_tot[w - 1] : 0);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (i0 + k < M) a[i0 + k] = run;
      run += x[k];
    }
    carry += warp_tot[nw - 1];
    __syncthreads();
  }
  int32_t* off = offsets + (size_t)h * (C + 1);
  for (int c = threadIdx.x; c < C; c += T) off[c] = a[(size_t)c * nchunk];
  if (threadIdx.x == 0) off[C] = N;
  __syncthreads();
  if (counts)
    for (int c = threadIdx.x; c < C; c += T) counts[(size_t)h * C + c] = off[c + 1] - off[c];
}

// One warp per chunk walks its tokens in order, 32 at a time; equal labels in a
// group of 32 are ranked by lane, so the scatter keeps the original order.
__global__ void k_scatter(const int32_t* __restrict__ labels, int N, int C, int nchunk,
                          const int32_t* __restrict__ bh, int32_t* __restrict__ perm) {
  extern __shared__ int32_t cnt[];
  const int h = blockIdx.y, chunk = blockIdx.x, lane = threadIdx.x;
  const int32_t* base = bh + (size_t)h * C * nchunk + chunk;
  for (int c = lane; c < C; c += 32) cnt[c] = base[(size_t)c * nchunk];
  __syncwarp();
  const int32_t* lab = labels + (size_t)h * N;
  int32_t* pm = perm + (size_t)h * N;
  const int beg = chunk * kSortChunk, end = min(N, beg + kSortChunk);
  for (int g = beg; g < end; g += 32) {
    const int i = g + lane;
    int l = (i < end) ? lab[i] : -1;
    if ((unsigned)l >= (unsigned)C) l = -1;  // out of range: reported by the histogram
    const unsigned peers = __match_any_sync(0xffffffffu, l);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (l >= 0) pos = cnt[l] + rank;
    __syncwarp();
    if (l >= 0 && rank == 0) cnt[l] += __popc(peers);
    __syncwarp();
    if (l >= 0) pm[pos] = i;
  }
}

}  // namespace

size_t sort_ws_bytes(int H, int N, int C) {
  const int nchunk = (N + kSortChunk - 1) / kSortChunk;
  return align_up((size_t)H * C * nchunk * sizeof(int32_t), 256);
}

cudaError_t cluster_sort(const int32_t* labels, int H, int N, int C, int32_t* counts,
                         int32_t* offsets, int32_t* perm, void* ws, cudaStream_t st) {
  const int nchunk = (N + kSortChunk - 1) / kSortChunk;
  int32_t* bh = static_cast<int32_t*>(ws);
  const size_t sh = (size_t)C * sizeof(int32_t);
  k_chunk_hist<<<dim3(nchunk, H), 256, sh, st>>>(labels, N, C, nchunk, bh, status_word()); note_launch();
  k_scan<<<H, 1024, 0, st>>>(bh, C, nchunk, N, counts, offsets); note_launch();
  if (perm) { k_scatter<<<dim3(nchunk, H), 32, sh, st>>>(labels, N, C, nchunk, bh, perm); note_launch(); }
  return cudaGetLastError();
}

}  // namespace svg
