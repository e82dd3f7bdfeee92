// Host-side launchers shared between the translation units of libsvgear.so.
// Every launcher only enqueues on `st` and returns cudaGetLastError().
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/svgear.h"

namespace svg {

// Device status word of the current device (see svgear_get_status).
int* status_word();

// Counts kernel launches issued by the library (svgear_launch_count).
void note_launch();

// Self-test of the bounded in-kernel waits: one block whose wait on a barrier
// that nothing completes gives up after limit_ns (ST_TIMEOUT).
cudaError_t selftest_wait_run(uint64_t limit_ns, cudaStream_t st);

// Host-side validation of an operator parameter block (svgear_status code).
int params_status(const svgear_params* p);

// ---- stable counting sort of labels (shared by k-means update and permute)
// chunk = tokens per scatter chunk; nchunk = ceil(N / chunk)
constexpr int kSortChunk = 2048;
size_t sort_ws_bytes(int H, int N, int C);
// Fills counts [H,C], offsets [H,C+1] and (if perm != null) perm [H,N].
cudaError_t cluster_sort(const int32_t* labels, int H, int N, int C, int32_t* counts,
                         int32_t* offsets, int32_t* perm, void* ws, cudaStream_t st);

// ---- k-means
size_t kmeans_ws_bytes(int H, int N, int d, int C);
cudaError_t kmeans_run(const void* X, int dtype, int H, int N, int d, int C, int iters,
                       const float* init, float* cent, int32_t* labels, int32_t* counts,
                       int32_t* offsets_out, int32_t* perm_out, void* ws, cudaStream_t st);

// ---- permute / value centroids / per-key scalars
cudaError_t gather_rows(const void* X, int dtype, const int32_t* perm, int H, int N, int d,
                        void* Xp, cudaStream_t st);
cudaError_t value_stats(const void* Vp, int dtype, const int32_t* off, int H, int N, int d,
                        int C, float* Vbar, float* key_scalars, cudaStream_t st);

// ---- block error
// Workspace: centroid logits [H,Cq,Ck] float, then (tensor-core path) the
// hi/lo query-centroid operand.
size_t block_error_ws_bytes(int H, int Cq, int Ck, int d, int dtype);
cudaError_t block_error_run(const float* Qbar, const float* Kbar, const float* Vbar,
                            const void* Kp, const void* Vp, const int32_t* k_off,
                            const float* key_scalars, int dtype, int H, int Nk, int d, int Cq,
                            int Ck, float scale, float* E, float* M, void* ws, cudaStream_t st,
                            int router = 0, bool allow_tc = true);
// tensor-core kernel (block_error_tc.cu); L and M already computed
bool block_error_tc_shape_ok(int dtype, int d, int Cq);
bool block_error_tc_supported(int dtype, int d, int Cq, int Nk);
size_t block_error_tc_ws_bytes(int H, int d);
cudaError_t block_error_tc_run(const float* Qbar, const void* Kp, const int32_t* k_off, const float* ks,
                               const float* L, const float* M, int H, int Nk, int d, int Cq, int Ck,
                               float scale, float* E, void* ws, cudaStream_t st, bool value_agnostic);

// ---- routing
cudaError_t route_run(const float* E, const int32_t* k_counts, const int32_t* q_counts,
                      int H, int Nk, int Cq, int Ck, float rho, uint8_t* mask, int32_t* sel,
                      int32_t* n_sel, int64_t* exec_pairs, cudaStream_t st,
                      const float* M_global = nullptr, int Nq = 0);
// floor(rho * Nq * Nk) in exact integer arithmetic (global budget, pairs)
long long route_global_budget(float rho, long long Nq, long long Nk);

// ---- hybrid attention
size_t attn_ws_bytes(int H, int Nq, int Nk, int d, int Cq, int Ck);
cudaError_t attn_run(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                     const int32_t* k_off, const int32_t* perm_q, const float* Kbar,
                     const float* Vbar, const int32_t* sel, const int32_t* n_sel, int dtype,
                     int H, int Nq, int Nk, int d, int Cq, int Ck, float scale, void* O,
                     void* ws, cudaStream_t st);

// ---- TMA tensor maps (tma_host.cu)
constexpr int kTmaMapBytes = 128;
bool tma_available();
// Tiled map of a bf16 tensor [d2][d1][d0] (d0 contiguous) with box
// {64, box1, 1} and 128-byte swizzle, written to `map` (kTmaMapBytes bytes,
// 64-byte aligned).  Out-of-range rows read as zeros.  False when the driver
// entry point is missing or the arguments are not encodable.
bool tma_map_bf16_3d(void* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over a caller-provided workspace.
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* p) : base(static_cast<char*>(p)) {}
  template <typename T> T* take(size_t n) {
    off = align_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
  size_t used() const { return align_up(off, 256); }
};

}  // namespace svg
