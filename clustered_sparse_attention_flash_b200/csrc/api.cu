// C ABI of libsvgear.so: validation, workspace layout and stage chaining.
// The declarations, with the argument contracts, are in include/svgear.h.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <vector>

#include "../../include/svgear.h"
#include "common.cuh"
#include "internal.h"
#include "attn_tc.cuh"

namespace svg {

__device__ int g_status_word;

static std::atomic<long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int* status_word() {
  static int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int esize(int dtype) { return dtype == DT_BF16 ? 2 : 4; }
inline cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }
inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? SVGEAR_OK : SVGEAR_ERR_CUDA; }

int check_shape(int H, int N, int d, int C, int dtype) {
  if (H < 1 || N < 1 || C < 1 || C > N) return SVGEAR_ERR_INVALID;
  if ((long long)H * N * 128 > (1LL << 40)) return SVGEAR_ERR_INVALID;
  if (dtype != SVGEAR_F32 && dtype != SVGEAR_BF16) return SVGEAR_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return SVGEAR_ERR_UNSUPPORTED;
  return SVGEAR_OK;
}

int check_params(const svgear_params* p) {
  if (!p) return SVGEAR_ERR_INVALID;
  int r = check_shape(p->H, p->Nq, p->d, p->Cq, p->dtype);
  if (r) return r;
  r = check_shape(p->H, p->Nk, p->d, p->Ck, p->dtype);
  if (r) return r;
  if (p->iters < 0 || p->iters > 1000) return SVGEAR_ERR_INVALID;
  if (!(p->rho >= 0.f && p->rho <= 1.f)) return SVGEAR_ERR_INVALID;
  if (std::isnan(p->scale) || std::isinf(p->scale)) return SVGEAR_ERR_INVALID;
  if (p->Ck > kMaxCkBits) return SVGEAR_ERR_UNSUPPORTED;
  if (p->router < SVGEAR_ROUTE_ERROR || p->router > SVGEAR_ROUTE_ERROR_NOV) return SVGEAR_ERR_INVALID;
  if (p->budget != SVGEAR_BUDGET_ROW && p->budget != SVGEAR_BUDGET_GLOBAL) return SVGEAR_ERR_INVALID;
  if (p->budget == SVGEAR_BUDGET_GLOBAL && (unsigned long long)p->Nq * (unsigned long long)p->Nk >= (1ull << 62))
    return SVGEAR_ERR_UNSUPPORTED;
  return SVGEAR_OK;
}

}  // namespace

int params_status(const svgear_params* p) { return check_params(p); }

namespace {

float eff_scale(const svgear_params* p) {
  return p->scale > 0.f ? p->scale : 1.0f / std::sqrt((float)p->d);
}

struct FwdLayout {
  float *cent_q, *cent_k, *vbar, *key_scalars, *E, *M;
  int32_t *labels_q, *labels_k, *counts_q, *counts_k, *perm_q, *perm_k, *off_q, *off_k, *sel, *n_sel;
  void *Qp, *Kp, *Vp, *scratch, *scratch_q;
  uint8_t* mask;
  int64_t* exec_pairs;
  size_t scratch_bytes, total;
};

FwdLayout layout(const svgear_params* p, void* ws) {
  const int H = p->H, Nq = p->Nq, Nk = p->Nk, d = p->d, Cq = p->Cq, Ck = p->Ck;
  const size_t es = esize(p->dtype);
  Carve cv(ws);
  FwdLayout L;
  L.cent_q = cv.take<float>((size_t)H * Cq * d);
  L.cent_k = cv.take<float>((size_t)H * Ck * d);
  L.vbar = cv.take<float>((size_t)H * Ck * d);
  L.labels_q = cv.take<int32_t>((size_t)H * Nq);
  L.labels_k = cv.take<int32_t>((size_t)H * Nk);
  L.counts_q = cv.take<int32_t>((size_t)H * Cq);
  L.counts_k = cv.take<int32_t>((size_t)H * Ck);
  L.perm_q = cv.take<int32_t>((size_t)H * Nq);
  L.perm_k = cv.take<int32_t>((size_t)H * Nk);
  L.off_q = cv.take<int32_t>((size_t)H * (Cq + 1));
  L.off_k = cv.take<int32_t>((size_t)H * (Ck + 1));
  L.Qp = cv.take<char>((size_t)H * Nq * d * es);
  L.Kp = cv.take<char>((size_t)H * Nk * d * es);
  L.Vp = cv.take<char>((size_t)H * Nk * d * es);
  L.key_scalars = cv.take<float>((size_t)3 * H * Nk);
  L.E = cv.take<float>((size_t)H * Cq * Ck);
  L.M = cv.take<float>((size_t)H * Cq);
  L.mask = cv.take<uint8_t>((size_t)H * Cq * Ck);
  L.sel = cv.take<int32_t>((size_t)H * Cq * Ck);
  L.n_sel = cv.take<int32_t>((size_t)H * Cq);
  L.exec_pairs = cv.take<int64_t>(H);
  // The query clustering runs beside the key clustering, so it has scratch of its own.
  L.scratch_q = cv.take<char>(kmeans_ws_bytes(H, Nq, d, Cq));
  size_t sb = kmeans_ws_bytes(H, Nk, d, Ck);
  sb = std::max(sb, block_error_ws_bytes(H, Cq, Ck, d, p->dtype));
  sb = std::max(sb, attn_ws_bytes(H, Nq, Nk, d, Cq, Ck));
  L.scratch = cv.take<char>(sb);
  L.scratch_bytes = sb;
  L.total = cv.used();
  return L;
}

// A second stream per host thread and device, at the device's highest priority:
// the key clustering and everything that follows it up to the block error run
// there, the query clustering stays on the caller's stream and fills the SMs the
// key chain leaves idle.  Fork and join are event waits, so the pair also records
// into a CUDA graph captured on the caller's stream.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

SideStream* side_stream() {
  thread_local SideStream cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& c = cache[dev];
  if (!c.s) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&c.s, cudaStreamNonBlocking, greatest) != cudaSuccess) {
      c.s = nullptr;
      return nullptr;
    }
    if (cudaEventCreateWithFlags(&c.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.join, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamDestroy(c.s);
      c = SideStream{};
      return nullptr;
    }
  }
  return &c;
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" {

const char* svgear_version(void) { return "svgear 0.1 (sm_100a)"; }

long long svgear_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* svgear_status_string(int s) {
  switch (s) {
    case SVGEAR_OK: return "ok";
    case SVGEAR_ERR_INVALID: return "invalid argument";
    case SVGEAR_ERR_UNSUPPORTED: return "unsupported configuration";
    case SVGEAR_ERR_CUDA: return "CUDA error";
    case SVGEAR_ERR_TIMEOUT: return "in-kernel wait timed out";
    case SVGEAR_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int svgear_get_status(void* stream) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return SVGEAR_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)) != cudaSuccess) return SVGEAR_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return SVGEAR_ERR_CUDA;
  if (v == ST_OK) return SVGEAR_OK;
  if (v == ST_TIMEOUT) return SVGEAR_ERR_TIMEOUT;
  return SVGEAR_ERR_INVALID;
}

int svgear_selftest_wait(long long limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000LL) return SVGEAR_ERR_INVALID;
  if (!status_word()) return SVGEAR_ERR_CUDA;
  return cuda_status(selftest_wait_run((uint64_t)limit_ns, S(stream)));
}

size_t svgear_kmeans_workspace_size(int H, int N, int d, int C) {
  if (check_shape(H, N, d, C, SVGEAR_F32)) return 0;
  return kmeans_ws_bytes(H, N, d, C);
}

int svgear_kmeans(const void* X, int dtype, int H, int N, int d, int C, int iters, const float* init,
                  float* cent, int32_t* labels, int32_t* counts, void* ws, size_t ws_bytes,
                  void* stream) {
  int r = check_shape(H, N, d, C, dtype);
  if (r) return r;
  if (iters < 0 || iters > 1000) return SVGEAR_ERR_INVALID;
  if (!X || !cent || !labels || !counts || !aligned16(X) || !aligned16(cent)) return SVGEAR_ERR_INVALID;
  if (init && !aligned16(init)) return SVGEAR_ERR_INVALID;
  if (!ws || ws_bytes < kmeans_ws_bytes(H, N, d, C)) return SVGEAR_ERR_WORKSPACE;
  return cuda_status(kmeans_run(X, dtype, H, N, d, C, iters, init, cent, labels, counts, nullptr,
                                nullptr, ws, S(stream)));
}

size_t svgear_permute_workspace_size(int H, int N, int C) {
  if (H < 1 || N < 1 || C < 1 || C > N) return 0;
  return sort_ws_bytes(H, N, C);
}

int svgear_permute(const void* X, int dtype, const int32_t* labels, int H, int N, int d, int C,
                   void* Xp, int32_t* perm, int32_t* offsets, const void* V, void* Vp,
                   float* Vbar, float* key_scalars, void* ws, size_t ws_bytes, void* stream) {
  int r = check_shape(H, N, d, C, dtype);
  if (r) return r;
  if (!X || !labels || !Xp || !perm || !offsets || !aligned16(X) || !aligned16(Xp))
    return SVGEAR_ERR_INVALID;
  if (V && (!Vp || !aligned16(V) || !aligned16(Vp))) return SVGEAR_ERR_INVALID;
  if (!V && (Vp || Vbar || key_scalars)) return SVGEAR_ERR_INVALID;
  if (!ws || ws_bytes < sort_ws_bytes(H, N, C)) return SVGEAR_ERR_WORKSPACE;
  cudaStream_t st = S(stream);
  cudaError_t e = cluster_sort(labels, H, N, C, nullptr, offsets, perm, ws, st);
  if (e == cudaSuccess) e = gather_rows(X, dtype, perm, H, N, d, Xp, st);
  if (e == cudaSuccess && V) e = gather_rows(V, dtype, perm, H, N, d, Vp, st);
  if (e == cudaSuccess && V && (Vbar || key_scalars))
    e = value_stats(Vp, dtype, offsets, H, N, d, C, Vbar, key_scalars, st);
  return cuda_status(e);
}

size_t svgear_block_error_workspace_size(const svgear_params* p) {
  if (check_params(p)) return 0;
  return block_error_ws_bytes(p->H, p->Cq, p->Ck, p->d, p->dtype);
}

int svgear_block_error(const float* Qbar, const float* Kbar, const float* Vbar, const void* Kp,
                       const void* Vp, const int32_t* k_off, const float* key_scalars,
                       const svgear_params* p, float* E, float* M, void* ws, size_t ws_bytes,
                       void* stream) {
  int r = check_params(p);
  if (r) return r;
  if (!Qbar || !Kbar || !k_off || !E || !M) return SVGEAR_ERR_INVALID;
  if (p->router != SVGEAR_ROUTE_MASS && !Kp) return SVGEAR_ERR_INVALID;
  if (p->router == SVGEAR_ROUTE_ERROR && !key_scalars) return SVGEAR_ERR_INVALID;
  if (!aligned16(Qbar) || !aligned16(Kbar) || !aligned16(Kp)) return SVGEAR_ERR_INVALID;
  if (!ws || ws_bytes < block_error_ws_bytes(p->H, p->Cq, p->Ck, p->d, p->dtype)) return SVGEAR_ERR_WORKSPACE;
  return cuda_status(block_error_run(Qbar, Kbar, Vbar, Kp, Vp, k_off, key_scalars, p->dtype, p->H,
                                     p->Nk, p->d, p->Cq, p->Ck, eff_scale(p), E, M, ws, S(stream),
                                     p->router));
}

int svgear_route(const float* E, const int32_t* k_counts, const int32_t* q_counts,
                 const svgear_params* p, uint8_t* mask, int32_t* sel, int32_t* n_sel,
                 int64_t* exec_pairs, void* stream) {
  int r = check_params(p);
  if (r) return r;
  if (!E || !k_counts || !q_counts || !mask || !sel || !n_sel || !exec_pairs) return SVGEAR_ERR_INVALID;
  return cuda_status(route_run(E, k_counts, q_counts, p->H, p->Nk, p->Cq, p->Ck, p->rho, mask, sel,
                               n_sel, exec_pairs, S(stream)));
}

int svgear_route_global(const float* E, const float* M, const int32_t* k_counts, const int32_t* q_counts,
                        const svgear_params* p, uint8_t* mask, int32_t* sel, int32_t* n_sel,
                        int64_t* exec_pairs, void* stream) {
  int r = check_params(p);
  if (r) return r;
  if (!E || !M || !k_counts || !q_counts || !mask || !sel || !n_sel || !exec_pairs) return SVGEAR_ERR_INVALID;
  if ((unsigned long long)p->Nq * (unsigned long long)p->Nk >= (1ull << 62)) return SVGEAR_ERR_UNSUPPORTED;
  return cuda_status(route_run(E, k_counts, q_counts, p->H, p->Nk, p->Cq, p->Ck, p->rho, mask, sel,
                               n_sel, exec_pairs, S(stream), M, p->Nq));
}

size_t svgear_hybrid_attn_workspace_size(const svgear_params* p) {
  if (check_params(p)) return 0;
  return attn_ws_bytes(p->H, p->Nq, p->Nk, p->d, p->Cq, p->Ck);
}

int svgear_hybrid_attn(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                       const int32_t* k_off, const int32_t* perm_q, const float* Kbar,
                       const float* Vbar, const int32_t* sel, const int32_t* n_sel,
                       const svgear_params* p, void* O, void* ws, size_t ws_bytes, void* stream) {
  int r = check_params(p);
  if (r) return r;
  if (!Qp || !Kp || !Vp || !q_off || !k_off || !perm_q || !Kbar || !Vbar || !sel || !n_sel || !O)
    return SVGEAR_ERR_INVALID;
  if (!aligned16(Qp) || !aligned16(Kp) || !aligned16(Vp) || !aligned16(O) || !aligned16(Kbar) ||
      !aligned16(Vbar))
    return SVGEAR_ERR_INVALID;
  if (!ws || ws_bytes < attn_ws_bytes(p->H, p->Nq, p->Nk, p->d, p->Cq, p->Ck)) return SVGEAR_ERR_WORKSPACE;
  return cuda_status(attn_run(Qp, Kp, Vp, q_off, k_off, perm_q, Kbar, Vbar, sel, n_sel, p->dtype,
                              p->H, p->Nq, p->Nk, p->d, p->Cq, p->Ck, eff_scale(p), O, ws, S(stream)));
}

size_t svgear_workspace_size(const svgear_params* p) {
  if (check_params(p)) return 0;
  return layout(p, nullptr).total;
}

int svgear_forward_views(const svgear_params* p, void* ws, size_t ws_bytes, svgear_views* out) {
  int r = check_params(p);
  if (r) return r;
  if (!ws || !out) return SVGEAR_ERR_INVALID;
  FwdLayout L = layout(p, ws);
  if (ws_bytes < L.total) return SVGEAR_ERR_WORKSPACE;
  out->cent_q = L.cent_q; out->cent_k = L.cent_k; out->vbar = L.vbar;
  out->labels_q = L.labels_q; out->labels_k = L.labels_k;
  out->counts_q = L.counts_q; out->counts_k = L.counts_k;
  out->perm_q = L.perm_q; out->perm_k = L.perm_k; out->off_q = L.off_q; out->off_k = L.off_k;
  out->Qp = L.Qp; out->Kp = L.Kp; out->Vp = L.Vp; out->key_scalars = L.key_scalars;
  out->E = L.E; out->M = L.M; out->mask = L.mask; out->sel = L.sel; out->n_sel = L.n_sel;
  out->exec_pairs = L.exec_pairs;
  return SVGEAR_OK;
}

int svgear_forward(const void* Q, const void* K, const void* V, const svgear_params* p,
                   const float* init_q, const float* init_k, void* O, void* ws, size_t ws_bytes,
                   void* stream, svgear_stats* stats) {
  int r = check_params(p);
  if (r) return r;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return SVGEAR_ERR_INVALID;
  if ((init_q && !aligned16(init_q)) || (init_k && !aligned16(init_k))) return SVGEAR_ERR_INVALID;
  if (!ws) return SVGEAR_ERR_WORKSPACE;
  FwdLayout L = layout(p, ws);
  if (ws_bytes < L.total) return SVGEAR_ERR_WORKSPACE;
  const int H = p->H, Nq = p->Nq, Nk = p->Nk, d = p->d, Cq = p->Cq, Ck = p->Ck, dt = p->dtype;
  const float sc = eff_scale(p);
  cudaStream_t st = S(stream);
  SideStream* side = side_stream();
  if (!side) return SVGEAR_ERR_CUDA;
  cudaEvent_t ev[9] = {};  // stage boundaries 0..6, then the attention kernel alone
  if (stats) {
    for (auto& e : ev)
      if (cudaEventCreate(&e) != cudaSuccess) return SVGEAR_ERR_CUDA;
  }
  auto mark = [&](int i) { if (stats) cudaEventRecord(ev[i], st); };
  cudaError_t e = cudaSuccess;
  mark(0);
  // The key chain on the side stream, the query clustering and gather on `st`.
  e = cudaEventRecord(side->fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side->s, side->fork, 0);
  const bool forked = e == cudaSuccess;
  cudaError_t ek = e, ej = e;
  if (forked) {
    cudaStream_t sk = side->s;
    ek = kmeans_run(K, dt, H, Nk, d, Ck, p->iters, init_k, L.cent_k, L.labels_k, L.counts_k,
                    L.off_k, L.perm_k, L.scratch, sk);
    if (stats) cudaEventRecord(ev[2], sk);
    if (ek == cudaSuccess) ek = gather_rows(K, dt, L.perm_k, H, Nk, d, L.Kp, sk);
    if (ek == cudaSuccess) ek = gather_rows(V, dt, L.perm_k, H, Nk, d, L.Vp, sk);
    if (ek == cudaSuccess) ek = value_stats(L.Vp, dt, L.off_k, H, Nk, d, Ck, L.vbar, L.key_scalars, sk);
    // Recorded whatever happened above: `st` always waits for the side stream.
    ej = cudaEventRecord(side->join, sk);
  }
  if (e == cudaSuccess)
    e = kmeans_run(Q, dt, H, Nq, d, Cq, p->iters, init_q, L.cent_q, L.labels_q, L.counts_q,
                   L.off_q, L.perm_q, L.scratch_q, st);
  mark(1);
  if (e == cudaSuccess) e = gather_rows(Q, dt, L.perm_q, H, Nq, d, L.Qp, st);
  if (forked) {
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, side->join, 0);
    if (ej != cudaSuccess) cudaStreamSynchronize(side->s);
  }
  if (e == cudaSuccess) e = ek;
  if (e == cudaSuccess) e = ej;
  mark(3);
  if (e == cudaSuccess)
    e = block_error_run(L.cent_q, L.cent_k, L.vbar, L.Kp, L.Vp, L.off_k, L.key_scalars, dt, H, Nk, d,
                        Cq, Ck, sc, L.E, L.M, L.scratch, st, p->router);
  mark(4);
  if (e == cudaSuccess)
    e = route_run(L.E, L.counts_k, L.counts_q, H, Nk, Cq, Ck, p->rho, L.mask, L.sel, L.n_sel,
                  L.exec_pairs, st, p->budget == SVGEAR_BUDGET_GLOBAL ? L.M : nullptr, Nq);
  mark(5);
  if (stats) attn_tc_time_next_kernel(ev[7], ev[8]);
  if (e == cudaSuccess)
    e = attn_run(L.Qp, L.Kp, L.Vp, L.off_q, L.off_k, L.perm_q, L.cent_k, L.vbar, L.sel, L.n_sel, dt,
                 H, Nq, Nk, d, Cq, Ck, sc, O, L.scratch, st);
  const bool kernel_timed = stats && attn_tc_kernel_was_timed();
  if (stats) attn_tc_time_next_kernel(nullptr, nullptr);
  mark(6);
  if (stats && e == cudaSuccess) {
    e = cudaStreamSynchronize(st);
    float t[6] = {};
    for (int i = 0; i < 6 && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&t[i], ev[i], ev[i + 1]);
    // Both clusterings start at ev[0]: ev[1] ends the query one, ev[2] (on the
    // side stream) the key one; the permute stage runs from ev[2] to the join.
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t[1], ev[0], ev[2]);
    if (e == cudaSuccess) {
      stats->ms_kmeans_q = t[0]; stats->ms_kmeans_k = t[1]; stats->ms_permute = t[2];
      stats->ms_block_error = t[3]; stats->ms_route = t[4]; stats->ms_attn = t[5];
      cudaEventElapsedTime(&stats->ms_total, ev[0], ev[6]);
      stats->ms_attn_kernel = stats->ms_attn;
      if (kernel_timed) cudaEventElapsedTime(&stats->ms_attn_kernel, ev[7], ev[8]);
      std::vector<int64_t> ep(H);
      std::vector<int32_t> cq((size_t)H * Cq), ck((size_t)H * Ck), ns((size_t)H * Cq);
      e = cudaMemcpy(ep.data(), L.exec_pairs, H * sizeof(int64_t), cudaMemcpyDeviceToHost);
      if (e == cudaSuccess) e = cudaMemcpy(cq.data(), L.counts_q, cq.size() * 4, cudaMemcpyDeviceToHost);
      if (e == cudaSuccess) e = cudaMemcpy(ck.data(), L.counts_k, ck.size() * 4, cudaMemcpyDeviceToHost);
      if (e == cudaSuccess) e = cudaMemcpy(ns.data(), L.n_sel, ns.size() * 4, cudaMemcpyDeviceToHost);
      int64_t pairs = 0, comp = 0;
      for (int h = 0; h < H && e == cudaSuccess; ++h) {
        pairs += ep[h];
        int nonempty = 0;
        for (int c = 0; c < Ck; ++c) nonempty += ck[(size_t)h * Ck + c] > 0;
        for (int a = 0; a < Cq; ++a)
          comp += (int64_t)cq[(size_t)h * Cq + a] * (nonempty - ns[(size_t)h * Cq + a]);
      }
      stats->exec_pairs = pairs;
      stats->comp_pairs = comp;
    }
  }
  if (stats)
    for (auto& x : ev) cudaEventDestroy(x);
  return cuda_status(e);
}

}  // extern "C"
