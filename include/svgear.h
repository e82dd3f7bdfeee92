/*
 * svgear.h -- C ABI of libsvgear.so, the B200 (sm_100a) SVG-EAR sparse-attention
 * operator.
 *
 * The operator is the inference pipeline of "SVG-EAR: Parameter-Free Linear
 * Compensation for Sparse Video Generation via Error-aware Routing"
 * (arXiv 2603.08982), as summarised by the paper.rainbus.top review
 * ("complete inference pipeline", steps (1)-(5)) and the gist.science technical
 * summaries (sections 2.A-2.C):
 *   (1) semantic k-means of queries and keys, tokens reordered so that every
 *       cluster is contiguous                         -> svgear_kmeans, svgear_permute
 *   (2) value-aware block error with the query-centroid proxy
 *                                                     -> svgear_block_error
 *   (3) error-to-cost greedy routing under the density budget rho
 *                                                     -> svgear_route
 *   (4) hybrid attention: exact softmax attention on routed blocks, centroid
 *       linear compensation on the rest, one joint softmax
 *                                                     -> svgear_hybrid_attn
 *   all of it on one stream                           -> svgear_forward
 *
 * Conventions (every entry point):
 *  - Tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates device memory; scratch comes from a caller-provided
 *    workspace whose size the matching *_workspace_size call returns.
 *  - Tensors are dense and row-major, per head h: X[h][n][t] at
 *    X + (h*N + n)*d + t.  Rows must be 16-byte aligned (d in {64, 128}).
 *    Element type of Q/K/V-like tensors is `dtype` (float32 or bfloat16);
 *    centroids, errors and per-key scalars are float32; indices int32.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream); every call only
 *    enqueues work and returns.  Calls on one stream run in order.
 *  - The return value reports host-side validation and launch errors only
 *    (svgear_status).  Nothing is enqueued when validation fails.  Faults
 *    and timed-out waits inside kernels are recorded in a device status word
 *    that svgear_get_status reads.
 *  - No exceptions or aborts cross the ABI.
 *  - The library looks up the device addresses of its own device variables
 *    (the status word; the scratch array of svgear_block_error_noalloc) once
 *    per device and keeps them for the life of the process.  After a
 *    cudaDeviceReset the module is loaded again at new addresses, so a
 *    process that resets a device must not call the library on it again.
 */
#ifndef SVGEAR_H
#define SVGEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVGEAR_API __attribute__((visibility("default")))
#else
#define SVGEAR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVGEAR_OK = 0,
  SVGEAR_ERR_INVALID = -1,     /* bad argument (null pointer, size, range) */
  SVGEAR_ERR_UNSUPPORTED = -2, /* valid but not implemented (d, dtype) */
  SVGEAR_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
  SVGEAR_ERR_TIMEOUT = -4,     /* a bounded in-kernel wait gave up */
  SVGEAR_ERR_WORKSPACE = -5    /* workspace missing or too small */
} svgear_status;

typedef enum { SVGEAR_F32 = 0, SVGEAR_BF16 = 1 } svgear_dtype;

/* What svgear_block_error stores in E, i.e. the signal the router ranks key
 * clusters by.  Only SVGEAR_ROUTE_ERROR is the method; the other two are
 * ablations that swap the ranking signal and keep every other step.
 *   SVGEAR_ROUTE_ERROR      value-aware error-to-cost ratio (review step (2),
 *                           gist.science 2.B): the default, 0.
 *   SVGEAR_ROUTE_MASS       estimated attention mass of each key cluster for
 *                           the query centroid, |k_c| e^{s qbar_a.kbar_c},
 *                           normalised to sum 1 over the non-empty clusters of
 *                           the row -- a score-based router in the manner of
 *                           the top-p selectors the pages compare against.
 *   SVGEAR_ROUTE_ERROR_NOV  value-agnostic error: eps^2 without the values,
 *                           (e^{s qbar_a.kbar_c} - e^{s qbar_a.k_j})^2, same
 *                           shift and per-key average as the default. */
typedef enum {
  SVGEAR_ROUTE_ERROR = 0,
  SVGEAR_ROUTE_MASS = 1,
  SVGEAR_ROUTE_ERROR_NOV = 2
} svgear_router;

/* How svgear_forward spends the density budget.
 *   SVGEAR_BUDGET_ROW     floor(rho * Nk) keys for every query cluster
 *                         (review step (3)): the default, 0.
 *   SVGEAR_BUDGET_GLOBAL  one budget of floor(rho * Nq * Nk) query-key pairs
 *                         per head over all blocks (svgear_route_global). */
typedef enum { SVGEAR_BUDGET_ROW = 0, SVGEAR_BUDGET_GLOBAL = 1 } svgear_budget;

/* Operator hyper-parameters of one attention layer. */
typedef struct {
  int H;        /* heads (independent problems) */
  int Nq, Nk;   /* query / key tokens per head */
  int d;        /* head dimension: 64 or 128 */
  int Cq, Ck;   /* query / key clusters, 1 <= C <= N */
  int iters;    /* k-means assign->update rounds (>= 0) */
  float rho;    /* density budget in [0, 1]: each query cluster computes at
                   most floor(rho * Nk) keys exactly */
  float scale;  /* softmax scale; <= 0 selects 1/sqrt(d) */
  int dtype;    /* svgear_dtype of Q, K, V and the output */
  int router;   /* svgear_router: what E ranks by; 0 (zero-initialised
                   params) is the method's value-aware error */
  int budget;   /* svgear_budget: per query cluster (0) or per head (1);
                   read by svgear_forward only */
} svgear_params;

/* Per-stage device times of one svgear_forward call (CUDA events).  The two
 * clusterings run side by side, so ms_kmeans_q and ms_kmeans_k both start at the
 * call's start and overlap; ms_permute runs from the end of the key clustering
 * to the point where both permuted halves are ready. */
typedef struct {
  float ms_kmeans_q, ms_kmeans_k, ms_permute, ms_block_error, ms_route, ms_attn;
  float ms_total;
  int64_t exec_pairs;   /* sum over heads of sum_a |q_a| * sum_{c routed} |k_c| */
  int64_t comp_pairs;   /* sum over heads of sum_a |q_a| * #compensated non-empty c */
  float ms_attn_kernel; /* the hybrid-attention kernel alone (ms_attn less its staging
                           kernels); equal to ms_attn on the float32 path */
} svgear_stats;

/* Device pointers to the intermediates svgear_forward leaves in its workspace. */
typedef struct {
  float *cent_q, *cent_k;          /* [H,Cq,d], [H,Ck,d] k-means centroids */
  float *vbar;                     /* [H,Ck,d] value centroids */
  int32_t *labels_q, *labels_k;    /* [H,Nq], [H,Nk] */
  int32_t *counts_q, *counts_k;    /* [H,Cq], [H,Ck] */
  int32_t *perm_q, *perm_k;        /* [H,Nq], [H,Nk]: perm[new] = old */
  int32_t *off_q, *off_k;          /* [H,Cq+1], [H,Ck+1] */
  void *Qp, *Kp, *Vp;              /* permuted copies, dtype */
  float *key_scalars;              /* [3,H,Nk] */
  float *E, *M;                    /* [H,Cq,Ck], [H,Cq] */
  uint8_t *mask;                   /* [H,Cq,Ck] */
  int32_t *sel, *n_sel;            /* [H,Cq,Ck], [H,Cq] */
  int64_t *exec_pairs;             /* [H] */
} svgear_views;

/* Library version string (static storage). */
SVGEAR_API const char* svgear_version(void);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all streams); a host-side counter, no device access. */
SVGEAR_API long long svgear_launch_count(void);

/* Human-readable text of a status code (static storage, never NULL). */
SVGEAR_API const char* svgear_status_string(int status);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device: SVGEAR_OK, or SVGEAR_ERR_TIMEOUT when a bounded in-kernel
 * wait expired since the last call; SVGEAR_ERR_CUDA if the synchronisation
 * itself failed (a sticky CUDA error). */
SVGEAR_API int svgear_get_status(void* stream);

/* Self-test of the failure detection (no counterpart in the pages): enqueues
 * on `stream` one block that waits on an mbarrier nothing ever completes,
 * with the wait routine and the abort protocol of the operator's tensor-core
 * kernels but a limit of `limit_ns` nanoseconds (1e3 .. 1e9; other values
 * return SVGEAR_ERR_INVALID).  The wait gives up, the block releases its
 * tensor memory and ends, and the next svgear_get_status returns
 * SVGEAR_ERR_TIMEOUT; the context stays usable.  No device memory is
 * allocated and nothing else is touched. */
SVGEAR_API int svgear_selftest_wait(long long limit_ns, void* stream);

/* ---------------------------------------------------------------------------
 * (1) k-means (Lloyd) on X [H,N,d] with C clusters.  Review step (1), "Flash
 * k-means" clustering of queries and keys; gist.science summary 2.A.
 *   init    [H,C,d] float32 initial centroid values; NULL selects the
 *           deterministic init mu_c = x_{floor(c*N/C)}.
 *   cent    [H,C,d] float32 out: centroids after `iters` rounds of
 *           assign->update (an empty cluster keeps its previous centroid).
 *   labels  [H,N] int32 out: argmin_c ||x - mu_c||^2 against the final
 *           centroids (ties -> smaller index).
 *   counts  [H,C] int32 out: cluster sizes of `labels`.
 *   ws      device scratch of at least svgear_kmeans_workspace_size bytes.
 * Labels are exact: near-ties of the float32 tensor-core scores are re-decided
 * in float64.  Centroid sums are deterministic (no float atomics).
 * ------------------------------------------------------------------------- */
SVGEAR_API size_t svgear_kmeans_workspace_size(int H, int N, int d, int C);
SVGEAR_API int svgear_kmeans(const void* X, int dtype, int H, int N, int d, int C, int iters,
                  const float* init, float* cent, int32_t* labels, int32_t* counts,
                  void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * (1') Reorder tokens so that each cluster is contiguous.  Review step (1).
 * Stable counting sort by label: perm[h][new] = old, clusters in index
 * order, original order inside a cluster; offsets [H,C+1] exclusive prefix
 * of the cluster sizes.  Xp[h][new] = X[h][perm[h][new]].
 * When V is non-NULL (the keys' values, same N), also
 *   Vp      [H,N,d] values gathered with the same perm,
 *   Vbar    [H,C,d] float32 mean of v over each cluster (0 if empty),
 *   key_scalars [3,H,N] float32 in permuted order: ||vbar_c - v_j||^2,
 *           (vbar_c - v_j).v_j, ||v_j||^2 -- the per-key terms of the
 *           value-aware error expansion.  Vbar / key_scalars may be NULL.
 * ------------------------------------------------------------------------- */
SVGEAR_API size_t svgear_permute_workspace_size(int H, int N, int C);
SVGEAR_API int svgear_permute(const void* X, int dtype, const int32_t* labels, int H, int N,
                   int d, int C, void* Xp, int32_t* perm, int32_t* offsets,
                   const void* V, void* Vp, float* Vbar, float* key_scalars,
                   void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * (2) Value-aware block error with the query-centroid proxy.  Review step (2);
 * gist.science 2.B ("lightweight probe", O(C_q N_k d)).  For query cluster a
 * and key cluster c (keys j of c, s = scale):
 *   eps^2(a,j) = || exp(s qbar_a.kbar_c) vbar_c - exp(s qbar_a.k_j) v_j ||^2
 *   E[h][a][c] = exp(-2 M_a) * (1/|k_c|) * sum_{j in c} eps^2(a,j)
 *   M[h][a]    = max over non-empty c of s qbar_a.kbar_c
 * E is the pages' error-to-cost ratio times the positive per-row factor
 * exp(-2 M_a), which keeps it in float32 range and leaves the routing order
 * unchanged.  Empty key clusters get E = 0.
 * p->router selects an ablation instead (M as above in every mode):
 *   SVGEAR_ROUTE_MASS:      E[h][a][c] = |k_c| e^{s qbar_a.kbar_c - M_a} /
 *                           sum over non-empty c' of the same; Kp, Vp and
 *                           key_scalars are not read.
 *   SVGEAR_ROUTE_ERROR_NOV: eps^2(a,j) = (e^{s qbar_a.kbar_c} -
 *                           e^{s qbar_a.k_j})^2 in the formula above; Vbar,
 *                           Vp and key_scalars are not read.
 * Router values outside svgear_router return SVGEAR_ERR_INVALID.
 *   Qbar [H,Cq,d], Kbar/Vbar [H,Ck,d] float32; Kp/Vp [H,Nk,d] dtype (keys in
 *   cluster order); k_off [H,Ck+1]; key_scalars [3,H,Nk] from svgear_permute.
 * ------------------------------------------------------------------------- */
SVGEAR_API size_t svgear_block_error_workspace_size(const svgear_params* p);
SVGEAR_API int svgear_block_error(const float* Qbar, const float* Kbar, const float* Vbar,
                       const void* Kp, const void* Vp, const int32_t* k_off,
                       const float* key_scalars, const svgear_params* p,
                       float* E, float* M, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * svgear_block_error without a workspace argument.  No counterpart in the
 * paper: this entry point exists for callers that cannot allocate device
 * memory at the point of the call -- for example a runtime that plans all of
 * its device memory ahead of time and hands the operator only its inputs and
 * outputs, or a plug-in running inside a host framework that owns the device
 * allocator and exposes none of it.
 * Same arguments, results and errors as svgear_block_error, except:
 *   - the scratch buffer is a file-scope device array of this library of
 *     2,097,152 floats (8 MiB), held on every GPU that loads the library
 *     until the process exits; H * Cq * Ck above that limit returns
 *     SVGEAR_ERR_WORKSPACE without enqueuing anything;
 *   - the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept for the process, so
 *     the entry must not be called again on a device after cudaDeviceReset;
 *   - every call shares the one array, so calls that overlap on the GPU
 *     (different streams, or different host threads on one device) race and
 *     must be ordered by the caller.  Each call writes the scratch fully
 *     before reading it, so nothing carries over between calls.
 * It calls no device allocator (cudaMalloc, cudaFree or a library that
 * allocates).
 * ------------------------------------------------------------------------- */
SVGEAR_API int svgear_block_error_noalloc(const float* Qbar, const float* Kbar, const float* Vbar,
                       const void* Kp, const void* Vp, const int32_t* k_off,
                       const float* key_scalars, const svgear_params* p,
                       float* E, float* M, void* stream);

/* ---------------------------------------------------------------------------
 * (3) Error-aware routing.  Review step (3); gist.science 2.B "Selektion".
 * Per (h, a): non-empty key clusters in E-descending order (equal E: smaller
 * c first); the longest prefix whose total size fits floor(rho*Nk) is routed
 * to exact attention.
 *   mask [H,Cq,Ck] uint8 out (1 = exact), sel [H,Cq,Ck] int32 out (routed
 *   clusters in routing order, first n_sel[h][a] valid), n_sel [H,Cq] out,
 *   exec_pairs [H] int64 out (sum_a |q_a| * sum_{c routed} |k_c|).
 *   k_counts [H,Ck], q_counts [H,Cq] int32.  Ck <= 4096.
 * ------------------------------------------------------------------------- */
SVGEAR_API int svgear_route(const float* E, const int32_t* k_counts, const int32_t* q_counts,
                 const svgear_params* p, uint8_t* mask, int32_t* sel, int32_t* n_sel,
                 int64_t* exec_pairs, void* stream);

/* ---------------------------------------------------------------------------
 * (3') Global-budget routing: the knapsack form of the error-aware routing
 * (gist.science 2.B) taken over all blocks of a head at once.  Every block
 * (a, c) with |q_a| > 0 and |k_c| > 0 costs |q_a| |k_c| pairs and is ranked
 * by its unshifted error-to-cost ratio E[h][a][c] e^{2 M[h][a]}, compared as
 * logf(E) + 2 M in float32 (E = 0 ranks last); equal keys: smaller a*Ck + c
 * first.  The longest prefix whose total cost fits floor(rho * Nq * Nk)
 * (exact integer arithmetic on the float32 rho) is routed.
 *   E [H,Cq,Ck], M [H,Cq] from svgear_block_error (any router); the other
 *   arguments and outputs as svgear_route.  sel lists each row's routed
 *   clusters in that row's order; rows with |q_a| = 0 route nothing.
 *   Ck <= 4096; Nq * Nk < 2^62 (else SVGEAR_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------- */
SVGEAR_API int svgear_route_global(const float* E, const float* M, const int32_t* k_counts,
                        const int32_t* q_counts, const svgear_params* p, uint8_t* mask,
                        int32_t* sel, int32_t* n_sel, int64_t* exec_pairs, void* stream);

/* ---------------------------------------------------------------------------
 * (4) Hybrid attention.  Review step (4); gist.science 2.A "lineare
 * Kompensation".  For query i of cluster a (permuted order):
 *   o_i = sum over routed c, j in c of e^{s q_i.k_j} v_j
 *         + sum over compensated non-empty c of |k_c| e^{s q_i.kbar_c} vbar_c
 *         divided by the same sums without v  (one max, one normaliser)
 * and o_i is written to O[h][perm_q[h][i]] (original token order).
 *   Qp [H,Nq,d], Kp/Vp [H,Nk,d] dtype; q_off [H,Cq+1], k_off [H,Ck+1];
 *   Kbar/Vbar [H,Ck,d] float32; sel/n_sel from svgear_route; O [H,Nq,d] dtype.
 * ------------------------------------------------------------------------- */
SVGEAR_API size_t svgear_hybrid_attn_workspace_size(const svgear_params* p);
SVGEAR_API int svgear_hybrid_attn(const void* Qp, const void* Kp, const void* Vp,
                       const int32_t* q_off, const int32_t* k_off, const int32_t* perm_q,
                       const float* Kbar, const float* Vbar, const int32_t* sel,
                       const int32_t* n_sel, const svgear_params* p, void* O,
                       void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * The whole operator: (1) -> (1') -> (2) -> (3) -> (4) on one stream
 * ((3') instead of (3) when p->budget is SVGEAR_BUDGET_GLOBAL).
 *   The key clustering, the key/value gathers and (1') run on a second,
 *   highest-priority stream the library keeps per host thread and device,
 *   forked from `stream` by an event and joined back before (2), while the
 *   query clustering runs on `stream` beside them; to the caller the call still
 *   behaves as work on `stream` alone (ordering, graph capture).  Concurrent
 *   calls from one host thread on different streams share that second stream
 *   and serialise their key chains.  The first call on a host thread creates
 *   that stream and sets the kernels' shared-memory attributes: make it outside
 *   stream capture before recording svgear_forward into a CUDA graph.
 *   Q [H,Nq,d], K/V [H,Nk,d], O [H,Nq,d] in `dtype`.
 *   init_q [H,Cq,d] / init_k [H,Ck,d] float32 k-means initial centroids
 *   (NULL: deterministic init, see svgear_kmeans).
 *   ws: at least svgear_workspace_size(p) bytes; holds every intermediate
 *   (svgear_forward_views locates them).
 *   stats: NULL, or filled with per-stage device times -- then the call
 *   records CUDA events and synchronises `stream` before returning.
 * ------------------------------------------------------------------------- */
SVGEAR_API size_t svgear_workspace_size(const svgear_params* p);
SVGEAR_API int svgear_forward_views(const svgear_params* p, void* ws, size_t ws_bytes,
                         svgear_views* out);
SVGEAR_API int svgear_forward(const void* Q, const void* K, const void* V, const svgear_params* p,
                   const float* init_q, const float* init_k, void* O, void* ws,
                   size_t ws_bytes, void* stream, svgear_stats* stats);

#ifdef __cplusplus
}
#endif
#endif /* SVGEAR_H */
