"""SVG-EAR CPU oracle -- TEST INFRASTRUCTURE ONLY.

This module is the plain, slow, float64 statement of what the SVG-EAR
sparse-attention operator computes.  Only the test-suite, the package's
``smoke()`` self-check and the benchmark's CPU-baseline leg may import it; the
operator itself never calls it (the CUDA library has no CPU fallback).  It
shares no code with the CUDA path: inputs come from the seeded generator module,
everything else is written here from the method's description.

Sources (web pages on arXiv 2603.08982, "SVG-EAR: Parameter-Free Linear
Compensation for Sparse Video Generation via Error-aware Routing"):

* [R]  paper.rainbus.top review of SVG-EAR, "complete inference pipeline"
       paragraph, steps (1)-(5).
* [DE] gist.science/de technical summary, sections 2.A (clustering and linear
       compensation), 2.B (error-aware routing), 2.C (kernels).
* [IT] gist.science/it "Sommario tecnico", sections 2.A and 2.B.
* [AB] the SVG-EAR abstract (chatpaper.ai page).

Readings taken where the pages are silent (each listed in the design notes):

* k-means: Lloyd iterations on the raw vectors with squared Euclidean distance;
  exactly ``iters`` assign->update rounds, then one final assignment against
  the final centroids (labels and counts come from that assignment); an empty
  cluster keeps its previous centroid; argmin ties go to the smaller index.
* The value centroid of key cluster c is the mean of v_j over the keys whose
  final label is c (v travels with its key); 0 for an empty cluster.
* The block error is reported shifted by a per-query-cluster constant:
  E[a, c] = exp(-2 M_a) * (1/|k_c|) sum_{j in c} eps^2(a, j) with
  M_a = max over non-empty c of scale * qbar_a . kbar_c.  A positive per-row
  factor leaves the routing order unchanged.
* Routing: per query cluster, non-empty key clusters sorted by ratio
  descending (equal ratios: smaller index first); the longest prefix whose
  key count fits floor(rho * N_k) is computed exactly, rho taken as the
  float32 value the operator receives.
* Hybrid attention: every compensated key cluster contributes |k_c| copies of
  its centroid term, i.e. a logit bias log|k_c|, inside the same softmax as the
  exact keys (one maximum, one normaliser).
* Ablations (not the method; they swap one ingredient of the routing): a
  score-based signal, the attention weight |k_c| e^{s qbar.kbar_c} the query
  centroid gives each key cluster, normalised per row; the block error without
  the values; one budget of floor(rho N_q N_k) pairs per head over all blocks,
  ranked by the unshifted ratio.

Arrays are per head: X [N, d]; centroids [C, d]; labels [N] ints.

Precision: every function computes in float64.  `timing_precision` lets the
benchmark's CPU-baseline leg time the same code in float32 (the arithmetic
and the step order are unchanged, only the element type); parity checks
never use it.
"""
from __future__ import annotations

import math
from typing import Dict

import numpy as np

_ROW_CHUNK = 2048
_REAL = np.float64


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=_REAL)


class timing_precision:
    """Context manager: run the oracle in `dtype` (np.float32 for the CPU
    timing baseline) instead of float64 inside the `with` block."""

    def __init__(self, dtype):
        self.dtype = dtype

    def __enter__(self):
        global _REAL
        self.old, _REAL = _REAL, self.dtype
        return self

    def __exit__(self, *exc):
        global _REAL
        _REAL = self.old


# --------------------------------------------------------------------------
# (1) semantic clustering: k-means on queries and on keys      [R] step (1);
#     [DE] 2.A "Clustering"; [IT] 2.A
# --------------------------------------------------------------------------

def sq_dists(X, mu) -> np.ndarray:
    """Squared Euclidean distances ||x_i - mu_c||^2, [n, C], float64.

    Written as ||x||^2 - 2 x.mu + ||mu||^2 with a float64 matrix product; the
    same quantity up to float64 rounding."""
    X = _f64(X)
    mu = _f64(mu)
    return ((X * X).sum(1)[:, None] - 2.0 * (X @ mu.T)
            + (mu * mu).sum(1)[None, :])


def assign(X, mu) -> np.ndarray:
    """label(x) = argmin_c ||x - mu_c||^2, first index on ties."""
    X = _f64(X)
    out = np.empty(X.shape[0], dtype=np.int64)
    for s in range(0, X.shape[0], _ROW_CHUNK):
        out[s:s + _ROW_CHUNK] = np.argmin(sq_dists(X[s:s + _ROW_CHUNK], mu), axis=1)
    return out


def assign_margin(X, mu):
    """(labels, best distance, second-best distance) per point; the relative
    gap (d2 - d1) / d2 tells a genuine near-tie from a wrong label."""
    X = _f64(X)
    n, C = X.shape[0], np.asarray(mu).shape[0]
    lab = np.empty(n, dtype=np.int64)
    d1 = np.empty(n)
    d2 = np.full(n, np.inf)
    for s in range(0, n, _ROW_CHUNK):
        D = sq_dists(X[s:s + _ROW_CHUNK], mu)
        l = np.argmin(D, axis=1)
        lab[s:s + _ROW_CHUNK] = l
        d1[s:s + _ROW_CHUNK] = D[np.arange(D.shape[0]), l]
        if C > 1:
            D[np.arange(D.shape[0]), l] = np.inf
            d2[s:s + _ROW_CHUNK] = D.min(axis=1)
    return lab, d1, d2


def update(X, labels, mu_old):
    """mu_c = mean of the x with label c; an empty cluster keeps mu_old[c].
    Returns (mu [C, d] float64, counts [C])."""
    X = _f64(X)
    mu_old = _f64(mu_old)
    C = mu_old.shape[0]
    counts = np.bincount(labels, minlength=C)
    sums = np.zeros_like(mu_old)
    np.add.at(sums, labels, X)
    mu = mu_old.copy()
    nz = counts > 0
    mu[nz] = sums[nz] / counts[nz, None]
    return mu, counts


def kmeans(X, C: int, iters: int, init):
    """Lloyd's k-means: `iters` rounds of assign->update from the centroid
    values `init` [C, d], then a final assignment.  Returns
    (centroids [C, d] float64, labels [N], counts [C])."""
    mu = _f64(init).copy()
    assert mu.shape[0] == C
    for _ in range(iters):
        labels = assign(X, mu)
        mu, _ = update(X, labels, mu)
    labels = assign(X, mu)
    counts = np.bincount(labels, minlength=C)
    return mu, labels, counts


def inertia(X, mu, labels) -> float:
    X = _f64(X)
    mu = _f64(mu)
    return float(((X - mu[labels]) ** 2).sum())


# --------------------------------------------------------------------------
# (1') reorder tokens so every cluster is contiguous              [R] step (1)
# --------------------------------------------------------------------------

def permute(labels, C: int):
    """Stable counting-sort order: perm[new] = old, clusters in index order,
    original order inside a cluster.  Returns (perm, offsets [C+1], counts)."""
    labels = np.asarray(labels)
    perm = np.argsort(labels, kind="stable")
    counts = np.bincount(labels, minlength=C)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    return perm, offsets, counts


def value_centroids(V, k_labels, Ck: int) -> np.ndarray:
    """vbar_c = mean of v_j over key cluster c (0 for an empty cluster).
    [R] steps (2),(4); [AB] "keys and values ... summarized by centroids"."""
    V = _f64(V)
    counts = np.bincount(k_labels, minlength=Ck)
    sums = np.zeros((Ck, V.shape[1]), dtype=V.dtype)
    np.add.at(sums, k_labels, V)
    out = np.zeros_like(sums)
    nz = counts > 0
    out[nz] = sums[nz] / counts[nz, None]
    return out


def key_scalars(V, k_labels, Vbar) -> np.ndarray:
    """Per-key quantities a factored error kernel may precompute, in token
    order: [3, N] = (||vbar_c(j) - v_j||^2, (vbar_c(j) - v_j).v_j, ||v_j||^2)."""
    V = _f64(V)
    vb = _f64(Vbar)[k_labels]
    dv = vb - V
    return np.stack([(dv * dv).sum(1), (dv * V).sum(1), (V * V).sum(1)])


# --------------------------------------------------------------------------
# (2) value-aware block error with the query-centroid proxy
#     [R] step (2); [DE] 2.B; [IT] 2.B "Stima dell'Errore"
# --------------------------------------------------------------------------

def block_shift(Qbar, Kbar, k_counts, scale: float) -> np.ndarray:
    """M_a = max over non-empty key clusters of scale * qbar_a . kbar_c."""
    L = scale * (_f64(Qbar) @ _f64(Kbar).T)
    L[:, np.asarray(k_counts) == 0] = -np.inf
    return L.max(axis=1)


def block_error(Qbar, Kbar, Vbar, K, V, k_labels, k_counts, scale: float,
                key_chunk: int = 1024):
    """Per (query cluster a, key cluster c):

        eps^2(a, j) = || exp(s qbar_a.kbar_c) vbar_c - exp(s qbar_a.k_j) v_j ||^2
        E[a, c]     = exp(-2 M_a) * (1/|k_c|) * sum_{j in c} eps^2(a, j)

    E equals the pages' error-to-cost ratio sum_{(i,j) in block} eps^2 /
    (|q_a| |k_c|) times exp(-2 M_a): every query of cluster a uses the same
    proxy qbar_a, so the |q_a| identical rows cancel.  Empty key clusters get 0.
    Returns (E [Cq, Ck], M [Cq])."""
    Qbar, Kbar, Vbar, K, V = map(_f64, (Qbar, Kbar, Vbar, K, V))
    k_labels = np.asarray(k_labels)
    k_counts = np.asarray(k_counts)
    M = block_shift(Qbar, Kbar, k_counts, scale)
    Lbar = scale * (Qbar @ Kbar.T)
    E = np.zeros((Qbar.shape[0], Kbar.shape[0]), dtype=K.dtype)
    for s in range(0, K.shape[0], key_chunk):
        j = slice(s, s + key_chunk)
        c = k_labels[j]
        A = np.exp(Lbar[:, c] - M[:, None])                       # [Cq, n]
        B = np.exp(scale * (Qbar @ K[j].T) - M[:, None])          # [Cq, n]
        diff = A[:, :, None] * Vbar[c][None] - B[:, :, None] * V[j][None]
        eps2 = (diff * diff).sum(-1)                               # [Cq, n]
        np.add.at(E.T, c, eps2.T)
    nz = k_counts > 0
    E[:, nz] /= k_counts[nz][None, :]
    return E, M


def block_error_scale(Qbar, Kbar, Vbar, K, V, k_labels, k_counts, scale: float,
                      key_chunk: int = 1024) -> np.ndarray:
    """T[a, c] = (1/|k_c|) sum_j (A^2 ||vbar_c||^2 + B_j^2 ||v_j||^2) in the
    same shifted units as E: the size of the two terms whose difference E
    measures, used as an absolute floor when comparing E near zero."""
    Qbar, Kbar, Vbar, K, V = map(_f64, (Qbar, Kbar, Vbar, K, V))
    k_labels = np.asarray(k_labels)
    k_counts = np.asarray(k_counts)
    M = block_shift(Qbar, Kbar, k_counts, scale)
    Lbar = scale * (Qbar @ Kbar.T)
    T = np.zeros((Qbar.shape[0], Kbar.shape[0]))
    vbn = (Vbar * Vbar).sum(1)
    for s in range(0, K.shape[0], key_chunk):
        j = slice(s, s + key_chunk)
        c = k_labels[j]
        A = np.exp(Lbar[:, c] - M[:, None])
        B = np.exp(scale * (Qbar @ K[j].T) - M[:, None])
        t = A * A * vbn[c][None] + B * B * (V[j] * V[j]).sum(1)[None]
        np.add.at(T.T, c, t.T)
    nz = k_counts > 0
    T[:, nz] /= k_counts[nz][None, :]
    return T


# --------------------------------------------------------------------------
# (2') routing-signal ablations.  The pages contrast error-aware routing with
#      selectors that rank blocks by attention score ([AB]; [DE] 2.B; [IT]
#      2.B): these two swap the ranking signal and keep every other step.
# --------------------------------------------------------------------------

def block_mass(Qbar, Kbar, k_counts, scale: float):
    """Score-based signal: the attention weight the query centroid qbar_a
    gives key cluster c when every key of c is replaced by kbar_c,

        P[a, c] = |k_c| exp(s qbar_a.kbar_c) / sum_{c' non-empty} |k_c'| exp(s qbar_a.kbar_c'),

    0 for empty clusters; each row sums to 1.  Returns (P [Cq, Ck], M [Cq])
    with M as in block_error."""
    k_counts = np.asarray(k_counts)
    M = block_shift(Qbar, Kbar, k_counts, scale)
    L = scale * (_f64(Qbar) @ _f64(Kbar).T)
    nz = k_counts > 0
    P = np.zeros_like(L)
    P[:, nz] = k_counts[nz][None, :] * np.exp(L[:, nz] - M[:, None])
    P /= P.sum(axis=1, keepdims=True)
    return P, M


def block_error_value_agnostic(Qbar, Kbar, K, k_labels, k_counts, scale: float,
                               key_chunk: int = 1024):
    """The block error with the values left out:

        eps^2(a, j) = (exp(s qbar_a.kbar_c) - exp(s qbar_a.k_j))^2
        E[a, c]     = exp(-2 M_a) * (1/|k_c|) * sum_{j in c} eps^2(a, j)

    Returns (E [Cq, Ck], M [Cq]); empty key clusters get 0."""
    Qbar, Kbar, K = map(_f64, (Qbar, Kbar, K))
    k_labels = np.asarray(k_labels)
    k_counts = np.asarray(k_counts)
    M = block_shift(Qbar, Kbar, k_counts, scale)
    Lbar = scale * (Qbar @ Kbar.T)
    E = np.zeros((Qbar.shape[0], Kbar.shape[0]))
    for s in range(0, K.shape[0], key_chunk):
        j = slice(s, s + key_chunk)
        c = k_labels[j]
        A = np.exp(Lbar[:, c] - M[:, None])
        B = np.exp(scale * (Qbar @ K[j].T) - M[:, None])
        np.add.at(E.T, c, ((A - B) ** 2).T)
    nz = k_counts > 0
    E[:, nz] /= k_counts[nz][None, :]
    return E, M


ROUTERS = ("error", "mass", "error_nov")


def routing_signal(router: str, Qbar, Kbar, Vbar, K, V, k_labels, k_counts, scale: float):
    """(E, M) for the named signal: "error" (the method), "mass" or
    "error_nov" (the ablations above)."""
    if router == "error":
        return block_error(Qbar, Kbar, Vbar, K, V, k_labels, k_counts, scale)
    if router == "mass":
        return block_mass(Qbar, Kbar, k_counts, scale)
    if router == "error_nov":
        return block_error_value_agnostic(Qbar, Kbar, K, k_labels, k_counts, scale)
    raise ValueError(router)


# --------------------------------------------------------------------------
# (3) error-aware routing under the density budget rho
#     [R] step (3); [DE] 2.B "Selektion"; [IT] 2.B "Selezione Greedy"
# --------------------------------------------------------------------------

def route_budget(rho, Nk: int) -> int:
    """floor(rho * N_k), rho as the float32 the operator receives."""
    return int(math.floor(float(np.float32(rho)) * float(Nk)))


def route_order(E_row, k_counts) -> np.ndarray:
    """Non-empty key clusters by ratio descending, smaller index first on ties."""
    Ck = E_row.shape[0]
    order = np.lexsort((np.arange(Ck), -_f64(E_row)))
    return order[np.asarray(k_counts)[order] > 0]


def route(E, k_counts, q_counts, rho):
    """Greedy error-to-cost routing per query cluster: walk the ratio order and
    keep the longest prefix whose total key count fits the budget.
    Returns (mask [Cq, Ck] uint8, sel list of arrays in selection order,
    exec_pairs = sum_a |q_a| * sum_{c in S_a} |k_c|)."""
    E = _f64(E)
    k_counts = np.asarray(k_counts, dtype=np.int64)
    q_counts = np.asarray(q_counts, dtype=np.int64)
    Cq, Ck = E.shape
    budget = route_budget(rho, int(k_counts.sum()))
    mask = np.zeros((Cq, Ck), dtype=np.uint8)
    sel = []
    pairs = 0
    for a in range(Cq):
        order = route_order(E[a], k_counts)
        csum = np.cumsum(k_counts[order])
        n = int(np.searchsorted(csum, budget, side="right"))
        chosen = order[:n]
        mask[a, chosen] = 1
        sel.append(chosen)
        pairs += int(q_counts[a]) * int(k_counts[chosen].sum())
    return mask, sel, pairs


def route_global_budget(rho, Nq: int, Nk: int) -> int:
    """floor(rho * N_q * N_k) pairs, rho as the float32 the operator receives,
    in exact rational arithmetic."""
    from fractions import Fraction
    return int(math.floor(Fraction(float(np.float32(rho))) * Nq * Nk))


def route_global(E, M, k_counts, q_counts, rho):
    """Global-budget routing (the knapsack form of [DE] 2.B taken over all
    blocks of a head at once): every block (a, c) with |q_a| > 0 and
    |k_c| > 0 is an item of cost |q_a| |k_c| and value the unshifted
    error-to-cost ratio E[a, c] exp(2 M_a); items in ratio order (descending;
    equal ratios: smaller a * Ck + c first); the longest prefix whose total
    cost fits floor(rho N_q N_k) is routed.  Ratios are compared as
    log E + 2 M (E = 0 is -inf).  Returns (mask, sel per row in that row's
    order, exec_pairs) like route."""
    E = _f64(E)
    M = _f64(M)
    k_counts = np.asarray(k_counts, dtype=np.int64)
    q_counts = np.asarray(q_counts, dtype=np.int64)
    Cq, Ck = E.shape
    budget = route_global_budget(rho, int(q_counts.sum()), int(k_counts.sum()))
    with np.errstate(divide="ignore"):
        key = np.log(np.maximum(E, 0.0)) + 2.0 * M[:, None]
    valid = (q_counts[:, None] > 0) & (k_counts[None, :] > 0)
    idx = np.arange(Cq * Ck)
    order = np.lexsort((idx, -key.ravel()))
    order = order[valid.ravel()[order]]
    cost = (q_counts[:, None] * k_counts[None, :]).ravel()[order]
    n = int(np.searchsorted(np.cumsum(cost), budget, side="right"))
    mask = np.zeros((Cq, Ck), dtype=np.uint8)
    mask.ravel()[order[:n]] = 1
    sel = [order[:n][order[:n] // Ck == a] % Ck for a in range(Cq)]
    pairs = int(cost[:n].sum())
    return mask, sel, pairs


# --------------------------------------------------------------------------
# (4) hybrid attention: exact routed blocks + centroid compensation, one
#     softmax                                [R] step (4); [DE] 2.A; [IT] 2.A
# --------------------------------------------------------------------------

def hybrid_attention(Q, K, V, q_labels, k_labels, Kbar, Vbar, k_counts, mask,
                     scale: float) -> np.ndarray:
    """o_i (query i in cluster a) = softmax over
         { s q_i.k_j          : j in a routed key cluster }
       U { s q_i.kbar_c + log|k_c| : c compensated and non-empty }
    applied to the matching v_j / vbar_c.  Output in the original token order."""
    Q, K, V, Kbar, Vbar = map(_f64, (Q, K, V, Kbar, Vbar))
    q_labels = np.asarray(q_labels)
    k_labels = np.asarray(k_labels)
    k_counts = np.asarray(k_counts)
    O = np.zeros_like(Q)
    nonempty = k_counts > 0
    for a in range(mask.shape[0]):
        rows = np.nonzero(q_labels == a)[0]
        if rows.size == 0:
            continue
        routed = (mask[a] > 0) & nonempty
        comp = (mask[a] == 0) & nonempty
        keys = np.nonzero(routed[k_labels])[0]
        cc = np.nonzero(comp)[0]
        for s in range(0, rows.size, _ROW_CHUNK):
            r = rows[s:s + _ROW_CHUNK]
            L = np.concatenate([scale * (Q[r] @ K[keys].T),
                                scale * (Q[r] @ Kbar[cc].T)
                                + np.log(k_counts[cc].astype(Q.dtype))[None]],
                               axis=1)
            W = np.exp(L - L.max(axis=1, keepdims=True))
            Vals = np.concatenate([V[keys], Vbar[cc]], axis=0)
            O[r] = (W @ Vals) / W.sum(axis=1, keepdims=True)
    return O


def dense_attention(Q, K, V, scale: float) -> np.ndarray:
    """softmax(s Q K^T) V, row-chunked, float64."""
    Q, K, V = map(_f64, (Q, K, V))
    O = np.empty_like(Q)
    for s in range(0, Q.shape[0], _ROW_CHUNK):
        L = scale * (Q[s:s + _ROW_CHUNK] @ K.T)
        W = np.exp(L - L.max(axis=1, keepdims=True))
        O[s:s + _ROW_CHUNK] = (W @ V) / W.sum(axis=1, keepdims=True)
    return O


# --------------------------------------------------------------------------
# whole operator, one head
# --------------------------------------------------------------------------

def forward(Q, K, V, Cq: int, Ck: int, iters: int, rho, scale: float,
            init_q, init_k, router: str = "error",
            budget: str = "row") -> Dict[str, object]:
    """All steps of one head in order; returns every intermediate.  `router`
    names the routing signal (ROUTERS; "error" is the method); `budget` is
    "row" (floor(rho N_k) keys per query cluster, the method) or "global"
    (route_global)."""
    Qbar, lq, cq = kmeans(Q, Cq, iters, init_q)
    Kbar, lk, ck = kmeans(K, Ck, iters, init_k)
    perm_q, off_q, _ = permute(lq, Cq)
    perm_k, off_k, _ = permute(lk, Ck)
    Vbar = value_centroids(V, lk, Ck)
    E, M = routing_signal(router, Qbar, Kbar, Vbar, K, V, lk, ck, scale)
    if budget == "row":
        mask, sel, pairs = route(E, ck, cq, rho)
    elif budget == "global":
        mask, sel, pairs = route_global(E, M, ck, cq, rho)
    else:
        raise ValueError(budget)
    O = hybrid_attention(Q, K, V, lq, lk, Kbar, Vbar, ck, mask, scale)
    return dict(Qbar=Qbar, Kbar=Kbar, Vbar=Vbar, q_labels=lq, k_labels=lk,
                q_counts=cq, k_counts=ck, perm_q=perm_q, perm_k=perm_k,
                off_q=off_q, off_k=off_k, E=E, M=M, mask=mask, sel=sel,
                exec_pairs=pairs, O=O)
