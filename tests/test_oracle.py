"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a library routine, a closed form worked by hand, an invariant
the method guarantees, or brute force on a tiny input."""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import svgear_oracle as ora
from clustered_sparse_attention_flash_b200 import synth


def _blobs(rng, C, per, d, spread=10.0, sigma=0.5):
    centers = rng.standard_normal((C, d)) * spread
    X = np.concatenate([centers[c] + sigma * rng.standard_normal((per, d)) for c in range(C)])
    return X, centers


# ---------------------------------------------------------------- k-means ----

def test_kmeans_matches_sklearn_lloyd():
    """Lloyd with a given init, fixed iteration count and a final E-step is
    what scikit-learn's KMeans(algorithm='lloyd', n_init=1, tol=0) computes
    (no empty clusters here, where scikit-learn relocates instead)."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(0)
    X, _ = _blobs(rng, 6, 40, 5, spread=3.0, sigma=1.0)
    X = X[rng.permutation(len(X))]
    for iters in (1, 3, 8):
        init = X[rng.choice(len(X), 6, replace=False)]
        km = KMeans(n_clusters=6, init=init, n_init=1, max_iter=iters, tol=0.0,
                    algorithm="lloyd").fit(X)
        mu, lab, cnt = ora.kmeans(X, 6, iters, init)
        assert (cnt > 0).all()
        np.testing.assert_array_equal(lab, km.labels_)
        np.testing.assert_allclose(mu, km.cluster_centers_, rtol=1e-10, atol=1e-10)


def _lloyd_loops(X, init, iters):
    """Triple-loop Lloyd, written independently for tiny inputs."""
    mu = [list(map(float, r)) for r in init]
    N, d, C = len(X), len(X[0]), len(mu)

    def lab_of(x):
        best, bc = None, -1
        for c in range(C):
            s = sum((x[t] - mu[c][t]) ** 2 for t in range(d))
            if best is None or s < best:
                best, bc = s, c
        return bc

    for _ in range(iters):
        labs = [lab_of(X[i]) for i in range(N)]
        for c in range(C):
            mem = [i for i in range(N) if labs[i] == c]
            if mem:
                mu[c] = [sum(X[i][t] for i in mem) / len(mem) for t in range(d)]
    labs = [lab_of(X[i]) for i in range(N)]
    return np.array(mu), np.array(labs)


def test_kmeans_bruteforce_with_empty_cluster():
    rng = np.random.default_rng(1)
    X, _ = _blobs(rng, 3, 12, 4, spread=4.0)
    init = np.concatenate([X[[0, 13, 30]], np.full((1, 4), 1e3)])  # 4th stays empty
    mu_b, lab_b = _lloyd_loops(X.tolist(), init, 5)
    mu, lab, cnt = ora.kmeans(X, 4, 5, init)
    np.testing.assert_array_equal(lab, lab_b)
    np.testing.assert_allclose(mu, mu_b, rtol=1e-12, atol=1e-12)
    assert cnt[3] == 0 and np.array_equal(mu[3], init[3])


def test_kmeans_inertia_nonincreasing_and_fixed_point():
    cfg = synth.CONFIGS["tiny"]
    q, k, v, _ = synth.make_head(cfg, 0)
    init = synth.forgy_init(cfg, k, 0, 1, cfg.Ck)
    prev = math.inf
    for it in range(0, 8):
        mu, lab, _ = ora.kmeans(k, cfg.Ck, it, init)
        # inertia measured with the centroids the labels were assigned against
        val = ora.inertia(k, mu, lab)
        assert val <= prev * (1 + 1e-12)
        prev = val
    # a fixed point reproduces itself
    mu, lab, _ = ora.kmeans(k, cfg.Ck, 40, init)
    mu2, lab2, _ = ora.kmeans(k, cfg.Ck, 3, mu)
    np.testing.assert_array_equal(lab, lab2)
    np.testing.assert_allclose(mu, mu2, rtol=1e-12, atol=1e-12)


def test_assign_margin_consistent():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((300, 6))
    mu = rng.standard_normal((7, 6))
    lab, d1, d2 = ora.assign_margin(X, mu)
    D = ((X[:, None, :] - mu[None]) ** 2).sum(-1)
    np.testing.assert_array_equal(lab, D.argmin(1))
    np.testing.assert_allclose(d1, D.min(1), rtol=1e-12)
    np.testing.assert_allclose(d2, np.sort(D, 1)[:, 1], rtol=1e-12)


# ------------------------------------------------------------- permutation ----

def test_permute_is_stable_counting_sort():
    rng = np.random.default_rng(3)
    labels = rng.integers(0, 9, size=500)
    labels[labels == 4] = 5          # cluster 4 empty
    perm, off, cnt = ora.permute(labels, 9)
    assert sorted(perm.tolist()) == list(range(500))
    lp = labels[perm]
    assert (np.diff(lp) >= 0).all()
    for c in range(9):
        seg = perm[off[c]:off[c + 1]]
        assert (labels[seg] == c).all() and (np.diff(seg) > 0).all()
    assert cnt[4] == 0 and off[-1] == 500


def test_value_centroid_of_singleton_is_the_value():
    rng = np.random.default_rng(4)
    V = rng.standard_normal((20, 3))
    lab = rng.permutation(20)
    np.testing.assert_array_equal(ora.value_centroids(V, lab, 20)[lab], V)


# ------------------------------------------------------------- block error ----

def test_key_scalars_two_key_worked_example():
    """Values (1, 0) and (3, 2) in one cluster: vbar = (2, 1).  Key 0:
    vbar - v = (1, 1), so (2, 1, 1); key 1: vbar - v = (-1, -1), so
    (2, -5, 13).  Worked by hand."""
    V = np.array([[1.0, 0.0], [3.0, 2.0]])
    lab = np.array([0, 0])
    Vbar = np.array([[2.0, 1.0]])
    np.testing.assert_array_equal(ora.key_scalars(V, lab, Vbar),
                                  [[2.0, 2.0], [1.0, -5.0], [1.0, 13.0]])


def test_key_scalars_reproduce_the_literal_error_norm():
    """The block error's per-key term ||A vbar - B v||^2 equals
    A^2 (s1 + 2 w s2 + w^2 s3) with w = (A - B) / A, because
    A vbar - B v = A ((vbar - v) + w v).  Checked against the literal norm on
    random values, weights and clusters; and the cross term summed over a
    cluster is minus the summed squared deviation (sum_j (vbar - v_j).v_j =
    n ||vbar||^2 - sum_j ||v_j||^2)."""
    rng = np.random.default_rng(41)
    V = rng.standard_normal((50, 6))
    lab = rng.integers(0, 5, size=50)
    Vbar = ora.value_centroids(V, lab, 5)
    s1, s2, s3 = ora.key_scalars(V, lab, Vbar)
    A = np.exp(rng.standard_normal(50))
    B = np.exp(rng.standard_normal(50))
    w = (A - B) / A
    lit = ((A[:, None] * Vbar[lab] - B[:, None] * V) ** 2).sum(1)
    np.testing.assert_allclose(A * A * (s1 + 2 * w * s2 + w * w * s3), lit, rtol=1e-12)
    for c in range(5):
        m = lab == c
        assert s2[m].sum() == pytest.approx(-s1[m].sum(), rel=1e-12, abs=1e-12)
        assert s1[m].sum() == pytest.approx(m.sum() * np.var(V[m], axis=0).sum(), rel=1e-12)


def test_block_error_scale_worked_example():
    """d = 1, qbar = 1, scale 1, keys {0, ln 2} (kbar = ln2 / 2), values
    (1, 0) and (0, 2) with vbar = (1/2, 1): M = ln2 / 2, A = 1,
    B = {2^-1/2, 2^1/2}, ||vbar||^2 = 5/4, ||v||^2 = {1, 4}, so
    T = (1/2) ((5/4 + 1/2) + (5/4 + 8)) = 11/2.  Worked by hand."""
    ln2 = math.log(2.0)
    K = np.array([[0.0], [ln2]])
    V = np.array([[1.0, 0.0], [0.0, 2.0]])
    T = ora.block_error_scale(np.array([[1.0]]), np.array([[ln2 / 2]]), np.array([[0.5, 1.0]]),
                              K, V, np.array([0, 0]), np.array([2]), 1.0)
    assert T[0, 0] == pytest.approx(5.5, rel=1e-13)


def test_block_error_scale_bounds_the_error():
    """||a - b||^2 <= 2 (||a||^2 + ||b||^2) term by term, so E <= 2 T; with
    values of zero mean in every cluster (vbar = 0) the cross term vanishes
    and E = T exactly."""
    rng = np.random.default_rng(42)
    Qb = rng.standard_normal((3, 4))
    K = rng.standard_normal((40, 4))
    V = rng.standard_normal((40, 5))
    lab = rng.integers(0, 6, size=40)
    cnt = np.bincount(lab, minlength=6)
    Kb = ora.value_centroids(K, lab, 6)
    Vb = ora.value_centroids(V, lab, 6)
    E, _ = ora.block_error(Qb, Kb, Vb, K, V, lab, cnt, 0.6)
    T = ora.block_error_scale(Qb, Kb, Vb, K, V, lab, cnt, 0.6)
    assert (E <= 2 * T * (1 + 1e-12)).all()
    V0 = V - Vb[lab]  # zero mean per cluster
    E0, _ = ora.block_error(Qb, Kb, np.zeros_like(Vb), K, V0, lab, cnt, 0.6)
    T0 = ora.block_error_scale(Qb, Kb, np.zeros_like(Vb), K, V0, lab, cnt, 0.6)
    np.testing.assert_allclose(E0, T0, rtol=1e-12, atol=1e-300)


def test_block_error_zero_query_centroid_is_value_variance():
    """qbar = 0 makes every logit 0: A = B = 1, so E[a, c] is the
    within-cluster (population) variance of V, summed over dims."""
    rng = np.random.default_rng(5)
    K = rng.standard_normal((60, 4))
    V = rng.standard_normal((60, 4))
    lab = rng.integers(0, 5, size=60)
    cnt = np.bincount(lab, minlength=5)
    Kbar = ora.value_centroids(K, lab, 5)
    Vbar = ora.value_centroids(V, lab, 5)
    E, M = ora.block_error(np.zeros((2, 4)), Kbar, Vbar, K, V, lab, cnt, 0.5)
    for c in range(5):
        want = np.var(V[lab == c], axis=0).sum() if cnt[c] else 0.0
        np.testing.assert_allclose(E[:, c], want, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(M, 0.0)


def test_block_error_two_key_closed_form():
    """d = 1, qbar = 1, scale 1, keys {0, 2} (kbar = 1), values {3, 3}:
    M = 1, A = 1, B = {e^-1, e}, so E = (9/2) ((1 - e^-1)^2 + (e - 1)^2)."""
    K = np.array([[0.0], [2.0]])
    V = np.array([[3.0], [3.0]])
    lab = np.array([0, 0])
    E, M = ora.block_error(np.array([[1.0]]), np.array([[1.0]]), np.array([[3.0]]),
                           K, V, lab, np.array([2]), 1.0)
    e = math.e
    assert M[0] == pytest.approx(1.0)
    assert E[0, 0] == pytest.approx(4.5 * ((1 - 1 / e) ** 2 + (e - 1) ** 2), rel=1e-13)


def test_block_error_singletons_and_zero_variance_are_zero():
    rng = np.random.default_rng(6)
    Qb = rng.standard_normal((3, 5))
    # singleton clusters: kbar = k, vbar = v
    K = rng.standard_normal((8, 5)); V = rng.standard_normal((8, 5))
    lab = np.arange(8)
    E, _ = ora.block_error(Qb, K, V, K, V, lab, np.ones(8, int), 0.4)
    T = ora.block_error_scale(Qb, K, V, K, V, lab, np.ones(8, int), 0.4)
    assert (np.abs(E) <= 1e-13 * T).all()
    # zero-variance clusters: identical keys and values inside each cluster
    base_k = rng.standard_normal((3, 5)); base_v = rng.standard_normal((3, 5))
    lab = np.repeat(np.arange(3), 4)
    K = base_k[lab]; V = base_v[lab]
    E, _ = ora.block_error(Qb, base_k, base_v, K, V, lab, np.full(3, 4), 0.4)
    T = ora.block_error_scale(Qb, base_k, base_v, K, V, lab, np.full(3, 4), 0.4)
    assert (np.abs(E) <= 1e-13 * T).all() and (T > 0).all()


def test_block_error_equals_pairwise_ratio_bruteforce():
    """The pages define the routing ratio over all (query, key) pairs of a
    block divided by |q_a||k_c|; with the centroid proxy every query of
    cluster a contributes the same error, which the factored O(C_q N_k d)
    form relies on.  Brute force over every pair, tiny sizes."""
    rng = np.random.default_rng(7)
    Nq, Nk, d, Cq, Ck, s = 30, 26, 3, 3, 4, 0.7
    Q = rng.standard_normal((Nq, d)); K = rng.standard_normal((Nk, d))
    V = rng.standard_normal((Nk, d))
    lq = rng.integers(0, Cq, Nq); lk = rng.integers(0, Ck, Nk)
    cq = np.bincount(lq, minlength=Cq); ck = np.bincount(lk, minlength=Ck)
    Qb = ora.value_centroids(Q, lq, Cq); Kb = ora.value_centroids(K, lk, Ck)
    Vb = ora.value_centroids(V, lk, Ck)
    E, M = ora.block_error(Qb, Kb, Vb, K, V, lk, ck, s)
    for a in range(Cq):
        for c in range(Ck):
            tot = 0.0
            for i in range(Nq):
                if lq[i] != a:
                    continue
                for j in range(Nk):
                    if lk[j] != c:
                        continue
                    qa = Qb[lq[i]]
                    A = math.exp(s * float(qa @ Kb[c]))
                    B = math.exp(s * float(qa @ K[j]))
                    tot += float(((A * Vb[c] - B * V[j]) ** 2).sum())
            want = tot / (cq[a] * ck[c]) * math.exp(-2 * M[a]) if cq[a] and ck[c] else 0.0
            assert E[a, c] == pytest.approx(want, rel=1e-11, abs=1e-300)


# ------------------------------------------------------ routing ablations ----

def test_block_mass_is_the_compensated_attention_weight():
    """With every block compensated, hybrid attention of the query centroid
    gives cluster c the weight |k_c| e^{s qbar.kbar_c} / sum; reading those
    weights out through one-hot value centroids must give block_mass."""
    rng = np.random.default_rng(21)
    Nk, d, Cq, Ck, s = 50, 6, 3, 6, 0.8       # d = Ck: the one-hot values fit the output rows
    K = rng.standard_normal((Nk, d))
    lk = rng.integers(0, Ck - 1, Nk)            # cluster Ck-1 stays empty
    ck = np.bincount(lk, minlength=Ck)
    Kb = ora.value_centroids(K, lk, Ck)
    Qb = rng.standard_normal((Cq, d))
    P, M = ora.block_mass(Qb, Kb, ck, s)
    O = ora.hybrid_attention(Qb, K, np.zeros((Nk, Ck)), np.arange(Cq), lk, Kb, np.eye(Ck), ck,
                             np.zeros((Cq, Ck), np.uint8), s)
    np.testing.assert_allclose(P, O, rtol=1e-12, atol=1e-15)
    assert (P[:, -1] == 0).all()
    np.testing.assert_allclose(P.sum(1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(M, ora.block_shift(Qb, Kb, ck, s))


def test_block_mass_equal_logits_is_cluster_share():
    """qbar = 0: every logit is 0, so the mass of c is |k_c| / N_k."""
    ck = np.array([3, 0, 5, 2])
    P, _ = ora.block_mass(np.zeros((2, 3)), np.ones((4, 3)), ck, 0.7)
    np.testing.assert_allclose(P, np.broadcast_to(ck / ck.sum(), P.shape), rtol=1e-15)


def test_value_agnostic_error_is_value_aware_with_constant_values():
    """v_j = vbar_c = u with |u| = 1 turns eps^2 into (A - B_j)^2."""
    rng = np.random.default_rng(22)
    Nk, d, Cq, Ck, s = 40, 5, 4, 5, 0.6
    K = rng.standard_normal((Nk, d))
    lk = rng.integers(0, Ck, Nk)
    ck = np.bincount(lk, minlength=Ck)
    Kb = ora.value_centroids(K, lk, Ck)
    Qb = rng.standard_normal((Cq, d))
    u = rng.standard_normal(d); u /= np.linalg.norm(u)
    Ev, Mv = ora.block_error(Qb, Kb, np.tile(u, (Ck, 1)), K, np.tile(u, (Nk, 1)), lk, ck, s)
    En, Mn = ora.block_error_value_agnostic(Qb, Kb, K, lk, ck, s)
    np.testing.assert_allclose(En, Ev, rtol=1e-12, atol=1e-300)
    np.testing.assert_array_equal(Mn, Mv)


def test_value_agnostic_two_key_closed_form():
    """The two-key case of the value-aware pin without its values:
    E = (1/2) ((1 - e^-1)^2 + (e - 1)^2)."""
    E, M = ora.block_error_value_agnostic(np.array([[1.0]]), np.array([[1.0]]),
                                          np.array([[0.0], [2.0]]), np.array([0, 0]), np.array([2]), 1.0)
    e = math.e
    assert M[0] == pytest.approx(1.0)
    assert E[0, 0] == pytest.approx(0.5 * ((1 - 1 / e) ** 2 + (e - 1) ** 2), rel=1e-13)


def test_routing_signal_dispatch():
    rng = np.random.default_rng(23)
    K = rng.standard_normal((30, 3)); V = rng.standard_normal((30, 3))
    lk = rng.integers(0, 4, 30); ck = np.bincount(lk, minlength=4)
    Kb = ora.value_centroids(K, lk, 4); Vb = ora.value_centroids(V, lk, 4)
    Qb = rng.standard_normal((2, 3))
    args = (Qb, Kb, Vb, K, V, lk, ck, 0.5)
    np.testing.assert_array_equal(ora.routing_signal("error", *args)[0], ora.block_error(*args)[0])
    np.testing.assert_array_equal(ora.routing_signal("mass", *args)[0], ora.block_mass(Qb, Kb, ck, 0.5)[0])
    np.testing.assert_array_equal(ora.routing_signal("error_nov", *args)[0],
                                  ora.block_error_value_agnostic(Qb, Kb, K, lk, ck, 0.5)[0])
    with pytest.raises(ValueError):
        ora.routing_signal("score", *args)


# ----------------------------------------------------------------- routing ----

def test_route_extremes_and_budget():
    rng = np.random.default_rng(8)
    Cq, Ck = 5, 40
    E = rng.random((Cq, Ck))
    kc = rng.integers(0, 30, Ck); kc[3] = 0
    qc = rng.integers(1, 10, Cq)
    m1, _, p1 = ora.route(E, kc, qc, 1.0)
    assert (m1 == (kc > 0)[None]).all()
    assert p1 == int(qc.sum()) * int(kc.sum())
    m0, _, p0 = ora.route(E, kc, qc, 0.0)
    assert m0.sum() == 0 and p0 == 0
    for rho in (0.05, 0.1, 0.3, 0.77):
        m, sel, _ = ora.route(E, kc, qc, rho)
        budget = math.floor(float(np.float32(rho)) * kc.sum())
        for a in range(Cq):
            assert (kc * m[a]).sum() <= budget
            order = [c for c in sorted(range(Ck), key=lambda c: (-E[a, c], c)) if kc[c] > 0]
            n = len(sel[a])
            assert list(sel[a]) == order[:n]            # a prefix of the order
            if n < len(order):                          # the next one does not fit
                assert (kc * m[a]).sum() + kc[order[n]] > budget


def test_route_tie_break_and_float32_rho():
    E = np.array([[1.0, 2.0, 2.0, 1.0]])
    kc = np.array([1, 1, 1, 1])
    m, sel, _ = ora.route(E, kc, np.array([1]), 0.5)
    assert list(sel[0]) == [1, 2]
    m, sel, _ = ora.route(E, kc, np.array([1]), 0.75)
    assert list(sel[0]) == [1, 2, 0]
    # rho enters as float32: 0.15f * 75600 = 11340.0004... -> 11340
    assert ora.route_budget(0.15, 75600) == 11340


def test_route_knapsack_gap_reported():
    """Exhaustive subsets on a tiny case: the greedy prefix is feasible and
    never better than the 0-1 knapsack optimum (the pages call greedy an
    approximation of the knapsack problem); the gap is only reported."""
    rng = np.random.default_rng(9)
    gaps = []
    for _ in range(20):
        Ck = 10
        kc = rng.integers(1, 8, Ck); E = rng.random((1, Ck))
        rho = 0.4
        m, _, _ = ora.route(E, kc, np.array([1]), rho)
        budget = ora.route_budget(rho, int(kc.sum()))
        best = 0.0
        for bits in itertools.product((0, 1), repeat=Ck):
            b = np.array(bits)
            if (b * kc).sum() <= budget:
                best = max(best, float((b * kc * E[0]).sum()))
        got = float((m[0] * kc * E[0]).sum())
        assert got <= best + 1e-12 and (m[0] * kc).sum() <= budget
        gaps.append(1 - got / best)
    print("greedy/knapsack mean gap", float(np.mean(gaps)))


# -------------------------------------------------------- hybrid attention ----

def _sdpa64(Q, K, V, scale, bias=None):
    q = torch.from_numpy(np.ascontiguousarray(Q, dtype=np.float64))[None, None]
    k = torch.from_numpy(np.ascontiguousarray(K, dtype=np.float64))[None, None]
    v = torch.from_numpy(np.ascontiguousarray(V, dtype=np.float64))[None, None]
    m = None if bias is None else torch.from_numpy(np.broadcast_to(bias, (Q.shape[0], K.shape[0])).copy())[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)[0, 0].numpy()


def _small_case(seed, N=200, d=8, Cq=5, Ck=9):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((N, d)); K = rng.standard_normal((N, d)); V = rng.standard_normal((N, d))
    return Q, K, V, Cq, Ck


def test_hybrid_rho_one_is_dense_sdpa():
    Q, K, V, Cq, Ck = _small_case(10)
    s = 1 / math.sqrt(8)
    out = ora.forward(Q, K, V, Cq, Ck, 3, 1.0, s, Q[:Cq], K[:Ck])
    np.testing.assert_allclose(out["O"], _sdpa64(Q, K, V, s), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(ora.dense_attention(Q, K, V, s), _sdpa64(Q, K, V, s), rtol=1e-10, atol=1e-12)


def test_hybrid_singletons_exact_for_any_mask():
    Q, K, V, Cq, _ = _small_case(11, N=60)
    s = 0.3
    lk = np.arange(60)
    lq = np.random.default_rng(0).integers(0, Cq, 60)
    mask = (np.random.default_rng(1).random((Cq, 60)) < 0.3).astype(np.uint8)
    O = ora.hybrid_attention(Q, K, V, lq, lk, K, V, np.ones(60, int), mask, s)
    np.testing.assert_allclose(O, _sdpa64(Q, K, V, s), rtol=1e-10, atol=1e-12)


def test_hybrid_single_key_cluster_rho_zero_is_value_mean():
    Q, K, V, Cq, _ = _small_case(12)
    out = ora.forward(Q, K, V, Cq, 1, 2, 0.0, 0.5, Q[:Cq], K[:1])
    np.testing.assert_allclose(out["O"], np.broadcast_to(V.mean(0), V.shape), rtol=1e-12, atol=1e-12)


def test_hybrid_rho_zero_is_biased_centroid_attention():
    """rho = 0: pure compensation, softmax(s Q Kbar^T + log|k_c|) Vbar over the
    non-empty clusters -- SDPA over centroids with an additive bias."""
    Q, K, V, Cq, Ck = _small_case(13)
    s = 0.4
    out = ora.forward(Q, K, V, Cq, Ck, 4, 0.0, s, Q[:Cq], K[:Ck])
    nz = out["k_counts"] > 0
    want = _sdpa64(Q, out["Kbar"][nz], out["Vbar"][nz], s,
                   bias=np.log(out["k_counts"][nz].astype(float))[None, :])
    np.testing.assert_allclose(out["O"], want, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------- global budget ----

def test_route_global_worked_example():
    """Two query clusters (sizes 2, 1), three key clusters (sizes 1, 2, 3):
    18 pairs, rho = 10/18 gives a budget of 10.  With M = (0, ln 2) the
    unshifted ratios are row 0: .5 .2 .1 and row 1 (x4): .04 .6 .16, so the
    order is (1,1) .6 cost 2, (0,0) .5 cost 2, (0,1) .2 cost 4, (1,2) .16
    cost 3, (0,2) .1 cost 6, (1,0) .04 cost 1; running costs 2 4 8 11 ...
    The first three fit; (1,0) would fit the 2 left over but lies after the
    first item that does not, so the prefix stops there."""
    E = np.array([[0.5, 0.2, 0.1], [0.01, 0.15, 0.04]])
    M = np.array([0.0, math.log(2.0)])
    kc, qc = np.array([1, 2, 3]), np.array([2, 1])
    rho = np.float32(10 / 18)
    assert ora.route_global_budget(rho, 3, 6) == 10
    mask, sel, pairs = ora.route_global(E, M, kc, qc, rho)
    np.testing.assert_array_equal(mask, [[1, 1, 0], [0, 1, 0]])
    assert [list(x) for x in sel] == [[0, 1], [1]]
    assert pairs == 8
    # the shift enters with the sign that undoes exp(-2 M): flipping it
    # reorders row 1 below row 0 and must change the routing
    m2, _, _ = ora.route_global(E, -M, kc, qc, rho)
    assert not np.array_equal(m2, mask)


def test_route_global_equal_ratios_go_to_the_smaller_block_index():
    """Four blocks of one pair each with the same ratio and a budget of two
    pairs: the blocks (0,0) and (0,1), first in a*Ck + c order, are routed."""
    E = np.full((2, 2), 0.5)
    mask, sel, pairs = ora.route_global(E, np.zeros(2), np.array([1, 1]), np.array([1, 1]), 0.5)
    np.testing.assert_array_equal(mask, [[1, 1], [0, 0]])
    assert pairs == 2 and [list(x) for x in sel] == [[0, 1], []]


def test_route_global_budget_is_exact():
    """float32(0.1) = 0.100000001490116119384765625; times 75,600^2 =
    5,715,360,000 gives 571,536,008.5166..., floor 571,536,008."""
    assert ora.route_global_budget(0.1, 75600, 75600) == 571536008
    assert ora.route_global_budget(1.0, 75600, 75600) == 75600 * 75600
    assert ora.route_global_budget(0.0, 10, 10) == 0


def test_route_global_depends_on_unshifted_ratio_only():
    """Moving exp(2 M_a) into E (and M to 0) leaves the routing unchanged."""
    rng = np.random.default_rng(31)
    Cq, Ck = 7, 11
    E = rng.random((Cq, Ck)) * np.exp(rng.normal(size=(Cq, Ck)))
    M = rng.normal(size=Cq)
    kc = rng.integers(0, 9, Ck); kc[0] = 3
    qc = rng.integers(0, 9, Cq); qc[0] = 2
    for rho in (0.05, 0.3, 0.7):
        a = ora.route_global(E, M, kc, qc, rho)
        b = ora.route_global(E * np.exp(2 * M)[:, None], np.zeros(Cq), kc, qc, rho)
        np.testing.assert_array_equal(a[0], b[0])
        assert a[2] == b[2] <= ora.route_global_budget(rho, qc.sum(), kc.sum())


def test_route_global_one_query_cluster_is_row_routing():
    """With a single query cluster the pair budget floor(rho N_q N_k) over
    costs N_q |k_c| is the key budget floor(rho N_k), and the global order is
    the row's order: the two routings coincide."""
    rng = np.random.default_rng(33)
    for trial in range(20):
        Ck = int(rng.integers(1, 40))
        E = rng.random((1, Ck)) ** 2
        kc = rng.integers(0, 7, Ck); kc[rng.integers(Ck)] += 1
        qc = np.array([int(rng.integers(1, 50))])
        rho = float(rng.random())
        mg, sg, pg = ora.route_global(E, rng.normal(size=1), kc, qc, rho)
        mr, sr, pr = ora.route(E, kc, qc, rho)
        np.testing.assert_array_equal(mg, mr)
        assert list(sg[0]) == list(sr[0]) and pg == pr


def test_route_global_extremes():
    rng = np.random.default_rng(32)
    E = rng.random((4, 6)); M = rng.normal(size=4)
    kc = np.array([3, 0, 2, 5, 1, 4]); qc = np.array([2, 0, 7, 1])
    mask, _, pairs = ora.route_global(E, M, kc, qc, 1.0)
    np.testing.assert_array_equal(mask, (qc[:, None] > 0) & (kc[None, :] > 0))
    assert pairs == qc.sum() * kc.sum()
    mask, sel, pairs = ora.route_global(E, M, kc, qc, 0.0)
    assert mask.sum() == 0 and pairs == 0 and all(len(x) == 0 for x in sel)


@pytest.mark.parametrize("router", ["mass", "error_nov"])
def test_ablation_routers_rho_one_is_dense(router):
    """Whatever the ranking signal, rho = 1 routes every non-empty cluster."""
    Q, K, V, Cq, Ck = _small_case(15)
    s = 1 / math.sqrt(8)
    out = ora.forward(Q, K, V, Cq, Ck, 3, 1.0, s, Q[:Cq], K[:Ck], router=router)
    np.testing.assert_allclose(out["O"], _sdpa64(Q, K, V, s), rtol=1e-10, atol=1e-12)


def test_global_budget_forward_rho_one_is_dense():
    Q, K, V, Cq, Ck = _small_case(16)
    s = 1 / math.sqrt(8)
    out = ora.forward(Q, K, V, Cq, Ck, 3, 1.0, s, Q[:Cq], K[:Ck], budget="global")
    np.testing.assert_allclose(out["O"], _sdpa64(Q, K, V, s), rtol=1e-10, atol=1e-12)


def test_forward_invariant_to_token_permutation():
    Q, K, V, Cq, Ck = _small_case(14)
    s = 0.35
    iq, ik = Q[:Cq].copy(), K[3:3 + Ck].copy()
    a = ora.forward(Q, K, V, Cq, Ck, 5, 0.3, s, iq, ik)
    p = np.random.default_rng(5).permutation(Q.shape[0])
    b = ora.forward(Q[p], K[p], V[p], Cq, Ck, 5, 0.3, s, iq, ik)
    np.testing.assert_allclose(b["O"], a["O"][p], rtol=1e-10, atol=1e-12)
    np.testing.assert_array_equal(b["mask"], a["mask"])
    np.testing.assert_allclose(b["E"], a["E"], rtol=1e-10, atol=1e-300)


def test_tiny_config_forward_is_close_to_dense():
    cfg = synth.CONFIGS["tiny"]
    q, k, v, _ = synth.make_head(cfg, 0)
    s = 1 / math.sqrt(cfg.d)
    out = ora.forward(q, k, v, cfg.Cq, cfg.Ck, cfg.iters, cfg.rho, s,
                      synth.forgy_init(cfg, q, 0, 0, cfg.Cq), synth.forgy_init(cfg, k, 0, 1, cfg.Ck))
    dense = ora.dense_attention(q, k, v, s)
    rel = np.linalg.norm(out["O"] - dense) / np.linalg.norm(dense)
    budget = ora.route_budget(cfg.rho, cfg.N)
    assert all((out["k_counts"] * out["mask"][a]).sum() <= budget for a in range(cfg.Cq))
    assert rel < 0.2, rel
