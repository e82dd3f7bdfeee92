"""Property tests of the CPU oracle on random small inputs (hypothesis): the
invariants the method guarantees whatever the data -- budgets are met and
the routed set is the maximal prefix of its order, outputs are convex
combinations of the values they mix, error estimates are non-negative, mass
rows sum to one, labels are the nearest centroid."""
import math

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import svgear_oracle as ora

SETTINGS = settings(max_examples=60, deadline=None)


def _case(seed, Cq, Ck):
    rng = np.random.default_rng(seed)
    E = rng.random((Cq, Ck)) * np.exp(rng.normal(size=(Cq, Ck)))
    M = rng.normal(size=Cq)
    kc = rng.integers(0, 6, Ck)
    kc[rng.integers(Ck)] += 1
    qc = rng.integers(0, 6, Cq)
    qc[rng.integers(Cq)] += 1
    return E, M, kc, qc


@SETTINGS
@given(seed=st.integers(0, 2**31), Cq=st.integers(1, 6), Ck=st.integers(1, 12), rho=st.floats(0.0, 1.0))
def test_route_meets_budget_and_is_maximal_prefix(seed, Cq, Ck, rho):
    E, _, kc, qc = _case(seed, Cq, Ck)
    mask, sel, pairs = ora.route(E, kc, qc, rho)
    budget = ora.route_budget(rho, int(kc.sum()))
    assert pairs == sum(int(qc[a]) * int(kc[sel[a]].sum()) for a in range(Cq))
    for a in range(Cq):
        order = ora.route_order(E[a], kc)
        n = len(sel[a])
        assert list(sel[a]) == list(order[:n])             # a prefix of the ratio order
        assert kc[order[:n]].sum() <= budget                 # within the budget
        if n < order.size:                                   # the next one does not fit
            assert kc[order[:n + 1]].sum() > budget
        assert (mask[a, kc == 0] == 0).all()


@SETTINGS
@given(seed=st.integers(0, 2**31), Cq=st.integers(1, 6), Ck=st.integers(1, 12), rho=st.floats(0.0, 1.0))
def test_route_global_meets_budget_and_is_maximal_prefix(seed, Cq, Ck, rho):
    E, M, kc, qc = _case(seed, Cq, Ck)
    mask, sel, pairs = ora.route_global(E, M, kc, qc, rho)
    budget = ora.route_global_budget(rho, int(qc.sum()), int(kc.sum()))
    cost = qc[:, None] * kc[None, :]
    assert pairs == int((cost * mask).sum()) <= budget
    # every routed block ranks above every block left out that would have fit
    # next: the first valid block outside the routed set does not fit
    key = np.log(E) + 2 * M[:, None]
    valid = cost > 0
    out = valid & (mask == 0)
    if out.any():
        idx = np.arange(Cq * Ck).reshape(Cq, Ck)
        cand = np.lexsort((idx[out], -key[out]))
        first = np.argwhere(out)[cand[0]]
        assert pairs + cost[first[0], first[1]] > budget
        assert key[mask > 0].min(initial=np.inf) >= key[first[0], first[1]]
    assert (mask[~valid] == 0).all()


@SETTINGS
@given(seed=st.integers(0, 2**31), N=st.integers(2, 40), Ck=st.integers(1, 8), rho=st.floats(0.0, 1.0))
def test_hybrid_output_is_a_convex_combination(seed, N, Ck, rho):
    rng = np.random.default_rng(seed)
    d = 3
    Q, K, V = (rng.normal(size=(N, d)) for _ in range(3))
    lk = rng.integers(0, Ck, N)
    kc = np.bincount(lk, minlength=Ck)
    Kb, Vb = ora.value_centroids(K, lk, Ck), ora.value_centroids(V, lk, Ck)
    lq = rng.integers(0, 2, N)
    mask = (rng.random((2, Ck)) < rho).astype(np.uint8)
    O = ora.hybrid_attention(Q, K, V, lq, lk, Kb, Vb, kc, mask, 0.7)
    vals = np.concatenate([V, Vb[kc > 0]])
    lo, hi = vals.min(0), vals.max(0)
    assert (O >= lo - 1e-12).all() and (O <= hi + 1e-12).all()


@SETTINGS
@given(seed=st.integers(0, 2**31), N=st.integers(1, 30), Ck=st.integers(1, 6))
def test_error_signals_non_negative_and_mass_normalised(seed, N, Ck):
    rng = np.random.default_rng(seed)
    d = 3
    K, V = rng.normal(size=(N, d)), rng.normal(size=(N, d))
    lk = rng.integers(0, Ck, N)
    kc = np.bincount(lk, minlength=Ck)
    Kb, Vb = ora.value_centroids(K, lk, Ck), ora.value_centroids(V, lk, Ck)
    Qb = rng.normal(size=(3, d))
    for router in ora.ROUTERS:
        E, M = ora.routing_signal(router, Qb, Kb, Vb, K, V, lk, kc, 0.6)
        assert (E >= 0).all() and (E[:, kc == 0] == 0).all()
        assert np.isfinite(M).all()
        if router == "mass":
            np.testing.assert_allclose(E.sum(1), 1.0, rtol=1e-12)


@SETTINGS
@given(seed=st.integers(0, 2**31), N=st.integers(1, 60), C=st.integers(1, 8), iters=st.integers(0, 4))
def test_kmeans_labels_are_the_nearest_centroid(seed, N, C, iters):
    C = min(C, N)
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(N, 4))
    init = X[rng.choice(N, C, replace=False)]
    mu, lab, cnt = ora.kmeans(X, C, iters, init)
    D2 = ((X[:, None, :] - mu[None]) ** 2).sum(-1)
    assert (D2[np.arange(N), lab] <= D2.min(1) + 1e-12).all()
    np.testing.assert_array_equal(cnt, np.bincount(lab, minlength=C))
    assert cnt.sum() == N
