"""Shared helpers for the GPU parity tests: seeded cases, device transfer and
the comparison rules (tolerances are those the operator's spec states)."""
from __future__ import annotations

import functools
import math

import numpy as np

from clustered_sparse_attention_flash_b200 import svgear as sv
from clustered_sparse_attention_flash_b200 import synth
from oracle import svgear_oracle as ora

# output tolerance |gpu - ref| <= ATOL + RTOL * |ref|
OUT_TOL = {"f32": (1e-4, 1e-4), "bf16": (1e-2, 1e-2)}
E_RTOL, E_FLOOR = 1e-3, 1e-6       # block error: 1e-3 relative, floor 1e-6 * T
TIE_REL = 1e-4                     # near-tie exemption for labels / routing


def torch_dtype(cfg):
    import torch
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def dev(x, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    import torch
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


class Case:
    """Seeded inputs of a config restricted to a few heads."""

    def __init__(self, cfg, heads, rho=None):
        self.cfg = cfg
        self.heads = list(heads)
        self.H = len(self.heads)
        self.rho = cfg.rho if rho is None else rho
        self.q, self.k, self.v = synth.make_inputs(cfg, self.heads)
        self.init_q = np.stack([synth.forgy_init(cfg, self.q[i], h, 0, cfg.Cq) for i, h in enumerate(self.heads)])
        self.init_k = np.stack([synth.forgy_init(cfg, self.k[i], h, 1, cfg.Ck) for i, h in enumerate(self.heads)])
        self.scale = 1.0 / math.sqrt(cfg.d)

    def params(self, **kw):
        c = self.cfg
        d = dict(H=self.H, Nq=c.N, Nk=c.N, d=c.d, Cq=c.Cq, Ck=c.Ck, iters=c.iters, rho=self.rho,
                 scale=self.scale, dtype=sv.SVGEAR_BF16 if c.dtype == "bf16" else sv.SVGEAR_F32)
        d.update(kw)
        return sv.params(**d)

    def dq(self):
        return dev(self.q, torch_dtype(self.cfg))

    def dk(self):
        return dev(self.k, torch_dtype(self.cfg))

    def dv(self):
        return dev(self.v, torch_dtype(self.cfg))

    @functools.cached_property
    def oracle(self):
        """Full oracle forward per head (float64)."""
        c = self.cfg
        return [ora.forward(self.q[i], self.k[i], self.v[i], c.Cq, c.Ck, c.iters, self.rho,
                            self.scale, self.init_q[i], self.init_k[i]) for i in range(self.H)]


@functools.lru_cache(maxsize=None)
def case(name, heads=None, rho=None):
    cfg = synth.CONFIGS[name]
    if heads is None:
        heads = (0,) if cfg.H == 1 else (0, 5)
    return Case(cfg, heads, rho)


def assert_close(got, ref, atol, rtol, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    lim = atol + rtol * np.abs(ref)
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} (atol {atol}, rtol {rtol})")


def label_mismatches_are_ties(X, mu, gpu_labels):
    """Every label that differs from the float64 argmin must be a near-tie
    ((d2 - d1) / d2 < TIE_REL).  Returns the number of differing labels."""
    lab, d1, d2 = ora.assign_margin(X, mu)
    diff = np.nonzero(lab != gpu_labels)[0]
    if diff.size:
        gap = (d2[diff] - d1[diff]) / np.maximum(d2[diff], 1e-300)
        assert (gap < TIE_REL).all(), (f"{int((gap >= TIE_REL).sum())} labels differ from the exact "
                                      f"argmin at non-tied points, e.g. index {diff[gap >= TIE_REL][:5]}")
    return int(diff.size)


def _tied_route_row(Erow, kc):
    """True when two adjacent ratios of the row's routing order are within
    TIE_REL of each other (the routed set may then differ legitimately)."""
    order = ora.route_order(Erow, kc)
    v = Erow[order]
    return bool((np.abs(np.diff(v)) <= TIE_REL * np.maximum(np.abs(v[:-1]), 1e-300)).any())


def stratified_rows(lq, Cq, n, rng):
    """About n query rows spread over the query clusters: ceil(n / Cq) rows
    (or all of them) from every non-empty cluster."""
    per = -(-n // Cq)
    rows = []
    for a in range(Cq):
        members = np.nonzero(lq == a)[0]
        if members.size:
            rows.append(rng.choice(members, min(per, members.size), replace=False))
    return np.sort(np.concatenate(rows))


def check_forward_given_gpu_clusters(views, O, h, Q, K, V, Cq, Ck, rho, scale, dtype, rows=None,
                                     budget_global=False):
    """One head of an svgear_forward result against the oracle given the
    GPU's own inputs to every stage, so that a near-tie that moved a label in
    the ten chained k-means rounds never turns the comparison off:

    * labels are the exact argmin for the GPU's final centroids (ties exempt);
    * counts, offsets and the stable permutations follow the labels; the
      value centroids are the member means;
    * the block error from these clusters is within 1e-3 relative (floor
      1e-6 T);
    * the routing from the GPU's errors equals the oracle's (rows with
      near-tied ratios exempt) and meets the budget;
    * the output on `rows` (all rows if None) equals the oracle's hybrid
      attention for the GPU's clusters and routing.

    Q, K, V: [N, d] inputs of the head (the values the GPU received)."""
    g = lambda n: host(views[n][h])
    cq, ck, vbar = (g(n).astype(np.float64) for n in ("cent_q", "cent_k", "vbar"))
    lq, lk = g("labels_q").astype(np.int64), g("labels_k").astype(np.int64)
    label_mismatches_are_ties(Q, cq, lq)
    label_mismatches_are_ties(K, ck, lk)
    cnt_q, cnt_k = g("counts_q"), g("counts_k")
    assert np.array_equal(cnt_q, np.bincount(lq, minlength=Cq))
    assert np.array_equal(cnt_k, np.bincount(lk, minlength=Ck))
    assert np.array_equal(g("off_k"), np.concatenate([[0], np.cumsum(cnt_k)]))
    assert np.array_equal(g("off_q"), np.concatenate([[0], np.cumsum(cnt_q)]))
    assert np.array_equal(g("perm_k"), np.argsort(lk, kind="stable"))
    assert np.array_equal(g("perm_q"), np.argsort(lq, kind="stable"))
    assert_close(vbar, ora.value_centroids(V, lk, Ck), 1e-5, 1e-5, "value centroids")
    args = (cq, ck, vbar, K, V, lk, cnt_k, scale)
    Eo, Mo = ora.block_error(*args)
    T = ora.block_error_scale(*args)
    E = g("E").astype(np.float64)
    assert_close(g("M"), Mo, 1e-5, 1e-6, "row shift M")
    err = np.abs(E - Eo)
    lim = E_RTOL * np.abs(Eo) + E_FLOOR * T
    assert (err <= lim).all(), f"E: {int((err > lim).sum())} entries outside 1e-3 relative"
    mask = g("mask")
    if budget_global:
        mask_o, _, pairs_o = ora.route_global(E, g("M").astype(np.float64), cnt_k, cnt_q, rho)
        assert int((np.outer(cnt_q, cnt_k) * mask).sum()) <= ora.route_global_budget(rho, int(cnt_q.sum()),
                                                                                      int(cnt_k.sum()))
    else:
        mask_o, _, pairs_o = ora.route(E, cnt_k, cnt_q, rho)
        budget = ora.route_budget(rho, int(cnt_k.sum()))
        for a in range(Cq):
            assert (cnt_k * mask[a]).sum() <= budget
            if not np.array_equal(mask[a], mask_o[a]):
                assert _tied_route_row(E[a], cnt_k), f"routing row {a} differs without a tie"
    if np.array_equal(mask, mask_o):
        assert int(g("exec_pairs")) == pairs_o
    if rows is None:
        lq_s = lq
        sel = slice(None)
    else:
        lq_s = np.full_like(lq, -1)
        lq_s[rows] = lq[rows]
        sel = rows
    Oo = ora.hybrid_attention(Q, K, V, lq_s, lk, ck, vbar, cnt_k, mask, scale)
    atol, rtol = OUT_TOL[dtype]
    assert_close(np.asarray(O)[sel], Oo[sel], atol, rtol, f"output head {h} given the GPU's clusters")
