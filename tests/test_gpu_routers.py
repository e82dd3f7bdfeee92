"""GPU parity of the routing ablations against the oracle: the two ranking
signals (attention mass and the value-agnostic error) on the oracle's clusters,
global-budget routing on the oracle's errors, then whole forwards whose routing
and output are checked against the oracle given the GPU's own upstream results."""
import numpy as np
import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from oracle import svgear_oracle as ora
from helpers import E_FLOOR, E_RTOL, OUT_TOL, TIE_REL, assert_close, case, dev, host, torch_dtype

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROUTERS = {"mass": sv.SVGEAR_ROUTE_MASS, "error_nov": sv.SVGEAR_ROUTE_ERROR_NOV}
MASS_TOL = (1e-7, 1e-4)   # atol, rtol: float32 exp of float32 logits, float64 row sum


def _check_signal(router, Eg, Mg, qb, kb, vb, k, v, lk, kc, scale):
    Eo, Mo = ora.routing_signal(router, qb, kb, vb, k, v, lk, kc, scale)
    assert_close(Mg, Mo, 1e-5, 1e-6, "row shift M")
    if router == "mass":
        assert_close(Eg, Eo, *MASS_TOL, "attention mass")
        return
    # size of the two terms whose difference the value-agnostic error measures
    u = np.zeros((1, k.shape[1])); u[0, 0] = 1.0
    T = ora.block_error_scale(qb, kb, np.repeat(u, kb.shape[0], 0), k, np.repeat(u, k.shape[0], 0),
                              lk, kc, scale)
    err = np.abs(Eg - Eo)
    lim = E_RTOL * np.abs(Eo) + E_FLOOR * T
    assert (err <= lim).all(), f"E: {(err > lim).sum()} entries outside"


@pytest.mark.parametrize("router", list(ROUTERS))
@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_signal_given_oracle_clusters(name, router):
    cs = case(name)
    cfg = cs.cfg
    H = cs.H
    tdt = torch_dtype(cfg)
    f = lambda x: np.asarray(x, dtype=np.float32)
    Qb, Kb, Vb, Kp, Vp, koff, ks = [], [], [], [], [], [], []
    for i in range(H):
        o = cs.oracle[i]
        Qb.append(f(o["Qbar"])); Kb.append(f(o["Kbar"])); Vb.append(f(o["Vbar"]))
        Kp.append(cs.k[i][o["perm_k"]]); Vp.append(cs.v[i][o["perm_k"]])
        koff.append(o["off_k"].astype(np.int32))
        ks.append(ora.key_scalars(cs.v[i], o["k_labels"], Vb[-1].astype(np.float64))[:, o["perm_k"]])
    p = cs.params(router=ROUTERS[router])
    E = torch.empty((H, cfg.Cq, cfg.Ck), dtype=torch.float32, device="cuda")
    M = torch.empty((H, cfg.Cq), dtype=torch.float32, device="cuda")
    ws = sv.workspace(sv.svgear_block_error_workspace_size(p))
    sv.svgear_block_error(dev(np.stack(Qb)), dev(np.stack(Kb)), dev(np.stack(Vb)), dev(np.stack(Kp), tdt),
                          dev(np.stack(Vp), tdt), dev(np.stack(koff)),
                          dev(np.stack(ks, axis=1).astype(np.float32)), p, E, M, ws, ws.numel())
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    E, M = host(E), host(M)
    for i in range(H):
        o = cs.oracle[i]
        _check_signal(router, E[i], M[i], Qb[i], Kb[i], Vb[i], cs.k[i], cs.v[i], o["k_labels"],
                      o["k_counts"], cs.scale)


def _tied_rows(Erow, kc):
    order = ora.route_order(Erow, kc)
    v = Erow[order]
    return (np.abs(np.diff(v)) <= TIE_REL * np.maximum(np.abs(v[:-1]), 1e-300)).any()


@pytest.mark.parametrize("router", list(ROUTERS))
@pytest.mark.parametrize("name,rho", [("tiny", None), ("mid", None), ("mid", 0.1)])
def test_forward_with_ablation_router(name, rho, router):
    cs = case(name, rho=rho)
    cfg = cs.cfg
    O, ws, p, _ = sv.forward(cs.dq(), cs.dk(), cs.dv(), cfg.Cq, cfg.Ck, cfg.iters, cs.rho, cs.scale,
                             dev(cs.init_q), dev(cs.init_k), router=ROUTERS[router])
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    vw = sv.view_tensors(p, ws)
    O = host(O)
    atol, rtol = OUT_TOL[cfg.dtype]
    for i in range(cs.H):
        cq, ck, vbar = (host(vw[n][i]).astype(np.float64) for n in ("cent_q", "cent_k", "vbar"))
        lq, lk = host(vw["labels_q"][i]), host(vw["labels_k"][i])
        kc, qc = host(vw["counts_k"][i]), host(vw["counts_q"][i])
        E, mask = host(vw["E"][i]), host(vw["mask"][i])
        # the signal from the GPU's own clusters
        _check_signal(router, E, host(vw["M"][i]), cq, ck, vbar, cs.k[i], cs.v[i], lk, kc, cs.scale)
        # routing from the GPU's signal (rows with near-tied values exempt)
        mask_o, _, _ = ora.route(E, kc, qc, cs.rho)
        for a in range(cfg.Cq):
            if not np.array_equal(mask[a], mask_o[a]):
                assert _tied_rows(E[a], kc), f"routing row {a} differs without a tie"
        # hybrid attention from the GPU's clusters and routing
        Oo = ora.hybrid_attention(cs.q[i], cs.k[i], cs.v[i], lq, lk, ck, vbar, kc, mask, cs.scale)
        assert_close(O[i], Oo, atol, rtol, f"{router} forward output head {i}")


# ------------------------------------------------------------ global budget

def _global_keys(E, M):
    with np.errstate(divide="ignore"):
        return np.log(np.maximum(np.asarray(E, np.float64), 0.0)) + 2.0 * np.asarray(M, np.float64)[:, None]


def _check_global(mask, n_sel, sel, pairs, E, M, kc, qc, rho):
    """GPU global routing against the oracle's from the same float32 E, M:
    identical, or differing only on items whose keys are near-tied at the cut."""
    mask_o, sel_o, pairs_o = ora.route_global(E, M, kc, qc, rho)
    budget = ora.route_global_budget(rho, int(qc.sum()), int(kc.sum()))
    cost = qc[:, None].astype(np.int64) * kc[None, :]
    assert pairs == int((cost * mask).sum()) <= budget
    assert (mask[qc == 0] == 0).all() and (mask[:, kc == 0] == 0).all()
    diff = mask != mask_o
    if diff.any():
        key = _global_keys(E, M)[diff]
        assert np.isfinite(key).all() and key.max() - key.min() <= 1e-5 * max(1.0, np.abs(key).max()), \
            f"{diff.sum()} routing decisions differ away from the cut"
    else:
        assert pairs == pairs_o
        for a in range(mask.shape[0]):
            assert n_sel[a] == len(sel_o[a])
            # the row's order; near-equal keys inside a row may swap
            assert set(sel[a, :n_sel[a]]) == set(sel_o[a])


@pytest.mark.parametrize("name,rho", [("tiny", None), ("mid", None), ("mid", 0.05), ("mid", 0.0), ("mid", 1.0)])
def test_route_global_given_oracle_errors(name, rho):
    cs = case(name, rho=rho)
    cfg = cs.cfg
    H, Cq, Ck = cs.H, cfg.Cq, cfg.Ck
    E = np.stack([o["E"] for o in cs.oracle]).astype(np.float32)
    M = np.stack([o["M"] for o in cs.oracle]).astype(np.float32)
    kc = np.stack([o["k_counts"] for o in cs.oracle]).astype(np.int32)
    qc = np.stack([o["q_counts"] for o in cs.oracle]).astype(np.int32)
    # an empty query cluster routes nothing (members moved, total kept at N_q)
    qc[0, 0] += qc[0, 1]
    qc[0, 1] = 0
    p = cs.params()
    mask = torch.empty((H, Cq, Ck), dtype=torch.uint8, device="cuda")
    sel = torch.empty((H, Cq, Ck), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((H, Cq), dtype=torch.int32, device="cuda")
    pairs = torch.empty((H,), dtype=torch.int64, device="cuda")
    sv.svgear_route_global(dev(E), dev(M), dev(kc), dev(qc), p, mask, sel, n_sel, pairs)
    torch.cuda.synchronize()
    mask, sel, n_sel, pairs = host(mask), host(sel), host(n_sel), host(pairs)
    for i in range(H):
        _check_global(mask[i], n_sel[i], sel[i], int(pairs[i]), E[i], M[i], kc[i].astype(np.int64),
                      qc[i].astype(np.int64), cs.rho)
    if cs.rho == 1.0:
        assert (pairs == cfg.N * cfg.N).all()
    if cs.rho == 0.0:
        assert mask.sum() == 0


@pytest.mark.parametrize("name,rho", [("tiny", None), ("mid", None), ("mid", 0.1)])
def test_forward_with_global_budget(name, rho):
    cs = case(name, rho=rho)
    cfg = cs.cfg
    O, ws, p, _ = sv.forward(cs.dq(), cs.dk(), cs.dv(), cfg.Cq, cfg.Ck, cfg.iters, cs.rho, cs.scale,
                             dev(cs.init_q), dev(cs.init_k), budget=sv.SVGEAR_BUDGET_GLOBAL)
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    vw = sv.view_tensors(p, ws)
    O = host(O)
    atol, rtol = OUT_TOL[cfg.dtype]
    for i in range(cs.H):
        ck, vbar = (host(vw[n][i]).astype(np.float64) for n in ("cent_k", "vbar"))
        lq, lk = host(vw["labels_q"][i]), host(vw["labels_k"][i])
        kc, qc = host(vw["counts_k"][i]).astype(np.int64), host(vw["counts_q"][i]).astype(np.int64)
        mask = host(vw["mask"][i])
        _check_global(mask, host(vw["n_sel"][i]), host(vw["sel"][i]), int(host(vw["exec_pairs"][i])),
                      host(vw["E"][i]), host(vw["M"][i]), kc, qc, cs.rho)
        Oo = ora.hybrid_attention(cs.q[i], cs.k[i], cs.v[i], lq, lk, ck, vbar, kc, mask, cs.scale)
        assert_close(O[i], Oo, atol, rtol, f"global-budget forward output head {i}")
