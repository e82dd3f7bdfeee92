"""GPU parity: every C-ABI stage against the CPU oracle on the same seeded
inputs.  Stage tests feed the oracle's upstream results into the GPU stage so
that each comparison sees identical discrete inputs; the end-to-end test runs
both sides independently."""
import math

import numpy as np
import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from oracle import svgear_oracle as ora
from helpers import (E_FLOOR, E_RTOL, OUT_TOL, TIE_REL, assert_close, case, check_forward_given_gpu_clusters,
                     dev, host, label_mismatches_are_ties, stratified_rows, torch_dtype)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CONFIGS = ["tiny", "mid"]


def _kmeans_gpu(X, dtype, C, iters, init):
    H, N, d = X.shape
    cent = torch.empty((H, C, d), dtype=torch.float32, device="cuda")
    labels = torch.empty((H, N), dtype=torch.int32, device="cuda")
    counts = torch.empty((H, C), dtype=torch.int32, device="cuda")
    n = sv.svgear_kmeans_workspace_size(H, N, d, C)
    ws = sv.workspace(n)
    sv.svgear_kmeans(X, dtype, H, N, d, C, iters, init, cent, labels, counts, ws, ws.numel())
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    return host(cent), host(labels).astype(np.int64), host(counts)


def _code(cfg):
    return sv.SVGEAR_BF16 if cfg.dtype == "bf16" else sv.SVGEAR_F32


# ------------------------------------------------------------------ k-means

@pytest.mark.parametrize("name", CONFIGS)
def test_kmeans_labels_exact_given_oracle_centroids(name):
    cs = case(name)
    cfg = cs.cfg
    for X, init, C in ((cs.q, cs.init_q, cfg.Cq), (cs.k, cs.init_k, cfg.Ck)):
        mus = np.stack([ora.kmeans(X[i], C, 3, init[i])[0] for i in range(cs.H)]).astype(np.float32)
        _, lab, cnt = _kmeans_gpu(dev(X, torch_dtype(cfg)), _code(cfg), C, 0, dev(mus))
        for i in range(cs.H):
            label_mismatches_are_ties(X[i], mus[i], lab[i])
            np.testing.assert_array_equal(cnt[i], np.bincount(lab[i], minlength=C))


@pytest.mark.parametrize("name", CONFIGS)
def test_kmeans_update_given_same_labels(name):
    cs = case(name)
    cfg = cs.cfg
    X, init, C = cs.k, cs.init_k, cfg.Ck
    mus = np.stack([ora.kmeans(X[i], C, 2, init[i])[0] for i in range(cs.H)]).astype(np.float32)
    cent, _, _ = _kmeans_gpu(dev(X, torch_dtype(cfg)), _code(cfg), C, 1, dev(mus))
    for i in range(cs.H):
        lab = ora.assign(X[i], mus[i])
        want, _ = ora.update(X[i], lab, mus[i])
        err = np.linalg.norm(cent[i] - want, axis=1)
        assert (err <= 1e-5 * np.linalg.norm(want, axis=1) + 1e-7).all(), err.max()


@pytest.mark.parametrize("name", CONFIGS)
def test_kmeans_full_iterations_inertia(name):
    cs = case(name)
    cfg = cs.cfg
    for X, init, C in ((cs.q, cs.init_q, cfg.Cq), (cs.k, cs.init_k, cfg.Ck)):
        cent, lab, _ = _kmeans_gpu(dev(X, torch_dtype(cfg)), _code(cfg), C, cfg.iters, dev(init))
        for i in range(cs.H):
            mu, olab, _ = ora.kmeans(X[i], C, cfg.iters, init[i])
            gi = ora.inertia(X[i], cent[i], lab[i])
            oi = ora.inertia(X[i], mu, olab)
            assert abs(gi - oi) <= 1e-4 * oi, (gi, oi)
            # the GPU labels are the exact argmin against the GPU centroids
            label_mismatches_are_ties(X[i], cent[i], lab[i])


# ------------------------------------------------------------------ permute

@pytest.mark.parametrize("name", CONFIGS)
def test_permute_given_oracle_labels(name):
    cs = case(name)
    cfg = cs.cfg
    H, N, d, C = cs.H, cfg.N, cfg.d, cfg.Ck
    lab = np.stack([o["k_labels"] for o in cs.oracle]).astype(np.int32)
    tdt = torch_dtype(cfg)
    K, V = cs.dk(), cs.dv()
    Kp, Vp = torch.empty_like(K), torch.empty_like(V)
    perm = torch.empty((H, N), dtype=torch.int32, device="cuda")
    off = torch.empty((H, C + 1), dtype=torch.int32, device="cuda")
    vbar = torch.empty((H, C, d), dtype=torch.float32, device="cuda")
    ks = torch.empty((3, H, N), dtype=torch.float32, device="cuda")
    ws = sv.workspace(sv.svgear_permute_workspace_size(H, N, C))
    sv.svgear_permute(K, _code(cfg), dev(lab), H, N, d, C, Kp, perm, off, V, Vp, vbar, ks, ws, ws.numel())
    torch.cuda.synchronize()
    perm, off, Kp, Vp, vbar, ks = map(host, (perm, off, Kp, Vp, vbar, ks))
    for i in range(H):
        o = cs.oracle[i]
        np.testing.assert_array_equal(perm[i], o["perm_k"])
        np.testing.assert_array_equal(off[i], o["off_k"])
        np.testing.assert_array_equal(Kp[i], cs.k[i][o["perm_k"]])
        np.testing.assert_array_equal(Vp[i], cs.v[i][o["perm_k"]])
        assert_close(vbar[i], o["Vbar"], 1e-6, 1e-5, "value centroids")
        want = ora.key_scalars(cs.v[i], o["k_labels"], vbar[i].astype(np.float64))[:, o["perm_k"]]
        scale = want[2].mean()
        assert_close(ks[:, i], want, 1e-5 * scale, 1e-4, "key scalars")


# -------------------------------------------------------------- block error

def _oracle_stage_inputs(cs, i):
    """Oracle intermediates of head i rounded to the ABI's float32."""
    o = cs.oracle[i]
    f = lambda x: np.asarray(x, dtype=np.float32)
    return o, f(o["Qbar"]), f(o["Kbar"]), f(o["Vbar"])


@pytest.mark.parametrize("name", CONFIGS)
def test_block_error_given_oracle_clusters(name):
    cs = case(name)
    cfg = cs.cfg
    H, N, d = cs.H, cfg.N, cfg.d
    tdt = torch_dtype(cfg)
    Qb, Kb, Vb, Kp, Vp, koff, ks = [], [], [], [], [], [], []
    for i in range(H):
        o, qb, kb, vb = _oracle_stage_inputs(cs, i)
        Qb.append(qb); Kb.append(kb); Vb.append(vb)
        Kp.append(cs.k[i][o["perm_k"]]); Vp.append(cs.v[i][o["perm_k"]])
        koff.append(o["off_k"].astype(np.int32))
        ks.append(ora.key_scalars(cs.v[i], o["k_labels"], vb.astype(np.float64))[:, o["perm_k"]])
    p = cs.params()
    E = torch.empty((H, cfg.Cq, cfg.Ck), dtype=torch.float32, device="cuda")
    M = torch.empty((H, cfg.Cq), dtype=torch.float32, device="cuda")
    ws = sv.workspace(sv.svgear_block_error_workspace_size(p))
    ksd = dev(np.stack(ks, axis=1).astype(np.float32))
    sv.svgear_block_error(dev(np.stack(Qb)), dev(np.stack(Kb)), dev(np.stack(Vb)), dev(np.stack(Kp), tdt),
                          dev(np.stack(Vp), tdt), dev(np.stack(koff)), ksd, p, E, M, ws, ws.numel())
    torch.cuda.synchronize()
    E, M = host(E), host(M)
    for i in range(H):
        o = cs.oracle[i]
        kc = o["k_counts"]
        args = (Qb[i], Kb[i], Vb[i], cs.k[i], cs.v[i], o["k_labels"], kc, cs.scale)
        Eo, Mo = ora.block_error(*args)
        T = ora.block_error_scale(*args)
        assert_close(M[i], Mo, 1e-5, 1e-6, "row shift M")
        err = np.abs(E[i] - Eo)
        lim = E_RTOL * np.abs(Eo) + E_FLOOR * T
        assert (err <= lim).all(), f"E: {(err > lim).sum()} entries outside, worst {np.max(err / np.maximum(lim, 1e-300))}"


# ------------------------------------------------------------------- route

def _route_gpu(cs, E, kc, qc, p):
    H, Cq, Ck = cs.H, cs.cfg.Cq, cs.cfg.Ck
    mask = torch.empty((H, Cq, Ck), dtype=torch.uint8, device="cuda")
    sel = torch.empty((H, Cq, Ck), dtype=torch.int32, device="cuda")
    nsel = torch.empty((H, Cq), dtype=torch.int32, device="cuda")
    ep = torch.empty((H,), dtype=torch.int64, device="cuda")
    sv.svgear_route(dev(E.astype(np.float32)), dev(kc.astype(np.int32)), dev(qc.astype(np.int32)), p,
                    mask, sel, nsel, ep)
    torch.cuda.synchronize()
    return host(mask), host(sel), host(nsel), host(ep)


def _tied_rows(Erow, kc):
    """Rows whose ratio order has adjacent non-empty entries within TIE_REL."""
    order = ora.route_order(Erow, kc)
    v = Erow[order]
    gaps = np.abs(np.diff(v)) <= TIE_REL * np.maximum(np.abs(v[:-1]), 1e-300)
    return gaps.any()


@pytest.mark.parametrize("name,rho", [("tiny", None), ("mid", None), ("mid", 0.1), ("mid", 0.0), ("mid", 1.0)])
def test_route_given_oracle_errors(name, rho):
    cs = case(name)
    rho = cs.rho if rho is None else rho
    p = cs.params(rho=rho)
    E = np.stack([o["E"] for o in cs.oracle]).astype(np.float32)
    kc = np.stack([o["k_counts"] for o in cs.oracle])
    qc = np.stack([o["q_counts"] for o in cs.oracle])
    mask, sel, nsel, ep = _route_gpu(cs, E, kc, qc, p)
    for i in range(cs.H):
        # the oracle routes the same float32 values the GPU received
        om, osel, opairs = ora.route(E[i].astype(np.float64), kc[i], qc[i], rho)
        budget = ora.route_budget(rho, int(kc[i].sum()))
        for a in range(cs.cfg.Cq):
            assert (kc[i] * mask[i, a]).sum() <= budget
            if np.array_equal(mask[i, a], om[a]):
                np.testing.assert_array_equal(sel[i, a, :nsel[i, a]], osel[a])
            else:
                assert _tied_rows(E[i, a].astype(np.float64), kc[i]), f"row {a} differs without a tie"
        if np.array_equal(mask[i], om):
            assert ep[i] == opairs


# --------------------------------------------------------- hybrid attention

@pytest.mark.parametrize("name,rho", [("tiny", None), ("mid", None), ("mid", 0.0), ("mid", 1.0)])
def test_hybrid_attn_given_oracle_routing(name, rho):
    cs = case(name)
    cfg = cs.cfg
    rho = cs.rho if rho is None else rho
    H, N, d = cs.H, cfg.N, cfg.d
    tdt = torch_dtype(cfg)
    Qp, Kp, Vp, qoff, koff, pq, Kb, Vb, sel, nsel, want = [], [], [], [], [], [], [], [], [], [], []
    for i in range(H):
        o, qb, kb, vb = _oracle_stage_inputs(cs, i)
        m, s, _ = ora.route(o["E"], o["k_counts"], o["q_counts"], rho)
        Qp.append(cs.q[i][o["perm_q"]]); Kp.append(cs.k[i][o["perm_k"]]); Vp.append(cs.v[i][o["perm_k"]])
        qoff.append(o["off_q"]); koff.append(o["off_k"]); pq.append(o["perm_q"])
        Kb.append(kb); Vb.append(vb)
        srow = np.zeros((cfg.Cq, cfg.Ck), dtype=np.int32)
        for a in range(cfg.Cq):
            srow[a, :len(s[a])] = s[a]
        sel.append(srow); nsel.append(np.array([len(x) for x in s], dtype=np.int32))
        want.append(ora.hybrid_attention(cs.q[i], cs.k[i], cs.v[i], o["q_labels"], o["k_labels"],
                                         kb, vb, o["k_counts"], m, cs.scale))
    p = cs.params(rho=rho)
    O = torch.empty((H, N, d), dtype=tdt, device="cuda")
    ws = sv.workspace(sv.svgear_hybrid_attn_workspace_size(p))
    i32 = lambda xs: dev(np.stack(xs).astype(np.int32))
    sv.svgear_hybrid_attn(dev(np.stack(Qp), tdt), dev(np.stack(Kp), tdt), dev(np.stack(Vp), tdt), i32(qoff),
                          i32(koff), i32(pq), dev(np.stack(Kb)), dev(np.stack(Vb)), i32(sel), i32(nsel), p, O,
                          ws, ws.numel())
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    atol, rtol = OUT_TOL[cfg.dtype]
    O = host(O)
    for i in range(H):
        assert_close(O[i], want[i], atol, rtol, f"hybrid output head {i}")


# --------------------------------------------------------------- end to end

@pytest.mark.parametrize("name,rho", [("tiny", None), ("mid", None), ("mid", 0.1)])
def test_forward_end_to_end(name, rho):
    """Whole forwards: every head is checked stage by stage against the oracle
    given the GPU's own clusters (never skipped), and, where the ten chained
    k-means rounds reproduced the oracle's clustering, the block error and the
    output are also held to the independent oracle run."""
    cs = case(name, rho=rho)
    cfg = cs.cfg
    O, ws, p, _ = sv.forward(cs.dq(), cs.dk(), cs.dv(), cfg.Cq, cfg.Ck, cfg.iters, cs.rho, cs.scale,
                             dev(cs.init_q), dev(cs.init_k))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    views = sv.view_tensors(p, ws)
    O = host(O)
    for i in range(cs.H):
        check_forward_given_gpu_clusters(views, O[i], i, cs.q[i], cs.k[i], cs.v[i], cfg.Cq, cfg.Ck, cs.rho,
                                         cs.scale, cfg.dtype)
    lq, lk = host(views["labels_q"]), host(views["labels_k"])
    mask, E = host(views["mask"]), host(views["E"])
    atol, rtol = OUT_TOL[cfg.dtype]
    for i in range(cs.H):
        o = cs.oracle[i]
        if not (np.array_equal(lq[i], o["q_labels"]) and np.array_equal(lk[i], o["k_labels"])):
            continue  # a near-tie moved a label somewhere in the chained rounds
        err = np.abs(E[i] - o["E"])
        assert (err <= E_RTOL * np.abs(o["E"]) + 1e-6 * np.abs(o["E"]).max()).all()
        if np.array_equal(mask[i], o["mask"]):
            assert_close(O[i], o["O"], atol, rtol, f"forward output head {i}")


# -------------------------------------------------------------- edge cases

def _small(N, d, seed, dtype):
    rng = np.random.default_rng(seed)
    X = [rng.standard_normal((1, N, d)).astype(np.float32) for _ in range(3)]
    if dtype == "bf16":
        from clustered_sparse_attention_flash_b200.synth import to_bf16_f32
        X = [to_bf16_f32(x) for x in X]
    return X


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,d,Cq,Ck,rho", [
    (1000, 64, 7, 13, 0.3),      # ragged sizes
    (333, 128, 5, 1, 0.0),       # one key cluster, pure compensation -> mean of V
    (300, 64, 4, 300, 0.2),      # singleton key clusters: exact for any rho
    (517, 128, 6, 9, 1.0),       # rho = 1: dense attention
    (130, 64, 1, 2, 0.5),        # one query cluster
    (257, 128, 3, 5, 0.4),       # a query cluster of more than two 128-row tiles
])
def test_forward_edge_cases(dtype, N, d, Cq, Ck, rho):
    q, k, v = _small(N, d, N + Ck, dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    s = 1 / math.sqrt(d)
    iq, ik = q[:, :Cq].copy(), k[:, :Ck].copy()
    O, ws, p, _ = sv.forward(dev(q, tdt), dev(k, tdt), dev(v, tdt), Cq, Ck, 4, rho, s, dev(iq), dev(ik))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    O = host(O)[0]
    views = sv.view_tensors(p, ws)
    check_forward_given_gpu_clusters(views, O, 0, q[0], k[0], v[0], Cq, Ck, rho, s, dtype)
    atol, rtol = OUT_TOL[dtype]
    if rho == 1.0 or Ck == N:
        assert_close(O, ora.dense_attention(q[0], k[0], v[0], s), atol, rtol, "dense special case")
    if Ck == 1 and rho == 0.0:
        assert_close(O, np.broadcast_to(v[0].astype(np.float64).mean(0), O.shape), atol, rtol, "mean of V")


@pytest.mark.parametrize("N,Ck,rho", [(8192, 1000, 1.0), (16384, 2000, 0.7)])
def test_forward_many_routed_clusters(N, Ck, rho):
    """Query clusters that route more key clusters than the attention kernel
    stages in shared memory (512): its producers then walk the selection list
    instead of the staged ranges.  Random bf16 inputs, d = 128."""
    d, Cq = 128, 8
    q, k, v = _small(N, d, 7 + Ck, "bf16")
    s = 1 / math.sqrt(d)
    iq, ik = q[:, :Cq].copy(), k[:, :Ck].copy()
    bf = torch.bfloat16
    O, ws, p, _ = sv.forward(dev(q, bf), dev(k, bf), dev(v, bf), Cq, Ck, 3, rho, s, dev(iq), dev(ik))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    views = sv.view_tensors(p, ws)
    nsel = host(views["n_sel"])[0]
    assert nsel.max() > 512, nsel.max()
    lq = host(views["labels_q"])[0]
    rows = stratified_rows(lq, Cq, 512, np.random.default_rng(Ck))
    check_forward_given_gpu_clusters(views, host(O)[0], 0, q[0], k[0], v[0], Cq, Ck, rho, s, "bf16", rows=rows)


@pytest.mark.parametrize("d", [64, 128])
def test_forward_row_maximum_grows_late(d):
    """One key cluster whose logits exceed every other key's by about 20
    (natural units) for every query: in the blocks whose stage order brings
    it after the first stage, the running maximum of every row grows by far
    more than 2^9 there, so the attention kernel's speculative pass rejects
    that stage (row sums above 2^16), reloads S and rescales.  With rho = 1
    every cluster is routed, so the output is dense attention.  Both head
    dimensions of the tensor-core kernel."""
    N, Cq, Ck = 8192, 8, 64
    q, k, v = _small(N, d, 41, "bf16")
    rng = np.random.default_rng(42)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    hot = rng.choice(N, size=256, replace=False)
    from clustered_sparse_attention_flash_b200.synth import to_bf16_f32
    k = k.copy()
    k[0, hot] += 15.0 * u
    q = q + 15.0 * u
    q, k = to_bf16_f32(q.astype(np.float32)), to_bf16_f32(k.astype(np.float32))
    s = 1 / math.sqrt(d)
    iq, ik = q[:, :Cq].copy(), k[:, :Ck].copy()
    ik[0, 0] = k[0, hot[0]]                      # one initial centroid among the hot keys
    bf = torch.bfloat16
    O, ws, p, _ = sv.forward(dev(q, bf), dev(k, bf), dev(v, bf), Cq, Ck, 3, 1.0, s, dev(iq), dev(ik))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    views = sv.view_tensors(p, ws)
    lk = host(views["labels_k"])[0]
    hot_clusters = set(lk[hot].tolist())
    assert not (hot_clusters & set(np.delete(lk, hot).tolist())), "hot keys share a cluster with others"
    assert (host(views["mask"])[0][:, host(views["counts_k"])[0] > 0] == 1).all()
    rows = np.random.default_rng(3).choice(N, size=768, replace=False)
    want = ora.dense_attention(q[0][rows], k[0], v[0], s)
    assert_close(host(O)[0][rows], want, *OUT_TOL["bf16"], "late maximum growth")


def test_forward_empty_key_cluster():
    """An initial centroid far from every key never gains members: the
    cluster stays empty, is never routed and contributes no compensation."""
    q, k, v = _small(400, 64, 3, "f32")
    ik = k[:, :6].copy()
    ik[0, 5] = 1e3
    iq = q[:, :4].copy()
    s = 0.125
    O, ws, p, _ = sv.forward(dev(q), dev(k), dev(v), 4, 6, 3, 0.4, s, dev(iq), dev(ik))
    torch.cuda.synchronize()
    views = sv.view_tensors(p, ws)
    assert host(views["counts_k"])[0, 5] == 0
    assert host(views["mask"])[0, :, 5].sum() == 0
    o = ora.forward(q[0], k[0], v[0], 4, 6, 3, 0.4, s, iq[0], ik[0])
    assert_close(host(O)[0], o["O"], *OUT_TOL["f32"], "empty-cluster output")


# ------------------------------------- tensor-core assignment, wide shapes

@pytest.mark.parametrize("N,d,C,seed", [
    (75600, 128, 500, 0),    # Wan-shaped key clustering: two accumulator slots
    (20000, 128, 300, 1),    # second slot ends in a 16-column tail
    (9001, 64, 1000, 2),     # d = 64: four slots alternate between warpgroups
    (5000, 128, 100, 3),     # one slot, tiles alternate between warpgroups
    (30000, 128, 1000, 4),   # centroids in two segments of 512 columns (HunyuanVideo-shaped keys)
    (9001, 128, 700, 5),     # segments of 512 and 192 columns
    (5000, 128, 513, 6),     # second segment is one 16-column chunk
])
def test_kmeans_assign_wide(N, d, C, seed):
    from clustered_sparse_attention_flash_b200.synth import to_bf16_f32
    rng = np.random.default_rng(seed)
    centers = rng.standard_normal((C // 2, d)).astype(np.float32) * 1.3
    X = to_bf16_f32(centers[rng.integers(0, C // 2, N)] + 0.5 * rng.standard_normal((N, d)).astype(np.float32))
    mu = X[rng.choice(N, C, replace=False)].astype(np.float32)
    mu = (mu + 0.05 * rng.standard_normal(mu.shape)).astype(np.float32)
    _, lab, cnt = _kmeans_gpu(dev(X[None], torch.bfloat16), sv.SVGEAR_BF16, C, 0, dev(mu[None]))
    nd = label_mismatches_are_ties(X, mu, lab[0])
    assert nd <= 2, nd
    np.testing.assert_array_equal(cnt[0], np.bincount(lab[0], minlength=C))


def test_head_sharded_forward_one_rank_is_the_forward():
    """The head-sharded entry with a single process runs every head through
    svgear_forward and returns exactly the plain forward's output."""
    from clustered_sparse_attention_flash_b200.shard import forward_heads_sharded
    cs = case("mid")
    cfg = cs.cfg
    O1, _, _, _ = sv.forward(cs.dq(), cs.dk(), cs.dv(), cfg.Cq, cfg.Ck, cfg.iters, cs.rho, cs.scale,
                             dev(cs.init_q), dev(cs.init_k))
    O2, hr = forward_heads_sharded(cs.dq(), cs.dk(), cs.dv(), cfg.Cq, cfg.Ck, cfg.iters, cs.rho, cs.scale,
                                   dev(cs.init_q), dev(cs.init_k))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    assert hr == (0, cs.H)
    assert torch.equal(O1, O2)
