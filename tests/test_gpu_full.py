"""Parity at full size, in the launch configuration bench.py times: the
Wan-shaped layer (40 heads, N = 75,600, d = 128, Cq = 100, Ck = 500,
rho = 0.15), the HunyuanVideo-shaped layer (24 heads, N = 118,800, Cq = 100,
Ck = 1000, rho = 0.12) and the stress base point (16 heads, N = 32,768,
Cq = 64, Ck = 512, rho = 0.1), ten k-means rounds each, in one svgear_forward.
The oracle cannot run a whole layer, so on two sampled heads every stage is
checked against the oracle given the GPU's own inputs to that stage, and the
hybrid attention on 1,024 query rows per head sampled across the query
clusters."""
import math

import numpy as np
import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from clustered_sparse_attention_flash_b200 import synth
from oracle import svgear_oracle as ora

from helpers import E_FLOOR, E_RTOL, OUT_TOL, TIE_REL, assert_close, dev, host, label_mismatches_are_ties

ROWS = 1024
HEADS = {"wan": (0, 27), "hunyuan": (0, 23), "stress": (0, 11)}


def _tied_rows(Erow, kc):
    order = ora.route_order(Erow, kc)
    v = Erow[order]
    return (np.abs(np.diff(v)) <= TIE_REL * np.maximum(np.abs(v[:-1]), 1e-300)).any()


def _stratified_rows(lq, Cq, n, rng):
    """About n query rows spread over the query clusters: ceil(n / Cq) rows
    (or all of them) from every non-empty cluster."""
    per = -(-n // Cq)
    rows = []
    for a in range(Cq):
        members = np.nonzero(lq == a)[0]
        if members.size:
            rows.append(rng.choice(members, min(per, members.size), replace=False))
    return np.sort(np.concatenate(rows))


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["wan", "hunyuan", "stress"])
def test_full_layer_sampled_parity(name):
    import torch
    import bench
    cfg = synth.CONFIGS[name]
    q, k, v, iq, ik = bench.generate(cfg)
    s = 1.0 / math.sqrt(cfg.d)
    bf = torch.bfloat16
    O, ws, p, _ = sv.forward(dev(q, bf), dev(k, bf), dev(v, bf), cfg.Cq, cfg.Ck, cfg.iters, cfg.rho, s,
                             dev(iq), dev(ik))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    vw = sv.view_tensors(p, ws)
    rng = np.random.default_rng(20260)
    for h in HEADS[name]:
        Q, K, V = q[h], k[h], v[h]
        cq, ck, vbar = (host(vw[n][h]).astype(np.float64) for n in ("cent_q", "cent_k", "vbar"))
        lq, lk = host(vw["labels_q"][h]), host(vw["labels_k"][h])
        # a1: labels are the exact argmin for the final centroids (ties exempt)
        label_mismatches_are_ties(Q, cq, lq)
        label_mismatches_are_ties(K, ck, lk)
        # a3: counts, offsets and the stable permutation follow the labels;
        # value centroids are the member means
        cnt_k = host(vw["counts_k"][h])
        assert np.array_equal(cnt_k, np.bincount(lk, minlength=cfg.Ck))
        assert np.array_equal(host(vw["off_k"][h]), np.concatenate([[0], np.cumsum(cnt_k)]))
        assert np.array_equal(host(vw["perm_k"][h]), np.argsort(lk, kind="stable"))
        assert np.array_equal(host(vw["counts_q"][h]), np.bincount(lq, minlength=cfg.Cq))
        assert np.array_equal(host(vw["perm_q"][h]), np.argsort(lq, kind="stable"))
        assert_close(vbar, ora.value_centroids(V, lk, cfg.Ck), 1e-5, 1e-5, "value centroids")
        # a4: block error from these clusters
        args = (cq, ck, vbar, K, V, lk, cnt_k, s)
        Eo, Mo = ora.block_error(*args)
        T = ora.block_error_scale(*args)
        E = host(vw["E"][h])
        assert_close(host(vw["M"][h]), Mo, 1e-5, 1e-6, "row shift M")
        err = np.abs(E - Eo)
        lim = E_RTOL * np.abs(Eo) + E_FLOOR * T
        assert (err <= lim).all(), f"E: {(err > lim).sum()} entries outside"
        # a5: routing from the GPU's errors (rows with near-tied ratios exempt)
        cnt_q = host(vw["counts_q"][h])
        mask_o, _, pairs_o = ora.route(E, cnt_k, cnt_q, cfg.rho)
        mask = host(vw["mask"][h])
        for a in range(cfg.Cq):
            if not np.array_equal(mask[a], mask_o[a]):
                assert _tied_rows(E[a], cnt_k), f"routing row {a} differs without a tie"
        if np.array_equal(mask, mask_o):
            assert int(host(vw["exec_pairs"][h])) == pairs_o
        # a6: sampled query rows against the oracle's hybrid attention
        rows = _stratified_rows(lq, cfg.Cq, ROWS, rng)
        lq_s = np.full_like(lq, -1)
        lq_s[rows] = lq[rows]
        Oo = ora.hybrid_attention(Q, K, V, lq_s, lk, ck, vbar, cnt_k, mask, s)
        atol, rtol = OUT_TOL["bf16"]
        assert_close(host(O[h])[rows], Oo[rows], atol, rtol, f"{name} hybrid output head {h}")


@pytest.mark.gpu
def test_stress_yardstick_rows_match_oracle_dense():
    """The float32 dense attention the stress sweep measures against, on
    sampled rows of one head, equals the oracle's float64 dense attention."""
    import torch
    import bench
    cfg = synth.CONFIGS["stress"]
    q, k, v, _ = synth.make_head(cfg, 3)
    s = 1.0 / math.sqrt(cfg.d)
    torch.backends.cuda.matmul.allow_tf32 = False
    Qd, Kd, Vd = (torch.from_numpy(x).cuda()[None] for x in (q, k, v))
    ref = bench._dense_fp32(Qd, Kd, Vd, s)[0].cpu().numpy()
    rows = np.random.default_rng(5).choice(cfg.N, 256, replace=False)
    want = ora.dense_attention(q[rows], k, v, s)
    assert_close(ref[rows], want, 1e-5, 1e-4, "float32 dense yardstick")
