"""Parity at full size, in the launch configuration bench.py times: the
Wan-shaped layer (40 heads, N = 75,600, d = 128, Cq = 100, Ck = 500,
rho = 0.15), the HunyuanVideo-shaped layer (24 heads, N = 118,800, Cq = 100,
Ck = 1000, rho = 0.12) and the stress workload (16 heads, N = 32,768,
Cq = 64, Ck = 512) at its base point (sigma 0.35, rho 0.1) and at tight,
dispersed and fully routed points of its sweep, ten k-means rounds each, in
one svgear_forward.
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

from helpers import OUT_TOL, assert_close, check_forward_given_gpu_clusters, dev, host, stratified_rows

ROWS = 1024
HEADS = {"wan": (0, 27), "hunyuan": (0, 23), "stress": (0, 11)}


@pytest.mark.gpu
@pytest.mark.parametrize("name,sigma,rho", [
    ("wan", None, None),
    ("hunyuan", None, None),
    ("stress", None, None),      # base point: sigma 0.35, rho 0.1
    ("stress", 0.1, 0.2),        # tight clusters
    ("stress", 1.0, 0.4),        # dispersed clusters
    ("stress", 0.35, 1.0),       # every block routed: dense attention
])
def test_full_layer_sampled_parity(name, sigma, rho):
    import torch
    import bench
    cfg = synth.CONFIGS[name]
    if sigma is not None:
        cfg = cfg.with_(sigma=sigma)
    if rho is not None:
        cfg = cfg.with_(rho=rho)
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
        rows = stratified_rows(host(vw["labels_q"][h]), cfg.Cq, ROWS, rng)
        check_forward_given_gpu_clusters(vw, host(O[h]), h, q[h], k[h], v[h], cfg.Cq, cfg.Ck, cfg.rho, s,
                                         "bf16", rows=rows)
        if cfg.rho == 1.0:
            assert_close(host(O[h])[rows], ora.dense_attention(q[h][rows], k[h], v[h], s), *OUT_TOL["bf16"],
                         f"{name} rho = 1 head {h} against dense attention")


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
