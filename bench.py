#!/usr/bin/env python
"""Benchmark of the B200 SVG-EAR sparse-attention operator (one attention layer).

A step is one svgear_forward over the whole layer: k-means of queries and keys,
permutation, block error, routing and hybrid attention, on synthetic
video-DiT-shaped inputs already resident in HBM.  The headline value is the
dense-equivalent throughput 4*H*N^2*d / layer time; the line also carries the
per-layer ms, the executed-pair throughput of the attention stage, the routing
overhead and the per-stage breakdown.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config wan]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

With N > 1 (torchrun), every rank runs its own full layer (heads are
independent problems; no collective on the data path) and the value is the
work of all ranks over the slowest rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SVG-EAR attn layer ms & dense-equiv TFLOP/s at 75.6K tok; routing overhead %"
UNIT = "TFLOP/s (dense-equivalent 4*H*N^2*d per layer)"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="wan")
    ap.add_argument("--rho", type=float, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=None,
                    help="run only the first H heads of the workload (small profiler captures)")
    ap.add_argument("--shard-heads", action="store_true",
                    help="split one layer's heads over the ranks and all-gather O (strong scaling); "
                         "the default runs one whole layer per rank (weak scaling)")
    ap.add_argument("--stress", action="store_true",
                    help="error against dense attention over the noise sigma x budget rho grid "
                         "of the stress workload, for the method's router and two ablations")
    return ap.parse_args()


def _workload(cfg, rho):
    grid = "x".join(map(str, cfg.grid)) if cfg.grid else "uniform"
    return (f"{cfg.name}: H={cfg.H}, N={cfg.N} ({grid}), d={cfg.d}, {cfg.dtype}, Cq={cfg.Cq}, "
            f"Ck={cfg.Ck}, rho={rho}, kmeans iters={cfg.iters}, G={cfg.G} latent centers, "
            f"sigma={cfg.sigma}")


def _gen_head(args):
    cfg, h = args
    from clustered_sparse_attention_flash_b200 import synth
    q, k, v, _ = synth.make_head(cfg, h)
    iq = synth.forgy_init(cfg, q, h, 0, cfg.Cq)
    ik = synth.forgy_init(cfg, k, h, 1, cfg.Ck)
    return q, k, v, iq, ik


def generate(cfg):
    """All heads of the config, generated in a spawn pool (before any CUDA)."""
    import multiprocessing as mp
    import numpy as np
    from clustered_sparse_attention_flash_b200 import synth
    synth.logit_alpha(cfg)
    n = min(8, os.cpu_count() or 1, cfg.H)
    if n > 1:
        with mp.get_context("spawn").Pool(n) as pool:
            parts = pool.map(_gen_head, [(cfg, h) for h in range(cfg.H)])
    else:
        parts = [_gen_head((cfg, h)) for h in range(cfg.H)]
    return [np.stack([p[i] for p in parts]) for i in range(5)]


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons over a region.

    A reader thread stamps every sample with the host clock.  Entering waits
    (at most a few seconds) for the first sample, so that the sampler is up
    before the region starts; the summary keeps the samples taken inside the
    region plus the first one after it (a region shorter than the sampling
    interval still gets one)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 50

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []          # (host time, line)
        self.t0 = self.t1 = None
        self.thread = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.monotonic() + 5.0
            while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *a):
        self.t1 = time.monotonic()
        if self.proc is not None:
            deadline = self.t1 + 3.0 * self.INTERVAL_MS / 1e3 + 0.5
            while not any(t > self.t1 for t, _ in self.lines) and time.monotonic() < deadline \
                    and self.proc.poll() is None:
                time.sleep(0.01)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        inside = [ln for t, ln in self.lines if self.t0 <= t <= self.t1]
        after = [ln for t, ln in self.lines if t > self.t1][:1]
        rows = []
        for line in inside + after:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                rows.append((float(f[0]), float(f[1]), f[4], f[5], f[6], f[7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[2:]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["bf16_tflops_sustained"], p["hbm_gbs"], "measured"
    except Exception:
        return 1400.0, 6650.0, "fallback"


# DRAM traffic of the attention kernel from one ncu capture (dram__bytes_read.sum
# + dram__bytes_write.sum of k_attn_tc on the first 4 heads of the Wan-shaped
# workload: 278.3 + 63.5 = 341.9 MB, i.e. 85.5 MB per head; traffic grows with
# the heads).  The figure holds only for the kernel sources it was taken on,
# identified by hash (moved only over changes that left the device code as
# captured: comments and host-side code).
_ATTN_TRAFFIC = {"bytes_per_head": 341.860e6 / 4, "workload": "wan",
                 "sources": ("attn_tc.cu", "attn_tc.cuh", "tc_common.cuh"),
                 "sha1": "bd86ed4d39fdb3b58578bccfa9fbbdd4d2887eb7"}


def attn_traffic(cfg):
    """Per-launch DRAM bytes of k_attn_tc, or None when the capture does not
    apply (another workload, or kernel sources changed since)."""
    import hashlib
    if cfg.name != _ATTN_TRAFFIC["workload"]:
        return None
    h = hashlib.sha1()
    for f in _ATTN_TRAFFIC["sources"]:
        with open(os.path.join(ROOT, "clustered_sparse_attention_flash_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != _ATTN_TRAFFIC["sha1"]:
        return None
    return _ATTN_TRAFFIC["bytes_per_head"] * cfg.H


# ----------------------------------------------------------------- oracle

def _stratified(lq, C, n):
    """About n query rows spread over the query clusters: the first
    ceil(n / C) members of every non-empty cluster."""
    import numpy as np
    per = -(-n // C)
    return np.sort(np.concatenate([np.nonzero(lq == a)[0][:per] for a in range(C)]))


def oracle_sample(cfg, rho, q, k, v, iq, ik, key_frac=1, rows=1024):
    """Time the CPU oracle (float32 NumPy, multithreaded BLAS) on a bounded
    sample of one head and extrapolate to the whole layer: one k-means round
    of Q and of K (x iters), the final assignment, the permutation and value
    centroids, the block error on `key_frac` of the keys (all by default;
    scaled by 1 / key_frac), the routing, and the hybrid attention on `rows`
    query rows spread over the query clusters (scaled by N / rows); times H.
    Returns (extrapolated seconds per layer, description, stage seconds,
    measured seconds of the sample)."""
    import numpy as np
    from oracle import svgear_oracle as ora
    s = 1.0 / math.sqrt(cfg.d)
    t = {}
    w0 = time.perf_counter()
    with ora.timing_precision(np.float32):
        q, k, v, iq, ik = (np.asarray(x, dtype=np.float32) for x in (q, k, v, iq, ik))
        t0 = time.perf_counter()
        lab_q = ora.assign(q, iq); mu_q, _ = ora.update(q, lab_q, iq)
        t["kmeans_q_iter"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        lab_k = ora.assign(k, ik); mu_k, _ = ora.update(k, lab_k, ik)
        t["kmeans_k_iter"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        lq = ora.assign(q, mu_q); lk = ora.assign(k, mu_k)
        t["final_assign"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        pq, oq, cq = ora.permute(lq, cfg.Cq); pk, ok, ck = ora.permute(lk, cfg.Ck)
        Vbar = ora.value_centroids(v, lk, cfg.Ck)
        _ = (q[pq], k[pk], v[pk])
        t["permute"] = time.perf_counter() - t0
        nk = max(1, int(cfg.N * key_frac))
        t0 = time.perf_counter()
        E, M = ora.block_error(mu_q, mu_k, Vbar, k[:nk], v[:nk], lk[:nk], ck, s)
        t["block_error"] = (time.perf_counter() - t0) * cfg.N / nk
        t0 = time.perf_counter()
        mask, _, _ = ora.route(E, ck, cq, rho)
        t["route"] = time.perf_counter() - t0
        # attention time is linear in the rows plus a per-cluster cost (each
        # query cluster gathers its routed keys once): time one row per
        # cluster and the full sample, and extrapolate the line to N rows
        ta = []
        for n_rows in (cfg.Cq, rows):
            r = _stratified(lq, cfg.Cq, n_rows)
            lq_s = np.full_like(lq, -1)
            lq_s[r] = lq[r]
            t0 = time.perf_counter()
            ora.hybrid_attention(q, k, v, lq_s, lk, mu_k, Vbar, ck, mask, s)
            ta.append((r.size, time.perf_counter() - t0))
        (n1, t1), (n2, t2) = ta
        per_row = max(t2 - t1, 0.0) / max(n2 - n1, 1)
        t["attn"] = t1 + per_row * (cfg.N - n1)
    measured = time.perf_counter() - w0
    per_head = (cfg.iters * (t["kmeans_q_iter"] + t["kmeans_k_iter"]) + t["final_assign"]
                + t["permute"] + t["block_error"] + t["route"] + t["attn"])
    keys = "all keys" if nk == cfg.N else f"{nk} of {cfg.N} keys (x{cfg.N / nk:.2f})"
    desc = (f"oracle in float32 NumPy on head 0 ({measured:.1f} s measured): one k-means round of Q and "
            f"of K timed and x{cfg.iters}, final assignment, permutation and value centroids, block "
            f"error on {keys}, routing, hybrid attention on {n1} and on {n2} query rows spread over the "
            f"{cfg.Cq} query clusters (time extrapolated linearly to N rows); x {cfg.H} heads")
    return per_head * cfg.H, desc, t, measured


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else (os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def dense_flops(cfg):
    return 4.0 * cfg.H * cfg.N * cfg.N * cfg.d


def max_over_ranks(x, dist=None, device="cpu"):
    """The largest x over all ranks (the slowest rank's time); x itself with
    one process."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(cfg, world, ms):
    """Whole-job dense-equivalent TFLOP/s: every rank runs one full layer of
    cfg (weak scaling), timed by the slowest rank's ms per layer."""
    return world * dense_flops(cfg) / (ms / 1e3) / 1e12


def run_reference(a, cfg, rho):
    """The reference arm: the CPU oracle (float32 NumPy, the machine's host
    cores) on a bounded sample of the same workload per step, extrapolated
    to the layer.  The sample is sized so that warm-up + timed steps end
    within about three minutes; the line reports the measured sample time per
    step beside the extrapolated layer time."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from clustered_sparse_attention_flash_b200 import synth
    q, k, v, _ = synth.make_head(cfg, 0)
    iq = synth.forgy_init(cfg, q, 0, 0, cfg.Cq)
    ik = synth.forgy_init(cfg, k, 0, 1, cfg.Ck)
    n = a.warmup + a.steps
    # full sample (all keys, 1,024 rows) when few steps run; a quarter of the
    # keys and 256 rows per step otherwise
    key_frac, rows = (1, 1024) if n <= 6 else (0.25, 256)
    est_s, meas_s = [], []
    for i in range(n):
        est, desc, _, meas = oracle_sample(cfg, rho, q, k, v, iq, ik, key_frac=key_frac, rows=rows)
        if i >= a.warmup:
            est_s.append(est)
            meas_s.append(meas)
    layer_s = statistics.mean(est_s)
    val = dense_flops(cfg) / layer_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": layer_s * 1e3,
            "ms_per_step_basis": "extrapolated: each step times a bounded sample of one head and scales "
                                 "it to the whole layer (see cpu_baseline.sample)",
            "sample_ms_per_step_measured": statistics.mean(meas_s) * 1e3,
            "steps_timed": len(meas_s),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": _workload(cfg, rho)},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": _threads(), "kind": "oracle",
                             "sample": desc, "extrapolated": True},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------- head sharding

def run_shard_heads(a, cfg, rho):
    """One layer of cfg split by heads over the ranks (strong scaling): rank r
    runs heads head_range(H, world, r) through svgear_forward, then one NCCL
    all-gather assembles O [H, N, d] on every rank.  Both are inside the timed
    region; the time is the slowest rank's."""
    q_np, k_np, v_np, iq_np, ik_np = generate(cfg)   # before any CUDA call
    import torch
    from clustered_sparse_attention_flash_b200 import svgear as sv
    from clustered_sparse_attention_flash_b200.shard import forward_heads_sharded, head_range
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        dev = torch.device("cuda", local)
        tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        dQ, dK, dV = (torch.from_numpy(x).to(tdt).to(dev) for x in (q_np, k_np, v_np))
        iq, ik = torch.from_numpy(iq_np).to(dev), torch.from_numpy(ik_np).to(dev)
        s = 1.0 / math.sqrt(cfg.d)
        b, e = head_range(cfg.H, world, rank)
        p = sv.params(e - b, cfg.N, cfg.N, cfg.d, cfg.Cq, cfg.Ck, cfg.iters, rho, s,
                      sv.SVGEAR_BF16 if cfg.dtype == "bf16" else sv.SVGEAR_F32)
        ws = sv.workspace(sv.svgear_workspace_size(p), dev)
        stream = torch.cuda.current_stream(dev)

        def compute(q, k, v, Cq, Ck, iters, r, sc, iq_, ik_):
            O = torch.empty_like(q)
            sv.svgear_forward(q, k, v, p, iq_, ik_, O, ws, ws.numel(), stream)
            return O

        def step():
            return forward_heads_sharded(dQ, dK, dV, cfg.Cq, cfg.Ck, cfg.iters, rho, s, iq, ik,
                                         compute=compute)[0]

        for _ in range(a.warmup):
            step()
        torch.cuda.synchronize(dev)
        assert sv.svgear_get_status(stream) == sv.SVGEAR_OK
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        l0 = sv.svgear_launch_count()
        with Clocks(local) as clk:
            ev0.record(stream)
            for _ in range(a.steps):
                step()
            ev1.record(stream)
            torch.cuda.synchronize(dev)
        launches = sv.svgear_launch_count() - l0
        if dist is not None:
            dist.barrier()
        ms = max_over_ranks(ev0.elapsed_time(ev1) / a.steps, dist, dev)
        if rank == 0:
            line = {"metric": METRIC, "value": dense_flops(cfg) / (ms / 1e3) / 1e12, "unit": UNIT,
                    "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms,
                    "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": cfg.dtype,
                    "data": "synthetic",
                    "config": {"workload": _workload(cfg, rho),
                               "parallelism": f"heads sharded x{world} ({e - b} heads on rank 0), "
                                              f"all-gather of O over the process group"},
                    "gpu_launches": launches, "clocks": clk.summary()}
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ stress

def _dense_fp32(Q, K, V, scale, rows=4096):
    """softmax(s Q K^T) V per head in float32 (TF32 off), query rows chunked."""
    import torch
    O = torch.empty_like(Q)
    for h in range(Q.shape[0]):
        for r in range(0, Q.shape[1], rows):
            S = torch.matmul(Q[h, r:r + rows], K[h].T) * scale
            O[h, r:r + rows] = torch.matmul(torch.softmax(S, dim=-1), V[h])
    return O


def _nonincreasing(xs, slack=1.0):
    return all(b <= a * slack for a, b in zip(xs, xs[1:]))


def run_stress(a):
    """Relative L2 and max error of the operator's output against dense
    attention on the stress workload (H=16, N=32,768, d=128, Cq=64, Ck=512),
    for each within-center noise sigma and density budget rho, with the
    method's error-aware router, the two ablation signals, and the
    error-aware signal under one global budget per head.  The yardstick is
    float32 dense attention on the GPU; rows of it are checked in float64."""
    from clustered_sparse_attention_flash_b200 import synth
    base = synth.CONFIGS["stress"]
    if a.heads is not None:
        base = base.with_(H=a.heads)
    sigmas, rhos = synth.STRESS_SIGMAS, synth.STRESS_RHOS
    data = {sg: generate(base.with_(sigma=sg)) for sg in sigmas}   # before any CUDA call

    import numpy as np
    import torch
    from clustered_sparse_attention_flash_b200 import svgear as sv
    torch.backends.cuda.matmul.allow_tf32 = False
    torch.backends.cudnn.allow_tf32 = False
    dev = torch.device("cuda", 0)
    s = 1.0 / math.sqrt(base.d)
    G = sv.SVGEAR_BUDGET_GLOBAL
    routers = (("error", sv.SVGEAR_ROUTE_ERROR, 0), ("mass", sv.SVGEAR_ROUTE_MASS, 0),
               ("error_nov", sv.SVGEAR_ROUTE_ERROR_NOV, 0), ("error_global", sv.SVGEAR_ROUTE_ERROR, G))
    rows = []
    yard = {}
    t0 = time.perf_counter()
    for sg in sigmas:
        q, k, v, iq, ik = data[sg]
        dQ, dK, dV = (torch.from_numpy(x).to(dev).to(torch.bfloat16) for x in (q, k, v))
        diq, dik = torch.from_numpy(iq).to(dev), torch.from_numpy(ik).to(dev)
        Of = [x.float() for x in (dQ, dK, dV)]
        ref = _dense_fp32(*Of, s)
        # the yardstick against float64 on 256 rows of head 0
        r64 = torch.softmax(torch.matmul(Of[0][0, :256].double(), Of[1][0].double().T) * s, dim=-1) @ Of[2][0].double()
        yard[sg] = float((ref[0, :256].double() - r64).abs().max())
        nref = float(torch.linalg.vector_norm(ref.double()))
        ws = None
        for rname, rcode, bcode in routers:
            for rho in rhos:
                O, ws, p, st = sv.forward(dQ, dK, dV, base.Cq, base.Ck, base.iters, rho, s, diq, dik,
                                          ws=ws, stats=True, router=rcode, budget=bcode)
                if sv.svgear_get_status() != sv.SVGEAR_OK:
                    raise RuntimeError("device status not OK")
                d = O.float() - ref
                rows.append({"sigma": sg, "rho": rho, "router": rname,
                             "rel_l2": float(torch.linalg.vector_norm(d.double())) / nref,
                             "max_abs": float(d.abs().max()),
                             "density": st["exec_pairs"] / (base.H * base.N * base.N),
                             "ms": st["ms_total"]})
        del dQ, dK, dV, Of, ref
        torch.cuda.empty_cache()

    def err(sg, rho, r="error"):
        return next(x["rel_l2"] for x in rows if x["sigma"] == sg and x["rho"] == rho and x["router"] == r)

    trends = {
        # error against dense must not fall as the noise grows (fixed rho) ...
        "nondecreasing_in_sigma": {str(rho): _nonincreasing([err(sg, rho) for sg in sigmas][::-1])
                                   for rho in rhos},
        # ... and must not rise as the budget grows (fixed sigma)
        "nonincreasing_in_rho": {str(sg): _nonincreasing([err(sg, rho) for rho in rhos]) for sg in sigmas},
        "error_router_best": {f"{sg}/{rho}": min(("error", "mass", "error_nov"), key=lambda r: err(sg, rho, r))
                              for sg in sigmas for rho in rhos if rho < 1.0},
        "global_budget_better": {f"{sg}/{rho}": err(sg, rho, "error_global") < err(sg, rho)
                                 for sg in sigmas for rho in rhos if rho < 1.0},
    }
    line = {"stress": True, "workload": _workload(base, "swept"), "sigmas": sigmas, "rhos": rhos,
            "yardstick": "float32 dense attention on the GPU (TF32 off) from the same bf16 inputs",
            "yardstick_max_abs_vs_float64_256_rows": yard, "results": rows, "trends": trends,
            "seconds": time.perf_counter() - t0}
    print(json.dumps(line), flush=True)
    for r in rows:
        print(f"sigma {r['sigma']:<5} rho {r['rho']:<5} {r['router']:<12} rel_l2 {r['rel_l2']:.4e} "
              f"max {r['max_abs']:.4e} density {r['density']:.4f} {r['ms']:.2f} ms", file=sys.stderr)
    return 0


# -------------------------------------------------------------------- ours

def main():
    a = _args()
    if a.stress:
        return run_stress(a)
    from clustered_sparse_attention_flash_b200 import synth
    cfg = synth.CONFIGS[a.config]
    if a.heads is not None:
        cfg = cfg.with_(H=a.heads)
    rho = cfg.rho if a.rho is None else a.rho
    if a.impl == "reference":
        return run_reference(a, cfg, rho)
    if a.shard_heads:
        return run_shard_heads(a, cfg, rho)
    assert a.warmup >= 3, "at least 3 warm-up steps"

    q_np, k_np, v_np, iq_np, ik_np = generate(cfg)   # before any CUDA call

    import numpy as np
    import torch
    from clustered_sparse_attention_flash_b200 import svgear as sv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    dev = torch.device("cuda", local)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    Q = torch.from_numpy(q_np).to(tdt).pin_memory()
    K = torch.from_numpy(k_np).to(tdt).pin_memory()
    V = torch.from_numpy(v_np).to(tdt).pin_memory()
    dQ, dK, dV = Q.to(dev), K.to(dev), V.to(dev)
    iq, ik = torch.from_numpy(iq_np).to(dev), torch.from_numpy(ik_np).to(dev)
    dO = torch.empty_like(dQ)
    hO = torch.empty_like(Q).pin_memory()
    s = 1.0 / math.sqrt(cfg.d)
    p = sv.params(cfg.H, cfg.N, cfg.N, cfg.d, cfg.Cq, cfg.Ck, cfg.iters, rho, s,
                  sv.SVGEAR_BF16 if cfg.dtype == "bf16" else sv.SVGEAR_F32)
    ws = sv.workspace(sv.svgear_workspace_size(p), dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        sv.svgear_forward(dQ, dK, dV, p, iq, ik, dO, ws, ws.numel(), stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert sv.svgear_get_status(stream) == sv.SVGEAR_OK

    # ---- timed region: K steps on inputs resident in HBM
    props = torch.cuda.get_device_properties(dev)
    gpu_id = getattr(props, "uuid", None)
    gpu_id = f"GPU-{gpu_id}" if gpu_id is not None and not str(gpu_id).startswith("GPU-") else (gpu_id or local)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    l0 = sv.svgear_launch_count()
    with Clocks(gpu_id) as clk:
        ev0.record(stream)
        for _ in range(a.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    launches = sv.svgear_launch_count() - l0
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / a.steps, dist, dev)
    clocks = clk.summary()

    # ---- per-stage breakdown (library-internal CUDA events on the same stream)
    stats = []
    for _ in range(a.steps):
        st = sv.svgear_stats()
        sv.svgear_forward(dQ, dK, dV, p, iq, ik, dO, ws, ws.numel(), stream, st)
        stats.append(st.as_dict())
    avg = {k2: statistics.mean(x[k2] for x in stats) for k2 in stats[0]}
    exec_pairs, comp_pairs = avg["exec_pairs"], avg["comp_pairs"]
    # Everything before the attention stage; the two clusterings overlap, so
    # their stage times are not added.
    routing_ms = avg["ms_total"] - avg["ms_attn"]

    # ---- end to end: pinned host buffers in, result back to host, every step
    e2e = None
    if not a.no_e2e:
        # Pinned host Q, K, V in and O back every step, through the same C
        # entry point.  Two device buffer sets and three streams: the host
        # copies of one step overlap the layer of the neighbouring step, as a
        # serving loop would run it; each step still moves its own inputs in
        # and its own output out inside the timed region.
        sets = [(dQ, dK, dV, dO), tuple(torch.empty_like(x) for x in (dQ, dK, dV, dO))]
        hOs = [hO, torch.empty_like(hO).pin_memory()]
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        h2d_done = [torch.cuda.Event(), torch.cuda.Event()]
        fwd_done = [torch.cuda.Event(), torch.cuda.Event()]
        d2h_done = [torch.cuda.Event(), torch.cuda.Event()]

        def e2e_step(i):
            b = i & 1
            q, k, v, o = sets[b]
            s_in.wait_event(fwd_done[b])          # set b's inputs read by the layer two steps back
            with torch.cuda.stream(s_in):
                q.copy_(Q, non_blocking=True); k.copy_(K, non_blocking=True); v.copy_(V, non_blocking=True)
            h2d_done[b].record(s_in)
            s_cmp.wait_event(h2d_done[b])
            s_cmp.wait_event(d2h_done[b])         # set b's output read back two steps back
            sv.svgear_forward(q, k, v, p, iq, ik, o, ws, ws.numel(), s_cmp)
            fwd_done[b].record(s_cmp)
            s_out.wait_event(fwd_done[b])
            with torch.cuda.stream(s_out):
                hOs[b].copy_(o, non_blocking=True)
            d2h_done[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        # The window spans at least 10 steps: it opens with the first step's
        # input copy and closes with the last step's output copy, so one
        # layer and one output copy are not overlapped; over more steps that
        # fill and drain weigh less, as in a serving loop that keeps running.
        n_e2e = max(a.steps, 10)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        s_in.wait_event(d2h_done[0]); s_in.wait_event(d2h_done[1])
        e1.record(s_in)
        torch.cuda.synchronize(dev)
        assert sv.svgear_get_status(s_cmp) == sv.SVGEAR_OK
        ems = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist, dev)
        bi = 3 * Q.numel() * Q.element_size()
        bo = hO.numel() * hO.element_size()
        e2e = {"value": job_value(cfg, world, ems), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": ems, "steps": n_e2e,
               "overlap": "H2D of step i+1 and D2H of step i-1 run beside the layer of step i "
                          "(separate streams, two device buffer sets)"}

    peak_tc, peak_hbm, peak_src = _peaks()
    attn_flops = 4.0 * cfg.d * (exec_pairs + comp_pairs)
    achieved = attn_flops / (avg["ms_attn_kernel"] / 1e3) / 1e12
    roofline = {"kernel": "hybrid attention (svgear_hybrid_attn)", "bound": "tensor",
                "achieved": achieved, "peak": peak_tc, "unit": "TFLOP/s", "frac": achieved / peak_tc,
                "traffic": attn_traffic(cfg),
                "ms_per_launch": avg["ms_attn_kernel"],
                "note": f"algorithmic 4*d*(executed + compensated pairs) per launch over the attention "
                        f"kernel's CUDA-event time (its staging kernels excluded; they are in "
                        f"stage_ms.ms_attn); peak = {peak_src} sustained dense bf16; traffic = DRAM "
                        f"bytes per launch from an ncu capture of 4 heads, scaled by heads"}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        sec, desc, stages, meas = oracle_sample(cfg, rho, q_np[0], k_np[0], v_np[0], iq_np[0], ik_np[0])
        cpu = {"value": dense_flops(cfg) / sec / 1e12, "unit": UNIT, "cores": _threads(),
               "kind": "oracle", "sample": desc, "extrapolated": True, "layer_s_extrapolated": sec,
               "sample_s_measured": meas, "stage_s_per_head": stages}

    value = job_value(cfg, world, ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": _workload(cfg, rho),
                   "l2": "inputs (3 x %.2f GB) larger than the 126 MB L2; no flush" % (Q.numel() * Q.element_size() / 1e9),
                   "parallelism": f"replicas x{world} (heads independent; no data-path collective)"},
        "layer_ms": ms,
        "exec_pair_tflops": 4.0 * cfg.d * exec_pairs / (avg["ms_attn"] / 1e3) / 1e12,
        "exec_pair_frac_of_peak": (4.0 * cfg.d * exec_pairs / (avg["ms_attn"] / 1e3) / 1e12) / peak_tc,
        "routing_overhead_pct": 100.0 * routing_ms / avg["ms_total"],
        "routing_overhead_excl_kmeans_pct": 100.0 * (avg["ms_permute"] + avg["ms_block_error"] + avg["ms_route"]) / avg["ms_total"],
        "stage_ms": {k2: avg[k2] for k2 in ("ms_kmeans_q", "ms_kmeans_k", "ms_permute", "ms_block_error",
                                            "ms_route", "ms_attn", "ms_attn_kernel", "ms_total")},
        "density": exec_pairs / (cfg.H * cfg.N * cfg.N),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "gpu_launches_per_step": launches / a.steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
