"""bench.py's host-side helpers, no GPU: the DRAM-traffic figure is reported
only for the workload and kernel sources it was captured on, the stress
sweep's trend test, the workload description, the generator's configuration
override, the clock sampler (against a stand-in nvidia-smi), and the CPU
oracle legs: the reference arm's JSON line and the sampled extrapolation."""
import hashlib
import os

import numpy as np
import pytest

import bench
from clustered_sparse_attention_flash_b200 import synth


def _sources_hash():
    h = hashlib.sha1()
    for f in bench._ATTN_TRAFFIC["sources"]:
        with open(os.path.join(bench.ROOT, "clustered_sparse_attention_flash_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def test_attention_traffic_only_for_its_capture():
    wan = synth.CONFIGS["wan"]
    assert bench.attn_traffic(synth.CONFIGS["stress"]) is None
    t = bench.attn_traffic(wan)
    if _sources_hash() == bench._ATTN_TRAFFIC["sha1"]:
        assert t == pytest.approx(bench._ATTN_TRAFFIC["bytes_per_head"] * wan.H)
        assert bench.attn_traffic(wan.with_(H=4)) == pytest.approx(341.860e6)
    else:
        assert t is None


def test_trend_helper():
    assert bench._nonincreasing([3.0, 2.0, 2.0, 1.0])
    assert not bench._nonincreasing([1.0, 2.0])
    assert bench._nonincreasing([])
    assert bench._nonincreasing([1.0, 1.0 + 1e-9], slack=1.0 + 1e-6)


def test_workload_names_sizes():
    w = bench._workload(synth.CONFIGS["wan"], 0.15)
    for part in ("H=40", "N=75600", "21x45x80", "d=128", "Cq=100", "Ck=500", "rho=0.15"):
        assert part in w


def test_generator_honours_the_config_it_is_given():
    """The stress sweep overrides sigma; each head must be generated from the
    overridden configuration, not the registered one."""
    base = synth.CONFIGS["tiny"]
    a = bench._gen_head((base.with_(sigma=0.1), 0))
    b = bench._gen_head((base.with_(sigma=1.0), 0))
    c = bench._gen_head((base.with_(sigma=1.0), 0))
    assert not np.array_equal(a[0], b[0])
    for x, y in zip(b, c):
        np.testing.assert_array_equal(x, y)
    assert a[3].shape == (base.Cq, base.d) and a[4].shape == (base.Ck, base.d)


def test_clock_sampler_covers_a_short_region(tmp_path, monkeypatch):
    # A stand-in nvidia-smi that starts slowly and then prints one CSV sample
    # every 50 ms; a region much shorter than the start-up still gets samples
    # and the throttle reasons are read from the right columns.
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nsleep 0.3\nwhile true; do\n"
                    "  echo '1965, 1965, 700.5, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "  sleep 0.05\ndone\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ.get('PATH', '')}")
    import time
    with bench.Clocks(0) as clk:
        time.sleep(0.02)
    out = clk.summary()
    assert out["samples"] >= 1
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    with bench.Clocks(0) as clk:
        pass
    assert clk.summary()["reasons"] == ["unavailable"]


def test_reference_arm_runs_on_the_host():
    # `bench.py --impl reference` times the oracle on the host cores only:
    # one JSON line with the reference fields, no GPU needed (tiny workload).
    import json
    import subprocess
    import sys
    env = dict(os.environ, RANK="0")
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, env=env, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["dtype"] == "f32"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["steps_timed"] == 1 and d["sample_ms_per_step_measured"] > 0


def test_reference_arm_other_ranks_exit_quietly():
    import subprocess
    import sys
    env = dict(os.environ, RANK="1")
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=bench.ROOT)
    assert out.returncode == 0 and not out.stdout.strip()


def test_oracle_sample_extrapolates_every_stage():
    cfg = synth.CONFIGS["tiny"]
    q, k, v, _ = synth.make_head(cfg, 0)
    iq = synth.forgy_init(cfg, q, 0, 0, cfg.Cq)
    ik = synth.forgy_init(cfg, k, 0, 1, cfg.Ck)
    sec, desc, stages, meas = bench.oracle_sample(cfg, cfg.rho, q, k, v, iq, ik, rows=256)
    assert sec > 0 and meas > 0 and "float32" in desc
    for key in ("kmeans_q_iter", "kmeans_k_iter", "final_assign", "permute", "block_error", "route", "attn"):
        assert stages[key] >= 0, key
    # the layer estimate covers every stage of every head
    assert sec >= cfg.H * (stages["block_error"] + stages["attn"])
