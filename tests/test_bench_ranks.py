"""bench.py's multi-rank bookkeeping on CPU (gloo, two ranks): every rank
sees the slowest rank's time, and the job value counts the work of all
ranks over that time (weak scaling)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, times, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from clustered_sparse_attention_flash_b200 import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], dist, "cpu")
        cfg = synth.CONFIGS["wan"]
        out.put((rank, ms, bench.job_value(cfg, world, ms)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    import bench
    from clustered_sparse_attention_flash_b200 import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [40.0, 55.5]
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = synth.CONFIGS["wan"]
    for rank, ms, value in res:
        assert ms == 55.5
        assert value == pytest.approx(2 * 4.0 * cfg.H * cfg.N * cfg.N * cfg.d / 55.5e-3 / 1e12)
    # one process: the value is one layer over its own time
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_value(cfg, 1, 12.5) == pytest.approx(bench.dense_flops(cfg) / 12.5e-3 / 1e12)
