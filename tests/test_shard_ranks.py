"""Head-sharded forward on CPU (gloo): the head partition covers every head
once in contiguous slices, and two ranks that each compute their slice and
all-gather the result hold exactly the single-process output.  The per-slice
compute here is the CPU oracle (no GPU); on GPUs it is svgear_forward."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
H, N, D, CQ, CK, ITERS, RHO = 5, 300, 32, 4, 9, 3, 0.3


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(heads=H):
    rng = np.random.default_rng(17)
    q, k, v = (rng.standard_normal((heads, N, D)) for _ in range(3))
    return q, k, v, q[:, :CQ].copy(), k[:, :CK].copy()


def _oracle_compute(Q, K, V, Cq, Ck, iters, rho, scale, iq, ik):
    import torch
    from oracle import svgear_oracle as ora
    outs = [ora.forward(Q[i].numpy(), K[i].numpy(), V[i].numpy(), Cq, Ck, iters, rho, scale,
                        iq[i].numpy(), ik[i].numpy())["O"] for i in range(Q.shape[0])]
    return torch.from_numpy(np.stack(outs)) if outs else torch.empty((0,) + tuple(Q.shape[1:]), dtype=Q.dtype)


def _rank(rank, world, port, out, heads=H):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from clustered_sparse_attention_flash_b200.shard import forward_heads_sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, iq, ik = (torch.from_numpy(x) for x in _inputs(heads))
        O, hr = forward_heads_sharded(q, k, v, CQ, CK, ITERS, RHO, 1 / np.sqrt(D), iq, ik,
                                      compute=_oracle_compute)
        part, _ = forward_heads_sharded(q, k, v, CQ, CK, ITERS, RHO, 1 / np.sqrt(D), iq, ik,
                                        compute=_oracle_compute, gather=False)
        out.put((rank, hr, O.numpy(), part.numpy()))
    finally:
        dist.destroy_process_group()


def test_head_partition():
    from clustered_sparse_attention_flash_b200.shard import head_range
    for Hh in (1, 5, 24, 40):
        for world in (1, 2, 3, 8):
            ranges = [head_range(Hh, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == Hh
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [e - b for b, e in ranges]
            assert max(sizes) - min(sizes) <= 1 and sorted(sizes, reverse=True) == sizes
    assert head_range(40, 8, 3) == (15, 20)
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def test_two_ranks_gather_the_single_process_output():
    import torch
    sys.path.insert(0, ROOT)
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q_)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q_.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, iq, ik = (torch.from_numpy(x) for x in _inputs())
    want = _oracle_compute(q, k, v, CQ, CK, ITERS, RHO, 1 / np.sqrt(D), iq, ik).numpy()
    assert [r[1] for r in res] == [(0, 3), (3, 5)]
    for rank, (b, e), O, part in res:
        np.testing.assert_array_equal(O, want)
        np.testing.assert_array_equal(part, want[b:e])


def test_more_ranks_than_heads():
    # one head over two ranks: rank 1 owns no head, computes nothing and still
    # takes part in the all-gather
    import torch
    sys.path.insert(0, ROOT)
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q_, 1)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q_.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, iq, ik = (torch.from_numpy(x) for x in _inputs(1))
    want = _oracle_compute(q, k, v, CQ, CK, ITERS, RHO, 1 / np.sqrt(D), iq, ik).numpy()
    assert [r[1] for r in res] == [(0, 1), (1, 1)]
    for rank, (b, e), O, part in res:
        np.testing.assert_array_equal(O, want)
        assert part.shape[0] == e - b
