"""The forward runs its query clustering on a second stream of its own, forked
from the caller's stream and joined back before the block error.  These tests
check that the caller still sees stream-ordered work: on a non-default stream,
back to back on one workspace with no host synchronisation between the calls,
and recorded into a CUDA graph and replayed.  The forward is deterministic
(integer atomics only, stable counting sort), so every comparison is bitwise."""
import numpy as np
import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from helpers import case, dev, host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _inputs(name, seed_shift=0):
    cs = case(name)
    if seed_shift:
        # A second, different input set of the same shapes: the keys of one
        # case as the queries of the other and so on (rows stay 16-byte aligned).
        return cs, (cs.dk(), cs.dv(), cs.dq())
    return cs, (cs.dq(), cs.dk(), cs.dv())


def _eager(cs, qkv):
    cfg = cs.cfg
    O, ws, p, _ = sv.forward(*qkv, cfg.Cq, cfg.Ck, cfg.iters, cs.rho, cs.scale, dev(cs.init_q), dev(cs.init_k))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    return host(O), p


def test_forward_on_a_side_stream_back_to_back_on_one_workspace():
    cs, a = _inputs("mid")
    _, b = _inputs("mid", seed_shift=1)
    ref_a, p = _eager(cs, a)
    ref_b, _ = _eager(cs, b)
    assert not np.array_equal(ref_a, ref_b)
    cfg = cs.cfg
    ws = sv.workspace(sv.svgear_workspace_size(p))
    Oa, Ob = torch.empty_like(a[0]), torch.empty_like(b[0])
    iq, ik = dev(cs.init_q), dev(cs.init_k)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # Same workspace, no host synchronisation: the second call's query
        # clustering must not start before the first call's attention is done.
        sv.svgear_forward(*a, p, iq, ik, Oa, ws, ws.numel(), s.cuda_stream, None)
        sv.svgear_forward(*b, p, iq, ik, Ob, ws, ws.numel(), s.cuda_stream, None)
    s.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    np.testing.assert_array_equal(host(Oa), ref_a)
    np.testing.assert_array_equal(host(Ob), ref_b)


def test_forward_recorded_in_a_cuda_graph_replays_the_eager_result():
    cs, a = _inputs("mid")
    _, b = _inputs("mid", seed_shift=1)
    ref_a, p = _eager(cs, a)
    ref_b, _ = _eager(cs, b)
    ws = sv.workspace(sv.svgear_workspace_size(p))
    iq, ik = dev(cs.init_q), dev(cs.init_k)
    Qs, Ks, Vs = (x.clone() for x in a)
    O = torch.empty_like(Qs)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # One eager call first: the library sets its kernels' attributes and
        # creates its second stream outside the capture.
        sv.svgear_forward(Qs, Ks, Vs, p, iq, ik, O, ws, ws.numel(), s.cuda_stream, None)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sv.svgear_forward(Qs, Ks, Vs, p, iq, ik, O, ws, ws.numel(), s.cuda_stream, None)
    for src, ref in ((a, ref_a), (b, ref_b), (a, ref_a)):
        for dst, x in zip((Qs, Ks, Vs), src):
            dst.copy_(x)
        O.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert sv.svgear_get_status() == sv.SVGEAR_OK
        np.testing.assert_array_equal(host(O), ref)
    del g
