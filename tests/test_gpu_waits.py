"""Failure detection without a GPU fault: a bounded in-kernel wait on a
barrier that nothing completes gives up after a short limit, the kernel
returns, svgear_get_status reports the timeout, and the context stays usable
(the next operator call runs clean and matches the oracle)."""
import math
import time

import numpy as np
import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from oracle import svgear_oracle as ora

from helpers import OUT_TOL, assert_close, dev, host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_next_call_is_clean():
    assert sv.svgear_get_status() in (sv.SVGEAR_OK, sv.SVGEAR_ERR_TIMEOUT)  # start from a clear word
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    t0 = time.monotonic()
    sv.svgear_selftest_wait(2_000_000)          # 2 ms
    assert sv.svgear_get_status() == sv.SVGEAR_ERR_TIMEOUT
    assert time.monotonic() - t0 < 10.0
    assert sv.svgear_get_status() == sv.SVGEAR_OK   # reading cleared the word
    # the context is usable: a small forward runs clean and matches the oracle
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((1, 600, 64)).astype(np.float32) for _ in range(3))
    s = 1 / math.sqrt(64)
    iq, ik = q[:, :5].copy(), k[:, :9].copy()
    O, _, _, _ = sv.forward(dev(q), dev(k), dev(v), 5, 9, 3, 0.3, s, dev(iq), dev(ik))
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    o = ora.forward(q[0], k[0], v[0], 5, 9, 3, 0.3, s, iq[0], ik[0])
    assert_close(host(O)[0], o["O"], *OUT_TOL["f32"], "forward after a timed-out wait")


def test_selftest_rejects_out_of_range_limits():
    for bad in (0, 999, 2_000_000_000):
        with pytest.raises(sv.SvgearError):
            sv.svgear_selftest_wait(bad)
