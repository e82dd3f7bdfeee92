"""svgear_block_error_noalloc: the block-error entry point for callers that
cannot allocate device memory when they call the operator (a runtime with a
fixed memory plan, a plug-in inside a framework that owns the allocator).  It
keeps its scratch in a device array of the library, so it must give the same
errors as svgear_block_error with a caller workspace -- on every call, with the
array still holding the previous call's contents.

This file is collected last on purpose: a failure here leaves every other
test already run."""
import ctypes
import math

import numpy as np
import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from clustered_sparse_attention_flash_b200 import synth
from oracle import svgear_oracle as ora

from helpers import E_FLOOR, E_RTOL  # the block-error tolerance of the parity tests


def _intermediates(cfg, heads):
    """Run the operator once and return device tensors that feed block error."""
    import torch
    q, k, v = synth.make_inputs(cfg, heads)
    H = len(heads)
    iq = np.stack([synth.forgy_init(cfg, q[i], h, 0, cfg.Cq) for i, h in enumerate(heads)])
    ik = np.stack([synth.forgy_init(cfg, k[i], h, 1, cfg.Ck) for i, h in enumerate(heads)])
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    dq, dk, dv = (torch.from_numpy(x).to(tdt).cuda() for x in (q, k, v))
    _, ws, p, _ = sv.forward(dq, dk, dv, cfg.Cq, cfg.Ck, cfg.iters, cfg.rho, 1 / math.sqrt(cfg.d),
                             torch.from_numpy(iq).cuda(), torch.from_numpy(ik).cuda())
    torch.cuda.synchronize()
    return ws, p, sv.view_tensors(p, ws)


def _both(p, vw):
    """E, M from the workspace entry point and from the allocation-free one."""
    import torch
    H, Cq, Ck = p.H, p.Cq, p.Ck
    args = (vw["cent_q"], vw["cent_k"], vw["vbar"], vw["Kp"], vw["Vp"], vw["off_k"], vw["key_scalars"])
    E1 = torch.empty((H, Cq, Ck), dtype=torch.float32, device="cuda")
    M1 = torch.empty((H, Cq), dtype=torch.float32, device="cuda")
    ws = sv.workspace(sv.svgear_block_error_workspace_size(p))
    sv.svgear_block_error(*args, p, E1, M1, ws, ws.numel())
    E2 = torch.full_like(E1, float("nan"))
    M2 = torch.full_like(M1, float("nan"))
    sv.svgear_block_error_noalloc(*args, p, E2, M2)
    torch.cuda.synchronize()
    assert sv.svgear_get_status() == sv.SVGEAR_OK
    return [t.cpu().numpy() for t in (E1, M1, E2, M2)]


def _oracle_error(p, vw, i):
    """Oracle E and its floor scale T for head i, from the same intermediates
    (keys in cluster order; the label of a key follows from the offsets)."""
    f = lambda name: vw[name][i].float().cpu().numpy().astype(np.float64)
    off = vw["off_k"][i].cpu().numpy()
    counts = np.diff(off)
    labels = np.repeat(np.arange(p.Ck), counts)
    args = (f("cent_q"), f("cent_k"), f("vbar"), f("Kp"), f("Vp"), labels, counts, 1 / math.sqrt(p.d))
    return ora.block_error(*args)[0], ora.block_error_scale(*args)


@pytest.mark.gpu
def test_noalloc_block_error_matches_workspace_version_twice():
    """Both entry points within the parity tolerance of the oracle
    (|E - E_oracle| <= E_RTOL |E_oracle| + E_FLOOR T), and so within twice
    that of each other; the row shifts M agree to float rounding."""
    cases = [synth.CONFIGS["mid"].with_(H=2), synth.CONFIGS["wan"].with_(H=1)]
    heads = [(0, 3), (0,)]
    for cfg, hs in zip(cases, heads):
        _, p, vw = _intermediates(cfg, hs)
        E1, M1, E2, M2 = _both(p, vw)
        assert np.isfinite(E2).all() and np.isfinite(M2).all()
        for i in range(len(hs)):
            Eo, T = _oracle_error(p, vw, i)
            lim = E_RTOL * np.abs(Eo) + E_FLOOR * T
            assert (np.abs(E1[i] - Eo) <= lim).all()
            assert (np.abs(E2[i] - Eo) <= lim).all()
            assert (np.abs(E2[i] - E1[i]) <= 2 * lim).all()
        assert (np.abs(M2 - M1) <= 1e-6 * np.maximum(np.abs(M1), 1.0)).all()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """H * Cq * Ck above 2,097,152 is refused before anything is enqueued."""
    L = sv.lib()
    p = sv.params(40, 75600, 75600, 128, 100, 600, 10, 0.15)  # 2.4M > limit
    fake = 256  # aligned non-null pointers: validation only, nothing runs
    rc = L.svgear_block_error_noalloc(fake, fake, fake, fake, fake, fake, fake, ctypes.byref(p),
                                      fake, fake, None)
    assert rc == sv.SVGEAR_ERR_WORKSPACE
