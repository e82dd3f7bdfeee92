"""Shared helpers for the GPU parity tests: seeded cases, device transfer and
the comparison rules (tolerances are those the operator's spec states)."""
from __future__ import annotations

import functools
import math

import numpy as np

from clustered_sparse_attention_flash_b200 import svgear as sv
from clustered_sparse_attention_flash_b200 import synth
from oracle import svgear_oracle as ora

# output tolerance |gpu - ref| <= ATOL + RTOL * |ref|
OUT_TOL = {"f32": (1e-4, 1e-4), "bf16": (1e-2, 1e-2)}
E_RTOL, E_FLOOR = 1e-3, 1e-6       # block error: 1e-3 relative, floor 1e-6 * T
TIE_REL = 1e-4                     # near-tie exemption for labels / routing


def torch_dtype(cfg):
    import torch
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def dev(x, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    import torch
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


class Case:
    """Seeded inputs of a config restricted to a few heads."""

    def __init__(self, cfg, heads, rho=None):
        self.cfg = cfg
        self.heads = list(heads)
        self.H = len(self.heads)
        self.rho = cfg.rho if rho is None else rho
        self.q, self.k, self.v = synth.make_inputs(cfg, self.heads)
        self.init_q = np.stack([synth.forgy_init(cfg, self.q[i], h, 0, cfg.Cq) for i, h in enumerate(self.heads)])
        self.init_k = np.stack([synth.forgy_init(cfg, self.k[i], h, 1, cfg.Ck) for i, h in enumerate(self.heads)])
        self.scale = 1.0 / math.sqrt(cfg.d)

    def params(self, **kw):
        c = self.cfg
        d = dict(H=self.H, Nq=c.N, Nk=c.N, d=c.d, Cq=c.Cq, Ck=c.Ck, iters=c.iters, rho=self.rho,
                 scale=self.scale, dtype=sv.SVGEAR_BF16 if c.dtype == "bf16" else sv.SVGEAR_F32)
        d.update(kw)
        return sv.params(**d)

    def dq(self):
        return dev(self.q, torch_dtype(self.cfg))

    def dk(self):
        return dev(self.k, torch_dtype(self.cfg))

    def dv(self):
        return dev(self.v, torch_dtype(self.cfg))

    @functools.cached_property
    def oracle(self):
        """Full oracle forward per head (float64)."""
        c = self.cfg
        return [ora.forward(self.q[i], self.k[i], self.v[i], c.Cq, c.Ck, c.iters, self.rho,
                            self.scale, self.init_q[i], self.init_k[i]) for i in range(self.H)]


@functools.lru_cache(maxsize=None)
def case(name, heads=None, rho=None):
    cfg = synth.CONFIGS[name]
    if heads is None:
        heads = (0,) if cfg.H == 1 else (0, 5)
    return Case(cfg, heads, rho)


def assert_close(got, ref, atol, rtol, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    lim = atol + rtol * np.abs(ref)
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} (atol {atol}, rtol {rtol})")


def label_mismatches_are_ties(X, mu, gpu_labels):
    """Every label that differs from the float64 argmin must be a near-tie
    ((d2 - d1) / d2 < TIE_REL).  Returns the number of differing labels."""
    lab, d1, d2 = ora.assign_margin(X, mu)
    diff = np.nonzero(lab != gpu_labels)[0]
    if diff.size:
        gap = (d2[diff] - d1[diff]) / np.maximum(d2[diff], 1e-300)
        assert (gap < TIE_REL).all(), (f"{int((gap >= TIE_REL).sum())} labels differ from the exact "
                                      f"argmin at non-tied points, e.g. index {diff[gap >= TIE_REL][:5]}")
    return int(diff.size)
