"""Seeded synthetic inputs for the SVG-EAR operator.

This module only draws random numbers.  It holds none of the operator's
arithmetic, so both the CUDA path and the CPU oracle may take their inputs from
it without sharing any computation.

Workloads are shaped like the attention layers of the video DiTs the SVG-EAR
pages evaluate (Wan2.2, HunyuanVideo at 720p): tokens live on a
(frames, height, width) latent grid in raster order, and every token's
q/k/v is a latent "center" vector plus isotropic noise.  Centers are spatially
smooth (a token takes the center of the coarse voxel it falls in) with 10 % of
tokens reassigned to a uniformly random center, which gives the clustered,
mostly local structure that semantic k-means exploits.

Per head h the generator is ``numpy.random.default_rng([seed, h])`` with
``seed = 20260 + config index``; draws happen in a fixed order (centers q, k,
v; token-to-center map; noise q, k, v) so every head is reproducible on its own.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np

__all__ = ["Config", "CONFIGS", "make_head", "make_inputs", "forgy_init",
           "logit_alpha", "to_bf16_f32"]


@dataclasses.dataclass(frozen=True)
class Config:
    """One synthetic workload (all sizes per layer)."""
    name: str
    index: int                       # seed = 20260 + index
    H: int                           # heads
    N: int                           # tokens (N_q = N_k)
    d: int                           # head dim
    dtype: str                       # "f32" or "bf16"
    G: int                           # latent centers
    sigma: float                     # within-center noise std
    Cq: int
    Ck: int
    iters: int
    rho: float
    grid: Optional[Tuple[int, int, int]] = None    # (T, Hh, W) token grid
    vox: Optional[Tuple[int, int, int]] = None     # voxel grid, product G
    scale_logits: bool = True        # rescale q, k so q.k/sqrt(d) has std ~2
    reassign: float = 0.10           # fraction of tokens with a random center

    @property
    def seed(self) -> int:
        return 20260 + self.index

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, Config] = {
    # 1 head, N=4096, d=64, fp32; 32 centers, uniform center choice, sigma 0.35
    "tiny": Config("tiny", 0, H=1, N=4096, d=64, dtype="f32", G=32, sigma=0.35,
                   Cq=16, Ck=64, iters=10, rho=0.25, scale_logits=False,
                   reassign=0.0),
    # 8 heads, 16x32x32 grid, d=128, bf16, 256 centers on a 4x8x8 voxel grid
    "mid": Config("mid", 1, H=8, N=16384, d=128, dtype="bf16", G=256,
                  sigma=0.35, Cq=64, Ck=256, iters=10, rho=0.25,
                  grid=(16, 32, 32), vox=(4, 8, 8)),
    # Wan2.2-shaped: 40 heads, 21x45x80 grid (75,600 tokens), 1024 centers
    "wan": Config("wan", 2, H=40, N=75600, d=128, dtype="bf16", G=1024,
                  sigma=0.35, Cq=100, Ck=500, iters=10, rho=0.15,
                  grid=(21, 45, 80), vox=(4, 16, 16)),
    # HunyuanVideo-shaped: 24 heads, 33x45x80 grid (118,800 tokens), 1536 centers
    "hunyuan": Config("hunyuan", 3, H=24, N=118800, d=128, dtype="bf16",
                      G=1536, sigma=0.35, Cq=100, Ck=1000, iters=10, rho=0.12,
                      grid=(33, 45, 80), vox=(6, 16, 16)),
    # Stress sweep base point: 16 heads, 32^3 grid; sigma and rho are swept
    "stress": Config("stress", 4, H=16, N=32768, d=128, dtype="bf16", G=512,
                     sigma=0.35, Cq=64, Ck=512, iters=10, rho=0.1,
                     grid=(32, 32, 32), vox=(8, 8, 8)),
}

STRESS_SIGMAS = (0.1, 0.35, 1.0)
STRESS_RHOS = (0.05, 0.1, 0.2, 0.4, 1.0)


def to_bf16_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even) and
    return them widened back to float32, so every value is exactly a bf16."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    u = x.view(np.uint32)
    lsb = (u >> 16) & np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return x


def _center_ids(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    if cfg.grid is None:
        return rng.integers(0, cfg.G, size=cfg.N)
    T, Hh, W = cfg.grid
    Tv, Hv, Wv = cfg.vox
    assert T * Hh * W == cfg.N and Tv * Hv * Wv == cfg.G
    t = np.arange(T)[:, None, None]
    h = np.arange(Hh)[None, :, None]
    w = np.arange(W)[None, None, :]
    z = ((t * Tv // T) * Hv + (h * Hv // Hh)) * Wv + (w * Wv // W)
    z = np.broadcast_to(z, (T, Hh, W)).reshape(-1).copy()
    if cfg.reassign > 0:
        m = rng.random(cfg.N) < cfg.reassign
        z[m] = rng.integers(0, cfg.G, size=int(m.sum()))
    return z


def _raw_head(cfg: Config, h: int):
    rng = np.random.default_rng([cfg.seed, h])
    d = cfg.d
    mq = rng.standard_normal((cfg.G, d), dtype=np.float32)
    mk = rng.standard_normal((cfg.G, d), dtype=np.float32)
    mv = rng.standard_normal((cfg.G, d), dtype=np.float32)
    z = _center_ids(cfg, rng)
    s = np.float32(cfg.sigma)
    q = mq[z] + s * rng.standard_normal((cfg.N, d), dtype=np.float32)
    k = mk[z] + s * rng.standard_normal((cfg.N, d), dtype=np.float32)
    v = mv[z] + s * rng.standard_normal((cfg.N, d), dtype=np.float32)
    return q, k, v, z


_ALPHA_CACHE: Dict[Config, float] = {}


def logit_alpha(cfg: Config) -> float:
    """Common factor applied to q and k of every head so that q.k/sqrt(d) over
    65,536 random (i, j) pairs of head 0 has standard deviation 2."""
    if not cfg.scale_logits:
        return 1.0
    if cfg in _ALPHA_CACHE:
        return _ALPHA_CACHE[cfg]
    q, k, _, _ = _raw_head(cfg, 0)
    rng = np.random.default_rng([cfg.seed, 0, 99])
    i = rng.integers(0, cfg.N, size=65536)
    j = rng.integers(0, cfg.N, size=65536)
    dots = np.einsum("nd,nd->n", q[i].astype(np.float64), k[j].astype(np.float64))
    std = float(np.std(dots / math.sqrt(cfg.d)))
    a = math.sqrt(2.0 / std)
    _ALPHA_CACHE[cfg] = a
    return a


def make_head(cfg: Config, h: int):
    """(q, k, v, center_ids) of head h as float32 arrays [N, d]; for bf16
    configs the values are already rounded to bf16."""
    q, k, v, z = _raw_head(cfg, h)
    a = np.float32(logit_alpha(cfg))
    if a != 1.0:
        q *= a
        k *= a
    if cfg.dtype == "bf16":
        q, k, v = to_bf16_f32(q), to_bf16_f32(k), to_bf16_f32(v)
    return q, k, v, z


def make_inputs(cfg: Config, heads=None):
    """Stacked float32 arrays [H', N, d] for the requested heads (default all)."""
    heads = range(cfg.H) if heads is None else heads
    qs, ks, vs = [], [], []
    for h in heads:
        q, k, v, _ = make_head(cfg, h)
        qs.append(q); ks.append(k); vs.append(v)
    return np.stack(qs), np.stack(ks), np.stack(vs)


def forgy_init(cfg: Config, X: np.ndarray, h: int, which: int, C: int) -> np.ndarray:
    """Seeded Forgy initialisation: the values of C distinct tokens of X [N, d]
    (which = 0 for queries, 1 for keys), as float32 [C, d]."""
    rng = np.random.default_rng([cfg.seed, h, which])
    idx = rng.choice(X.shape[0], size=C, replace=False)
    return np.ascontiguousarray(X[idx], dtype=np.float32)
