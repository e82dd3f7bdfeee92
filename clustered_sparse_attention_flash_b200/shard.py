"""Head-sharded SVG-EAR forward over several GPUs (one process per GPU).

Every step of the operator works on one head at a time (clustering,
permutation, block error, routing and attention are all per head; SVG-EAR
review, "complete inference pipeline" steps (1)-(4)), so a layer of H heads
splits into contiguous head slices with no exchange inside the operator.
Rank r runs heads head_range(H, world, r) through the unchanged C entry point
on its own GPU; when every rank needs the whole output, one all-gather over
the process group (NCCL over NVLink) assembles O [H, N, d].  No operand of a
kernel ever lives in another GPU's memory.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """[begin, end) of the heads rank `rank` of `world` owns: contiguous
    slices, the first H % world ranks one head longer."""
    if world < 1 or not 0 <= rank < world or H < 0:
        raise ValueError("bad partition request")
    base, extra = divmod(H, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def forward_heads_sharded(Q, K, V, Cq: int, Ck: int, iters: int, rho: float, scale: float = 0.0,
                          init_q=None, init_k=None, group=None, gather: bool = True,
                          compute: Optional[Callable] = None, stream=None):
    """Run this rank's head slice of one SVG-EAR layer and, with gather=True,
    all-gather the slices into the full output on every rank.

    Q, K, V [H, N, d] and init_q [H, Cq, d], init_k [H, Ck, d] (or None) are
    the whole layer's tensors on this rank's device; only this rank's heads
    are read.  `compute(Q, K, V, Cq, Ck, iters, rho, scale, init_q, init_k)`
    returns the output of a head slice; it defaults to svgear_forward through
    the C ABI.  Returns (O, (begin, end)): O [H, N, d] when gathering, else
    this rank's slice [end - begin, N, d]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    H = Q.shape[0]
    b, e = head_range(H, world, rank)
    if compute is None:
        from . import svgear as sv

        def compute(q, k, v, cq, ck, it, r, s, iq, ik):
            return sv.forward(q, k, v, cq, ck, it, r, s, iq, ik, stream=stream)[0]
    sl = lambda x: None if x is None else x[b:e]
    if e > b:
        part = compute(Q[b:e], K[b:e], V[b:e], Cq, Ck, iters, rho, scale, sl(init_q), sl(init_k))
    else:  # more ranks than heads: this rank owns none, but joins the gather
        part = Q.new_empty((0,) + tuple(Q.shape[1:]))
    if not gather or world == 1:
        return part, (b, e)
    # equal-sized blocks for the collective: every rank contributes the
    # longest slice, zero-padded; the padding is dropped after the gather
    longest = max(hr[1] - hr[0] for hr in (head_range(H, world, r) for r in range(world)))
    buf = torch.zeros((longest,) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
    buf[: e - b] = part
    blocks = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(blocks, buf, group=group)
    O = torch.empty((H,) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
    for r in range(world):
        rb, re_ = head_range(H, world, r)
        O[rb:re_] = blocks[r][: re_ - rb]
    return O, (b, e)
