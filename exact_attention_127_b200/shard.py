"""One attention problem split across GPUs by heads.

Every head (b, h) is an independent problem, and within a head every query row
is ("GPU 学习日报 Day 21", section 6: the forward pass parallelises over
independent row blocks).  So N ranks, one per GPU, each run the single-GPU
kernel on a contiguous range of the B*H heads, with no exchange step.  The
only communication is the optional gather of O and LSE, when the caller wants
the whole result on every rank: one all-gather (NCCL over NVLink on GPUs, gloo
on CPU tensors), bit for bit (values travel as their raw bytes).

Layout: q, k, v, o are [B, H, N, d] and lse [B, H, N], so the heads of one
rank, flattened to [B*H, N, d] and [B*H, N], are one contiguous slice.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from ._lib import attn_fwd


def head_range(n_heads: int, world: int, rank: int):
    """Contiguous heads [start, stop) of `rank`: the B*H heads in `world`
    slices whose sizes differ by at most one, lower ranks first."""
    if world < 1 or not 0 <= rank < world or n_heads < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, n_heads >= 0")
    base, extra = divmod(n_heads, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def head_slice(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """This rank's heads of a [B, H, ...] tensor, as a contiguous [count, ...] view."""
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    flat = x.reshape(x.shape[0] * x.shape[1], *x.shape[2:])
    start, stop = head_range(flat.shape[0], world, rank)
    return flat[start:stop]


def attn_fwd_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                   scale: float | None = None, out: torch.Tensor | None = None,
                   lse: torch.Tensor | None = None, stream=None):
    """The forward pass on one rank's heads: q, k, v are [count, N, d] slices
    (head_slice), o and lse come back as [count, N, d] and [count, N]."""
    if q.dim() != 3:
        raise ValueError("expected [count, N, d] head slices")
    c, N, d = q.shape
    o4 = None if out is None else out.view(1, c, N, d)
    l3 = None if lse is None else lse.view(1, c, N)
    o, l = attn_fwd(q.view(1, c, N, d), k.view(1, c, N, d), v.view(1, c, N, d), causal=causal,
                    scale=scale, out=o4, lse=l3, stream=stream)
    return o.view(c, N, d), l.view(c, N)


def _all_gather_rows(local: torch.Tensor, n_heads: int, group=None) -> torch.Tensor:
    """All-gather [count_r, ...] slices of unequal size into [n_heads, ...]."""
    world = dist.get_world_size(group)
    counts = [head_range(n_heads, world, r) for r in range(world)]
    width = max(stop - start for start, stop in counts)
    pad = torch.zeros((width, *local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]].copy_(local)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:stop - start] for p, (start, stop) in zip(parts, counts)])


def gather_heads(o_local: torch.Tensor, lse_local: torch.Tensor, n_heads: int, group=None):
    """O [n_heads, N, d] and LSE [n_heads, N] of all ranks on every rank, from
    each rank's [count, N, d] and [count, N] slices.  The values travel as raw
    bytes, so the result is an exact copy whatever the dtype."""
    def gather(t):
        t = t.contiguous()
        return _all_gather_rows(t.view(torch.uint8), n_heads, group).view(t.dtype)
    return gather(o_local), gather(lse_local)
