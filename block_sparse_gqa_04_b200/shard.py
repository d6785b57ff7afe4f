"""Splitting one MSA problem across ranks.

The path has no exchange step: sequences never see one another, and the GQA
groups are independent too (each group has its own index-query head and its own
selection, "Substantial numerical differences with Minimax MSA attention vs
Minimax's Reference", section 原因分析: top-k per index head, never pooled; the
shared index-key head k_idx is read by every group).  So a problem shards by
sequence (decode batches) or by group (long prefills) with no collective on the
data path; each rank runs the library on its own slice.  Reassembling the output
on every rank is one all-gather, done here with torch.distributed.
"""
from __future__ import annotations

from typing import Tuple

import torch

from . import msa


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous share [lo, hi) of n items for `rank` of `world`: the first
    n % world ranks take one item more, so the shares differ by at most one."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad shard: n={n}, world={world}, rank={rank}")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def forward_sequence_shard(q, k, v, q_idx, k_idx, world: int, rank: int, **kw):
    """msa.forward on this rank's sequences [lo, hi) of the batch (dimension 0 of
    every tensor).  Returns (out of those sequences, (lo, hi)); a rank without
    sequences returns an empty output."""
    lo, hi = shard_range(q.shape[0], world, rank)
    if hi == lo:
        return q.new_empty((0,) + tuple(q.shape[1:]), dtype=v.dtype), (lo, hi)
    out = msa.forward(q[lo:hi], k[lo:hi], v[lo:hi], q_idx[lo:hi], k_idx[lo:hi], **kw)
    return out, (lo, hi)


def forward_group_shard(q, k, v, q_idx, k_idx, world: int, rank: int, **kw):
    """msa.forward on this rank's GQA groups [g0, g1): their query heads
    (g0 * G .. g1 * G - 1 of q), key/value heads and index-query heads; k_idx is
    shared by all groups and read whole.  The head slices are copied to
    contiguous tensors (a deployment would hold only its own heads).  Returns
    (out [B, Sq, (g1 - g0) * G, D], (g0, g1))."""
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    g0, g1 = shard_range(Hkv, world, rank)
    if g1 == g0:
        return q.new_empty(tuple(q.shape[:2]) + (0, q.shape[3]), dtype=v.dtype), (g0, g1)
    out = msa.forward(q[:, :, g0 * G:g1 * G].contiguous(), k[:, :, g0:g1].contiguous(),
                      v[:, :, g0:g1].contiguous(), q_idx[:, :, g0:g1].contiguous(), k_idx, **kw)
    return out, (g0, g1)


def all_gather_shards(part: torch.Tensor, n: int, world: int, dim: int,
                      item_size: int = 1) -> torch.Tensor:
    """Concatenates every rank's `part` along `dim` in rank order (the shares of
    shard_range over n items, each item_size entries of `dim`: 1 for sequences,
    the group size for query heads), on every rank, with one all_gather of
    padded equal-size pieces."""
    import torch.distributed as dist

    size = item_size * max(hi - lo for lo, hi in (shard_range(n, world, r) for r in range(world)))
    pad_shape = list(part.shape)
    pad_shape[dim] = size
    padded = part.new_zeros(pad_shape)
    padded.narrow(dim, 0, part.shape[dim]).copy_(part)
    pieces = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(pieces, padded)
    out = []
    for r in range(world):
        lo, hi = shard_range(n, world, r)
        out.append(pieces[r].narrow(dim, 0, (hi - lo) * item_size))
    return torch.cat(out, dim=dim)
