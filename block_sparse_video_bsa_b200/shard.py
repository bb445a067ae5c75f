"""Partition of one attention call's (batch, head) slices across ranks.

Every stage of the path is per (b, h): the anchor is the mean of that head's
video queries, the summaries, the block scores and the lists are all computed
inside one head ("Spark-H3: Block Sparse Attention Speeds Up MiniMax-H3 in
ComfyUI", section "What Spark-Attn changes": one anchor per head).  So a call
over B*H slices splits into contiguous slice ranges, one per rank, and the
forward needs no exchange at all: rank r runs bsa_forward on its own range
(a sub-call with B = 1, H = count).  The only collective is the optional
gather of O when one device must hold the whole output.

The slices of a [B, H, N, d] tensor are contiguous in memory in (b, h) order,
so a range of them is one contiguous sub-tensor.
"""

from __future__ import annotations

import torch


def head_range(total: int, world: int, rank: int):
    """(start, count) of the contiguous (b, h) slices rank ``rank`` owns.

    The split is balanced: counts differ by at most one, ranks in order cover
    [0, total) exactly once.  A rank may own nothing when total < world."""
    if world < 1 or not (0 <= rank < world) or total < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, total >= 0")
    start = rank * total // world
    end = (rank + 1) * total // world
    return start, end - start


def local_slices(X: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """The [1, count, N, d] view of this rank's slices of a [B, H, N, d] tensor."""
    B, H = X.shape[:2]
    start, count = head_range(B * H, world, rank)
    return X.reshape(B * H, *X.shape[2:])[start:start + count].unsqueeze(0)


def gather_heads(local: torch.Tensor, total: int, group=None) -> torch.Tensor:
    """All-gather of every rank's [1, count, ...] slices into [total, ...].

    Counts may differ by one between ranks, so each rank's block is padded to
    the largest count before the all-gather and the padding is dropped after.
    Works with NCCL (device tensors) and gloo (host tensors)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    _, count = head_range(total, world, rank)
    if local.shape[1] != count:
        raise ValueError(f"rank {rank} holds {local.shape[1]} slices, owns {count}")
    width = -(-total // world)
    pad = local.new_zeros((width,) + tuple(local.shape[2:]))
    pad[:count] = local[0]
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    out = local.new_empty((total,) + tuple(local.shape[2:]))
    for r in range(world):
        s, c = head_range(total, world, r)
        out[s:s + c] = parts[r][:c]
    return out
