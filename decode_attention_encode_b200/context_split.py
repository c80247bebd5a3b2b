"""Context split of one long sequence's decode across ranks.

Each rank holds a contiguous part of every sequence's latent store (the
cached tokens ``shard_range`` assigns it), runs any decode call of the
library on that part, and the ranks exchange their (out, lse) pairs with one
all-gather; ``lla_merge_attn`` then combines them exactly (a log-sum-exp
merge: softmax attention over the union of disjoint parts). The exchange is
B*H*(d_h + 1) floats per (layer, loop) step, independent of the context
length. The data path is the library's kernels; torch.distributed (NCCL on
GPUs, gloo on CPU) only moves the small partial results.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from ._lib import lla_merge_attn


def shard_range(N: int, world: int, rank: int):
    """The [start, stop) cached tokens rank `rank` of `world` holds: a
    contiguous split of N as even as possible (earlier ranks take the
    remainder)."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError("bad world, rank or N")
    base, extra = divmod(N, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def gather_and_merge(out: torch.Tensor, lse: torch.Tensor, group=None, merge=None):
    """All-gathers every rank's (out [..., d], lse [...]) and merges them.
    `merge` defaults to the library's lla_merge_attn (device tensors); a
    rank whose part is empty passes out = 0, lse = -inf."""
    world = dist.get_world_size(group)
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return (merge or lla_merge_attn)(torch.stack(outs), torch.stack(lses))
