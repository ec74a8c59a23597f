"""Several GPUs: independent shards, one process per GPU.

The coding path has no exchange step.  Chunks depend on one another only
through the exclusive scan of their sizes, and that scan stays inside one call
on one GPU, so a set of tensors is split across ranks in contiguous blocks
(shard_range) and each rank codes its share into its own streams and offsets,
with no collective on the data path.

Where the shards should read as one global stream (one offsets array over the
whole set, say for writing it out), global_base gathers every rank's word count
(8 bytes per rank, one all_gather) and returns the word index at which this
rank's part starts; hq_offsets_add then moves the rank's offsets by it on the
device.  Host logic only; the coding runs in libhq.so's kernels.
"""
from __future__ import annotations

import torch


def shard_range(n_items: int, world: int, rank: int) -> tuple[int, int]:
    """Items [lo, hi) of rank `rank` among `world`: contiguous blocks in item order,
    the first n_items % world ranks taking one item more."""
    if world < 1 or not 0 <= rank < world or n_items < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, n_items >= 0")
    q, r = divmod(n_items, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def global_base(local_words: int, group=None, device: torch.device | str | None = None) -> tuple[int, int]:
    """(first global word of this rank's part, total words of all ranks), from one
    all_gather of the ranks' word counts in rank order.  Without an initialised
    process group: (0, local_words).  device: where the 8-byte count lives for the
    collective (the rank's GPU for NCCL, the CPU for gloo)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 0, int(local_words)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    mine = torch.tensor([int(local_words)], dtype=torch.int64, device=device)
    counts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(counts, mine, group=group)
    c = [int(t.item()) for t in counts]
    return sum(c[:rank]), sum(c)
