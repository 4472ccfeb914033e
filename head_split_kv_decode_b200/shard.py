"""Sequence sharding across GPUs: which positions each rank's retrieval heads
keep, and the exchange of decode partials between ranks.

A sequence longer than one GPU's retrieval caches is split into contiguous
position ranges, one per rank (one process per GPU).  Every rank appends every
token (its streaming heads keep the whole window, its retrieval heads only its
range), decodes its share with ``DuoCache.decode_partial`` (rank 0 owns the
streaming heads), and the ranks exchange their (o, lse) partials with one
all-gather; each rank then merges them with ``cache.merge_partials``.  The
exchange is ``torch.distributed`` (NCCL over NVLink on GPUs); this module holds
only that plumbing, no attention arithmetic.
"""

import torch


def shard_ranges(capacity, world):
    """[(lo, hi)] per rank: contiguous ranges of ceil(capacity / world)
    positions; the last range is open-ended so the sequence can keep growing
    on the last rank."""
    if world < 1 or capacity < 1:
        raise ValueError("world and capacity must be positive")
    per = -(-capacity // world)
    out = [(r * per, (r + 1) * per) for r in range(world)]
    out[-1] = (out[-1][0], 1 << 62)
    return out


def owns_streaming(rank):
    """Rank 0 contributes the streaming heads (every rank holds them)."""
    return rank == 0


def gather_partials(o_part, lse_part, group=None):
    """All-gather every rank's partial: returns (o [world, ...], lse [world,
    ...]) stacked in rank order, contiguous, on the partials' device."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    o_list = [torch.empty_like(o_part) for _ in range(world)]
    lse_list = [torch.empty_like(lse_part) for _ in range(world)]
    dist.all_gather(o_list, o_part.contiguous(), group=group)
    dist.all_gather(lse_list, lse_part.contiguous(), group=group)
    return torch.stack(o_list), torch.stack(lse_list)
