"""Host-side helpers for running the decode path on several GPUs.

The paged decode is independent per sequence: every (sequence, kv head) reads only
its own blocks and writes only its own output rows.  So a batch shards by
sequence across ranks with no exchange on the data path -- each rank holds its own
KV pool and block manager for its sequences.  Sequences that share prefix blocks
(forks, a common system prompt) must stay on one rank, since a block lives in one
rank's pool; ``shard_ranges`` cuts only between such groups.

One process per GPU, ``torch.distributed`` for the plumbing (NCCL on GPUs, gloo
for the CPU tests).  Timing across ranks takes the maximum device time.
"""
from __future__ import annotations


def shard_ranges(costs, world: int, groups=None):
    """Contiguous, group-aligned [start, end) ranges of sequences, one per rank,
    balancing the summed ``costs`` (e.g. context lengths).

    groups: optional group label per sequence; sequences with the same label must
    be contiguous and are never split.  Ranks beyond the number of groups get
    empty ranges.
    """
    n = len(costs)
    if world < 1:
        raise ValueError("world must be >= 1")
    if groups is None:
        groups = list(range(n))
    if len(groups) != n:
        raise ValueError("groups must label every sequence")
    # group boundaries and the cost of each group
    bounds, cum = [0], [0.0]
    seen = set()
    for i in range(n):
        if i > 0 and groups[i] != groups[i - 1]:
            if groups[i] in seen:
                raise ValueError("sequences of one group must be contiguous")
            bounds.append(i)
            cum.append(0.0)
        seen.add(groups[i])
        cum[-1] += float(costs[i])
    cut_cost = [0.0]
    for c in cum:
        cut_cost.append(cut_cost[-1] + c)
    bounds.append(n)
    total = cut_cost[-1]
    # rank r ends at the group boundary whose prefix cost is closest to (r+1)/world of the total
    ranges, start_g = [], 0
    ngroups = len(bounds) - 1
    for r in range(world):
        if r == world - 1:
            end_g = ngroups
        else:
            target = total * (r + 1) / world
            end_g = start_g
            while end_g < ngroups and abs(cut_cost[end_g + 1] - target) <= abs(cut_cost[end_g] - target):
                end_g += 1
        ranges.append((bounds[start_g], bounds[end_g]))
        start_g = end_g
    return ranges


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a float over all ranks of the default process group (identity when
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
