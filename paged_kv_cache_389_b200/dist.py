"""Host-side helpers for running the decode path on several GPUs.

The paged decode is independent per sequence: every (sequence, kv head) reads only
its own blocks and writes only its own output rows.  So a batch shards by
sequence across ranks with no exchange on the data path -- each rank holds its own
KV pool and block manager for its sequences.  Sequences that share prefix blocks
(forks, a common system prompt) must stay on one rank, since a block lives in one
rank's pool; ``shard_ranges`` cuts only between such groups.

The other split is tensor-parallel (chenxutan "vLLM 深度拆解" 3.4: each layer is cut
across cards): every rank holds all sequences but only a contiguous range of kv
heads, with their query heads (a GQA group is never split), and the same block
tables (each rank's manager makes the same decisions).  Each rank decodes its heads
with no exchange; ``gather_heads`` is the one collective, an all-gather of the
output heads for a consumer that needs all of them on every rank.

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


def shard_kv_heads(num_kv_heads: int, world: int):
    """Contiguous [start, end) kv-head ranges, one per rank, as even as possible (the
    first num_kv_heads % world ranks take one more).  Rank r's query heads are
    [start * g, end * g) with g = num_q_heads / num_kv_heads."""
    if world < 1 or num_kv_heads < world:
        raise ValueError("need 1 <= world <= num_kv_heads")
    base, extra = divmod(num_kv_heads, world)
    ranges, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        ranges.append((lo, hi))
        lo = hi
    return ranges


def gather_heads(out_local, kv_ranges, group_size: int, group=None):
    """All-gather each rank's attention output [S, (end - start) * g, d] along the head
    axis into [S, num_kv_heads * g, d] on every rank.  Uneven shards are padded to
    the largest for the collective and trimmed after it."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if len(kv_ranges) != world:
        raise ValueError("one kv-head range per rank")
    widths = [(hi - lo) * group_size for lo, hi in kv_ranges]
    rank = dist.get_rank(group)
    if out_local.shape[1] != widths[rank]:
        raise ValueError("local output does not match this rank's heads")
    S, _, d = out_local.shape
    wmax = max(widths)
    padded = out_local.new_zeros((S, wmax, d))
    padded[:, :widths[rank]] = out_local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded.contiguous(), group=group)
    return torch.cat([p[:, :w] for p, w in zip(parts, widths)], dim=1)

