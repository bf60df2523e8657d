"""Host-side multi-GPU plumbing of the compression step (one process per GPU).

Pages: "TriAttention: trigonometric KV cache compression for long
reasoning" - "The KV cache, not the weights, is what runs out of memory"
(the deployment target is a single GPU).  The step has no exchange at all:
every (sequence, layer, KV head) unit is scored, selected and compacted on
its own.  Several GPUs therefore run independent caches - each rank owns
whole sequences - and need no collective on the data path.  The only
collective is the control-plane reduction of the step time (the slowest
rank decides the job's time) and of the freed-block count.
"""

from __future__ import annotations

from typing import List, Sequence


def shard_sequences(num_sequences: int, world: int, rank: int) -> List[int]:
    """Sequences owned by ``rank``: round-robin, so lengths mix evenly."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("need world >= 1 and 0 <= rank < world")
    return list(range(rank, num_sequences, world))


def shard_heads(num_kv_heads: int, world: int, rank: int) -> List[int]:
    """KV heads owned by ``rank`` when the heads are split across GPUs (as a
    tensor-parallel KV cache is): a contiguous slice of Hkv / world heads.
    Every sequence lives on every rank; each rank compresses its own heads
    in its own paged pool, and since every head keeps the same budget the
    ranks free the same number of blocks per sequence."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("need world >= 1 and 0 <= rank < world")
    if num_kv_heads % world:
        raise ValueError("the KV heads must divide evenly over the ranks")
    per = num_kv_heads // world
    return list(range(rank * per, (rank + 1) * per))


def freed_consistent(dist, freed_this_rank: int, device=None) -> bool:
    """Head sharding: all-reduce the freed-block count (min and max over the
    ranks) and return whether every rank freed the same number."""
    import torch
    if dist is None:
        return True
    lo = torch.tensor([int(freed_this_rank)], dtype=torch.int64, device=device)
    hi = lo.clone()
    dist.all_reduce(lo, op=dist.ReduceOp.MIN)
    dist.all_reduce(hi, op=dist.ReduceOp.MAX)
    return int(lo.item()) == int(hi.item())


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic cache (independent streams per rank)."""
    return int(base_seed) * 1000003 + int(rank)


def reduce_job(dist, step_ms_total: float, keys_this_rank: int, freed_this_rank: int, device=None):
    """Reduce per-rank results to the job's: max of the timed milliseconds,
    sum of keys and of freed blocks.  Every rank takes the same collective
    steps; ``dist`` may be None for a single process."""
    import torch
    if dist is None:
        return float(step_ms_total), int(keys_this_rank), int(freed_this_rank)
    t = torch.tensor([float(step_ms_total)], dtype=torch.float64, device=device)
    n = torch.tensor([int(keys_this_rank), int(freed_this_rank)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), int(n[0].item()), int(n[1].item())


def keys_per_second(total_keys: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' keys over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return total_keys * steps / (max_ms / 1e3)


def check_partition(shards: Sequence[Sequence[int]], num_sequences: int) -> bool:
    """True if the shards cover every sequence exactly once."""
    seen = sorted(s for sh in shards for s in sh)
    return seen == list(range(num_sequences))
