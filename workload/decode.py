"""Host-side stand-in for the serving engine of the decode-loop workload.

Pages cited (title, then section):
  [GeoTrick] "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
              Without Losing Accuracy", "Solving the Memory Fragmentation
              Problem" (compaction every ~128 decode steps; a paged block can
              be reclaimed only once it is empty)
  [Review]   "TriAttention: trigonometric KV cache compression for long
              reasoning", "The KV budget is a runtime knob that chat sessions
              should raise" (the budget is a soft target between compressions)

The engine owns a free list of pool blocks.  Appending tokens takes blocks
from it; after a compression step the blocks that the step reports as freed
go back to it and the sequence's block table is truncated.  This is plain
bookkeeping: it holds no scoring, selection or compaction arithmetic.
"""

from __future__ import annotations

from typing import List

import torch

from .gen import Workload, write_tokens


class PoolExhausted(RuntimeError):
    pass


def append_tokens(wl: Workload, s: int, count: int) -> None:
    """Append ``count`` freshly drawn tokens to sequence ``s``."""
    bs = wl.cfg.block_size
    length = int(wl.seq_len[s].item())
    have = (length + bs - 1) // bs
    need = (length + count + bs - 1) // bs
    if need > wl.max_blocks:
        raise PoolExhausted(f"sequence {s} needs {need} table entries, table has {wl.max_blocks}")
    if need - have > len(wl.free_blocks):
        raise PoolExhausted(f"pool has {len(wl.free_blocks)} free blocks, sequence {s} needs {need - have}")
    if need > have:
        new = [wl.free_blocks.pop(0) for _ in range(need - have)]
        wl.block_table[s, have:need] = torch.tensor(new, dtype=torch.int32, device=wl.device)
    write_tokens(wl, s, length, count)
    wl.seq_len[s] = length + count
    wl.cur_pos[s] += count


def recycle_freed(wl: Workload, old_len: List[int], freed_ids: torch.Tensor, freed_count: int) -> List[int]:
    """Return the blocks a compression step freed to the pool.

    ``old_len`` is each sequence's length before the step; the new lengths
    are read from ``wl.seq_len``.  Each sequence's table is truncated to the
    blocks it still uses, and the freed ids are checked against exactly the
    truncated entries (same ids, same order), so a step that reports wrong
    blocks is caught here.
    """
    bs = wl.cfg.block_size
    ids = freed_ids[:freed_count].cpu().tolist()
    new_len = wl.seq_len.cpu().tolist()
    table = wl.block_table.cpu()
    expect: List[int] = []
    for s, (lo, ln) in enumerate(zip(old_len, new_len)):
        keep = (ln + bs - 1) // bs
        had = (lo + bs - 1) // bs
        expect += table[s, keep:had].tolist()
        table[s, keep:had] = -1
    if ids != expect:
        raise AssertionError("freed block ids differ from the truncated table entries")
    wl.block_table.copy_(table.to(wl.device))
    wl.free_blocks.extend(ids)
    return ids
