"""The five workload shapes the path is measured and checked on.

Pages cited (title, then section):
  [Digest]   "TriAttention: Trigonometric KV Compression for Efficient Long Reasoning"
  [GeoTrick] "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
              Without Losing Accuracy"
  [Review]   "TriAttention: trigonometric KV cache compression for long reasoning"

The pages evaluate on long-reasoning generation (AIME25 / MATH500 with 32K
generated tokens, budgets 1024-3072, GQA 7B/8B-class models: [GeoTrick] "What
the Numbers Look Like", [Review] "Calibration statistics are tied to a
specific model").  Those datasets and models are not available, so these
synthetic shapes stand in for them: one bf16 post-RoPE key per cached token,
drawn around a per-head centre, with query statistics drawn to a target
concentration.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple


def geometric_offsets(hi: int) -> List[int]:
    """Future-query offsets 1, 2, 4, ..., hi (hi a power of two)."""
    out, d = [], 1
    while d <= hi:
        out.append(d)
        d *= 2
    return out


@dataclasses.dataclass
class WorkloadConfig:
    name: str
    L: int                      # layers
    Hkv: int                    # KV heads per layer
    G: int                      # query heads per KV head (GQA group)
    D: int                      # head dimension
    base: float                 # RoPE base
    lens: List[int]             # cached tokens per sequence
    deltas: List[int]           # future offsets averaged over
    budget: int                 # B: keys kept per (sequence, layer, KV head)
    window: int                 # W: most recent keys always kept (inside B)
    block_size: int = 16        # tokens per paged block
    key_noise: float = 0.3      # pre-RoPE key = centre + key_noise * N(0, I)
    # Query statistics: "direct" sets E|q_i| = qabs_ratio * |centre_i| with
    # R given; "samples" draws calibration samples around the centres with a
    # per-head noise scale chosen for a target concentration.
    stats: str = "samples"
    qabs_ratio: float = 1.2
    r_range: Tuple[float, float] = (0.6, 0.98)
    low_r_fraction: float = 0.0     # fraction of query heads forced to low R
    low_r_value: float = 0.3
    n_samples: int = 4096
    table: str = "identity"         # "identity" or "shuffled" block table
    pool_headroom: float = 0.0      # spare blocks in the shared pool
    extra_blocks_per_seq: int = 0   # table slack for appended tokens
    seed: int = 0
    # Decode loop (only for the decode workload).
    decode_rounds: int = 0
    decode_append: int = 0
    lens_range: Optional[Tuple[int, int]] = None   # drawn lengths (decode)

    @property
    def Hq(self) -> int:
        return self.Hkv * self.G

    @property
    def S(self) -> int:
        return len(self.lens)

    def replace(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


# 1 layer, 1 KV head, T = 4096 at positions 0..4095, next query at 4096;
# E|q_i| = 1.2 |c_q,i| given directly; offsets 1..1024; B = 512, W = 64.
HEAD1_T4096 = WorkloadConfig(
    name="single-head T=4096 B=512", L=1, Hkv=1, G=1, D=128, base=1e4,
    lens=[4096], deltas=geometric_offsets(1024), budget=512, window=64,
    stats="direct", qabs_ratio=1.2, table="identity")

# 32 layers x 8 KV heads, G = 4, one sequence of 32768, base 5e5,
# R ~ U(0.6, 0.98), offsets 1..4096, B = 2048, W = 128, compress once.
L32H8_T32K = WorkloadConfig(
    name="32Lx8H G=4 T=32768 B=2048", L=32, Hkv=8, G=4, D=128, base=5e5,
    lens=[32768], deltas=geometric_offsets(4096), budget=2048, window=128,
    stats="samples", r_range=(0.6, 0.98), table="identity")

# Decode loop: the L32H8_T32K model, 16 sequences with lengths U(8K, 32K) in one
# shared pool of 16-token blocks with 10 % headroom; every 128 appended
# tokens compress to B = 2048 and recycle the freed blocks
# ([GeoTrick] "Solving the Memory Fragmentation Problem": compaction every
# ~128 decode steps).
DECODE16 = WorkloadConfig(
    name="decode 16 seqs U(8K,32K) every 128 tokens B=2048", L=32, Hkv=8, G=4,
    D=128, base=5e5, lens=[0] * 16, deltas=geometric_offsets(4096),
    budget=2048, window=128, stats="samples", r_range=(0.6, 0.98),
    table="shuffled", pool_headroom=0.10, extra_blocks_per_seq=8,
    decode_rounds=16, decode_append=128, lens_range=(8192, 32768))

# Long context: one sequence of 131072, base 1e6, B = 4096, W = 256; 10 % of
# query heads at R ~ 0.3 so the norm term dominates there.
L32H8_T128K = WorkloadConfig(
    name="32Lx8H G=4 T=131072 B=4096", L=32, Hkv=8, G=4, D=128, base=1e6,
    lens=[131072], deltas=geometric_offsets(4096), budget=4096, window=256,
    stats="samples", r_range=(0.6, 0.98), low_r_fraction=0.10,
    low_r_value=0.3, table="identity")

# Wide model: 64 layers x 8 KV heads, G = 8, batch 4 x 65536 in a paged pool,
# R ~ U(0.3, 0.98), offsets 1..8192, B = 4096, W = 128.
L64H8G8_4X64K = WorkloadConfig(
    name="64Lx8H G=8 4x65536 B=4096", L=64, Hkv=8, G=8, D=128, base=1e6,
    lens=[65536] * 4, deltas=geometric_offsets(8192), budget=4096, window=128,
    stats="samples", r_range=(0.3, 0.98), table="shuffled")

CONFIGS = {
    "head1_t4096": HEAD1_T4096,
    "l32h8_t32k": L32H8_T32K,
    "decode16": DECODE16,
    "l32h8_t128k": L32H8_T128K,
    "l64h8g8_4x64k": L64H8G8_4X64K,
}
