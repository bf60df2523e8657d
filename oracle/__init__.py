"""Float64 CPU oracle of the TriAttention key-importance + eviction path.

TEST INFRASTRUCTURE ONLY: importable by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product library.
"""

from . import tri_oracle  # noqa: F401
from .tri_oracle import (  # noqa: F401
    as_bands, from_bands, calibrate, compact_rows, compress_step, compress_step_distance, compress_unit,
    distance_scores, distance_series, distance_table, effective_query, freed_blocks, future_phase_mean,
    group_query, head_score, rope_frequencies, select, unit_rows, unit_scores,
)
