"""Seeded synthetic inputs for the TriAttention key-importance + eviction path.

This package is shared by the tests, ``bench.py`` and ``__graft_entry__`` as
the single source of inputs for both the CUDA path and the float64 oracle.  It
holds none of the method's scoring, selection or compaction arithmetic: it
only draws keys, values and calibration samples, lays them out in a paged
pool, and (for the decode-loop workload) plays the part of the serving engine
that appends tokens and recycles freed blocks.
"""

from .configs import CONFIGS, WorkloadConfig, geometric_offsets  # noqa: F401
from .gen import (  # noqa: F401
    Workload,
    make_workload,
    rope_rotate_half,
    noise_scale_for_target_concentration,
)
