"""fp64 CPU oracle of the Star Attention hot path (test infrastructure only).

Only tests, the smoke check and the benchmark's CPU-baseline / reference leg
import this package. The product library never does.
"""
from .oracle import (  # noqa: F401
    bf16_bits,
    global_rows,
    lse_merge,
    phase1_gather_rows,
    phase1_full,
    phase1_ranges,
    phase1_rows,
    phase1_rows_selected,
    phase2_rows,
    rope,
    round_bf16,
)
