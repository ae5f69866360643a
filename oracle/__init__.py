"""fp64 CPU oracle for the exact attention forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product path.
"""
from .attention_fp64 import (  # noqa: F401
    MASK_FULL, MASK_CAUSAL, MASK_SLIDING_WINDOW,
    attention, attention_flops, kv_head_of, visible, visible_count_per_row,
    visible_pairs,
)
