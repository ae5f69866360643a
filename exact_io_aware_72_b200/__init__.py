"""Exact attention forward and backward for NVIDIA B200 (sm_100a).

``fwd`` and ``bwd`` run the hand-written tcgen05/TMA kernels of
``libattn_b200.so`` through its C ABI (include/attn.h); there is no CPU or
library fallback.
"""
from .attn import (AttnError, MASKS, bwd, bwd_debug_error, debug_error, fwd, fwd_host,  # noqa: F401
                   load_library, num_work_items)

__all__ = ["fwd", "fwd_host", "bwd", "bwd_debug_error", "debug_error", "load_library", "num_work_items",
           "AttnError", "MASKS"]
