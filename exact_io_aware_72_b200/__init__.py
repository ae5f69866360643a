"""Exact attention forward for NVIDIA B200 (sm_100a).

``fwd`` runs the hand-written tcgen05/TMA kernel of ``libattn_b200.so`` through
its C ABI (include/attn.h); there is no CPU or library fallback.
"""
from .attn import AttnError, MASKS, debug_error, fwd, fwd_host, load_library, num_work_items  # noqa: F401

__all__ = ["fwd", "fwd_host", "debug_error", "load_library", "num_work_items", "AttnError", "MASKS"]
