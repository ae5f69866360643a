"""Exact attention forward (bf16 and FP8 inputs), backward, paged-KV decoding and
ring attention across GPUs for NVIDIA B200 (sm_100a).

``fwd``, ``fwd_fp8``, ``bwd`` and ``decode`` (and ``fwd_host`` / ``fwd_fp8_host`` on host
tensors, with the copies overlapped) run the hand-written tcgen05/TMA kernels of
``libattn_b200.so`` through its C ABI (include/attn.h); there is no CPU or
library fallback.
"""
from .attn import (AttnError, MASKS, bwd, bwd_debug_error, debug_error, decode, decode_debug_error,  # noqa: F401
                   decode_num_splits, decode_static, decode_workspace_bytes, fwd, fwd_fp8, fwd_fp8_host, fwd_host, load_library,
                   merge, num_work_items)
from . import ring  # noqa: F401

__all__ = ["fwd", "fwd_fp8", "fwd_host", "fwd_fp8_host", "bwd", "bwd_debug_error", "decode", "decode_debug_error", "decode_num_splits", "decode_static",
           "decode_workspace_bytes", "debug_error", "load_library", "merge", "num_work_items", "ring", "AttnError",
           "MASKS"]
