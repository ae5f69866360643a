"""Helpers of the decoding parity tests: run the CUDA decoding step through the
C ABI and compare with the fp64 decoding oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from harness.inputs import MASK_NAMES, make_paged_kv
from oracle import attention_decode_fp64 as D
from tests.parity import compare, element_bound_p_bf16, to_np

# Decoding rounds P to bf16 (the step is bound by HBM reads; include/attn.h):
# its element bound is max(1e-2, one bf16 ulp of the exact value).
DECODE_BOUND = element_bound_p_bf16


def keep_from_for_window(lens, Nq, window):
    """Rolling window buffer: first position each sequence must keep."""
    return np.maximum(np.asarray(lens, dtype=np.int64) - Nq - window + 1, 0)


def run_decode(inp, mask, window=None, scale=None, num_splits=None, grid_ctas=0, max_seq_len=None, out=None,
               lse=None):
    from exact_io_aware_72_b200 import decode
    o, l = decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["block_table"], inp["seq_lens"],
                  max_seq_len=max_seq_len, scale=scale, mask=mask, window=window, num_splits=num_splits,
                  grid_ctas=grid_ctas, out=out, lse=lse)
    torch.cuda.synchronize()
    return o, l


def oracle_for(inp, mask, window=None, scale=None, seqs=None):
    """Oracle result for the sequences ``seqs`` (default all).  Only the pages
    those sequences' tables name are copied to the host, renumbered."""
    table = inp["block_table"].cpu().numpy()
    lens = inp["seq_lens"].cpu().numpy()
    seqs = list(range(table.shape[0])) if seqs is None else list(seqs)
    used = sorted({int(p) for b in seqs for p in table[b] if p >= 0})
    remap = {p: i for i, p in enumerate(used)}
    idx = torch.as_tensor(used, dtype=torch.long, device=inp["k_cache"].device)
    kc = to_np(inp["k_cache"].index_select(0, idx))
    vc = to_np(inp["v_cache"].index_select(0, idx))
    sub_table = np.array([[remap.get(int(p), -1) for p in table[b]] for b in seqs], dtype=np.int64)
    q = to_np(inp["q"][seqs])
    return D.decode_attention(q, kc, vc, sub_table, lens[seqs], scale, MASK_NAMES[mask], window)


def check_decode_case(B, Hq, Hkv, Nq, d, lens, page_size, mask, window=None, seed=0, scale=None,
                      num_splits=None, rolling=False, fill=float("nan"), extra_pages=1, grid_ctas=0):
    """Whole-output parity of one case; unused cache slots hold ``fill``."""
    from exact_io_aware_72_b200 import decode_debug_error
    decode_debug_error()  # start from a clear error word
    keep = keep_from_for_window(lens, Nq, window) if rolling else None
    inp = make_paged_kv(B, Hq, Hkv, Nq, d, lens, page_size, seed, device="cpu", keep_from=keep, fill=fill,
                        extra_pages=extra_pages)
    gpu = {k: v.cuda() for k, v in inp.items()}
    out, lse = run_decode(gpu, mask, window, scale, num_splits, grid_ctas)
    ref_o, ref_l = oracle_for(inp, mask, window, scale)
    what = f"{(B, Hq, Hkv, Nq, d, tuple(int(x) for x in lens), page_size, mask, window, num_splits)}"
    stats = compare(to_np(out), to_np(lse), ref_o, ref_l, what, bound=DECODE_BOUND)
    st, code = decode_debug_error()
    assert st == 0, f"{what}: device error {code:#x}"
    return stats
