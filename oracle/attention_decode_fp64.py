"""fp64 CPU oracle for attention decoding against a paged KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA path.

What it computes, restated from the pages:

* The KV cache keeps the keys and values of the tokens already processed so
  that a decoding step only computes attention for the new tokens ("Efficient
  Attention", giftedprocrastinator.com, section "What it does", KV-cache
  paragraph; "Attention Mechanism Variants Beyond Self-Attention",
  tempatgunting.com, section "Multi-Query and Grouped-Query Attention": the
  cache is what GQA/MQA shrink, one cached head per KV group).
* The cache is stored in fixed-size pages with a page table per sequence, and
  the attention reads K and V through that table without approximating
  anything ("Efficient attention: long context and sub-quadratic variants",
  stanleyjacob.dev, section "FlashAttention: exact attention, IO-aware",
  PagedAttention paragraph).
* Each new token's attention is the same masked softmax attention as the
  forward (``oracle.attention_fp64``): causal j <= i, sliding window
  i - w < j <= i, or every cached key.

Readings where the pages leave the step open:

* Layouts: q ``[B, Hq, Nq, d]``; each cache ``[num_pages, Hkv, page_size, d]``
  (one page holds ``page_size`` consecutive positions of every KV head);
  ``block_table[b, p]`` is the physical page of logical page p of sequence b,
  i.e. of positions ``p*page_size .. p*page_size + page_size - 1``;
  ``seq_lens[b]`` = L_b counts the cached keys including the Nq new ones.
* The Nq new tokens are the last Nq positions of their sequence: query t sits
  at position ``L_b - Nq + t`` (so Nq = 1 is plain decoding and Nq > 1 a
  multi-token step with the causal mask inside the new tokens).
* Rolling window buffer: under a sliding window the step reads only positions
  ``lo_b .. L_b - 1`` with ``lo_b = max(0, L_b - Nq - w + 1)``, the oldest key
  any of its queries can see; pages wholly before ``lo_b`` are never looked
  up, so a caller may recycle them (and leave their table entries stale).
  Slots at positions >= L_b of the last page are never read either.

Parity pins (``tests/test_oracle_decode.py``): equality with the forward
oracle's last Nq rows of the gathered sequence, invariance under any physical
page permutation, NaN in every slot the step must not read, closed forms
(single cached key, equal keys), brute force in pure Python on tiny inputs,
and planted mistakes that each pin catches.
"""
from __future__ import annotations

import numpy as np

from .attention_fp64 import MASK_CAUSAL, MASK_FULL, MASK_SLIDING_WINDOW, kv_head_of, visible


def query_positions(L: int, Nq: int) -> np.ndarray:
    """Positions of the Nq new tokens of a sequence with L cached keys: its
    last Nq positions, L - Nq .. L - 1."""
    if not 1 <= Nq <= L:
        raise ValueError("need 1 <= Nq <= L")
    return np.arange(L - Nq, L, dtype=np.int64)


def first_needed_position(L: int, Nq: int, mask_kind: int, window=None) -> int:
    """Oldest position any query of the step can see: the first query's
    window start under a sliding window, 0 otherwise."""
    if mask_kind == MASK_SLIDING_WINDOW:
        if window is None or window < 1:
            raise ValueError("sliding window needs window >= 1")
        return max(0, L - Nq - window + 1)
    if mask_kind in (MASK_FULL, MASK_CAUSAL):
        return 0
    raise ValueError(f"unknown mask kind {mask_kind}")


def gather_positions(cache, table_row, page_size: int, lo: int, L: int) -> np.ndarray:
    """Cached rows of positions lo .. L-1 of one sequence, every KV head:
    position t lives in physical page table_row[t // page_size] at slot
    t % page_size.  Returns [Hkv, L - lo, d] float64; only the pages that
    hold those positions are touched."""
    cache = np.asarray(cache)
    num_pages, Hkv, ps, d = cache.shape
    if ps != page_size:
        raise ValueError("page size disagrees with the cache")
    out = np.empty((Hkv, L - lo, d), dtype=np.float64)
    for lp in range(lo // page_size, (L - 1) // page_size + 1):   # logical pages holding lo .. L-1
        page = int(table_row[lp])
        if not 0 <= page < num_pages:
            raise ValueError(f"page table entry {page} out of range")
        p0 = max(lo, lp * page_size)                # first and one-past-last position
        p1 = min(L, (lp + 1) * page_size)           # of this page that the step reads
        out[:, p0 - lo:p1 - lo, :] = cache[page, :, p0 - lp * page_size:p1 - lp * page_size, :]
    return out


def decode_attention(q, k_cache, v_cache, block_table, seq_lens, scale=None,
                     mask_kind: int = MASK_CAUSAL, window=None):
    """Attention of the new tokens of every sequence against its paged cache.

    q [B, Hq, Nq, d]; k_cache, v_cache [num_pages, Hkv, page_size, d];
    block_table [B, max_pages] integers; seq_lens [B] integers with
    Nq <= L_b.  Returns (out [B, Hq, Nq, d], lse [B, Hq, Nq]) in float64,
    lse the natural log of each row's softmax normaliser over its visible,
    scaled scores.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, Nq, d = q.shape
    num_pages, Hkv, page_size, dk = np.asarray(k_cache).shape
    if dk != d or np.asarray(v_cache).shape != np.asarray(k_cache).shape:
        raise ValueError("q and cache shapes disagree")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    block_table = np.asarray(block_table)
    seq_lens = np.asarray(seq_lens)
    out = np.empty((B, Hq, Nq, d), dtype=np.float64)
    lse = np.empty((B, Hq, Nq), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        qpos = query_positions(L, Nq)
        lo = first_needed_position(L, Nq, mask_kind, window)
        kb = gather_positions(k_cache, block_table[b], page_size, lo, L)
        vb = gather_positions(v_cache, block_table[b], page_size, lo, L)
        keypos = np.arange(lo, L, dtype=np.int64)
        if mask_kind == MASK_FULL:
            allowed = np.ones((Nq, L - lo), dtype=bool)   # every cached key
        else:
            allowed = visible(qpos[:, None], keypos[None, :], mask_kind, window)
        for hq in range(Hq):
            hk = kv_head_of(hq, Hq, Hkv)
            s = np.where(allowed, _scores(q[b, hq], kb[hk], scale), -np.inf)   # [Nq, L - lo]
            out[b, hq], lse[b, hq] = _softmax_rows(s, vb[hk])
    return out, lse


def _scores(q_rows, k_rows, scale):
    """s_tj = scale * q_t . k_j for the gathered keys."""
    return (q_rows @ k_rows.T) * scale


def _softmax_rows(s, v_rows):
    """Row softmax of the masked scores applied to V, and each row's
    log-sum-exp m + ln(sum exp(s - m)) (m, the row maximum, only keeps fp64
    finite)."""
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ v_rows) / l, (m + np.log(l))[:, 0]


def decode_bytes(B: int, Hq: int, Hkv: int, Nq: int, d: int, seq_lens, mask_kind: int, window=None) -> int:
    """Bytes a decoding step must move at minimum: K and V (bf16) of the
    positions lo_b .. L_b - 1 of every sequence and KV head, q and out
    (bf16) and lse (fp32)."""
    keys = 0
    for L in np.asarray(seq_lens).tolist():
        keys += int(L) - first_needed_position(int(L), Nq, mask_kind, window)
    return 2 * 2 * d * Hkv * keys + B * Hq * Nq * (2 * 2 * d + 4)
