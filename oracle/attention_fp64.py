"""fp64 CPU oracle for the exact attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA path.

What it computes is the plain definition of masked softmax attention, written
out in float64 with the scores materialised:

* "Efficient attention: long context and sub-quadratic variants"
  (stanleyjacob.dev), section "Implementation, twice", ``masked_attention``:
  scores = q k^T * scale, masked entries set to -inf before the softmax, each
  row renormalised over its visible set, result = softmax(scores) v.
* same page, section "Sliding-window and local attention" and
  ``sliding_window_mask``: query i sees keys j with i - w < j <= i.
* "Efficient Attention: Flash Attention, Sliding Window, Sparse"
  (creativeworksofknowledge.com), section "Code": causal attention is SDPA's
  ``is_causal=True`` (j <= i).
* "Attention Mechanism Variants Beyond Self-Attention" (tempatgunting.com),
  section "Multi-Query and Grouped-Query Attention": Hq query heads share Hkv
  key/value heads through ``repeat_interleave(Hq // Hkv, dim=1)``, i.e. query
  head h reads key/value head h // (Hq // Hkv).
* FlashAttention computes exactly this result (first page, section
  "FlashAttention: exact attention, IO-aware"), so the definition is the
  oracle; the online softmax is not reproduced here.

The per-row log-sum-exp is not printed on the pages; it is read as the natural
log of the sum of exp over the scaled, masked scores of the row:
lse_i = m_i + ln(sum_j exp(s_ij - m_i)) with m_i the row maximum (subtracting
m_i only keeps fp64 finite; it does not change the value).

Parity pins: every function here is pinned in ``tests/test_oracle.py`` against
facts the pages or the mathematics fix (mask sets of both pages' mask
functions, window >= N == causal, GQA == repeated-KV MHA, closed forms for
equal keys / dominant keys / row 0 / w = 1, brute force in pure Python on tiny
inputs, torch's CPU float64 SDPA as a library special case, and invariants).
"""
from __future__ import annotations

import numpy as np

MASK_FULL = 0
MASK_CAUSAL = 1
MASK_SLIDING_WINDOW = 2


def kv_head_of(hq: int, Hq: int, Hkv: int) -> int:
    """KV head read by query head ``hq``: consecutive groups of Hq//Hkv query
    heads share one KV head, as ``repeat_interleave`` on the head axis does
    (tempatgunting.com, "Multi-Query and Grouped-Query Attention")."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // (Hq // Hkv)


def visible(i, j, mask_kind: int, window=None):
    """Boolean visibility of key j to query i (broadcasting numpy arrays).

    full: every key; causal: j <= i; sliding window: i - w < j <= i
    (stanleyjacob.dev, "Sliding-window and local attention" and
    ``sliding_window_mask``; True means allowed).
    """
    i = np.asarray(i)
    j = np.asarray(j)
    if mask_kind == MASK_FULL:
        return np.ones(np.broadcast(i, j).shape, dtype=bool)
    if mask_kind == MASK_CAUSAL:
        return j <= i
    if mask_kind == MASK_SLIDING_WINDOW:
        if window is None or window < 1:
            raise ValueError("sliding window needs window >= 1")
        return (j <= i) & (j > i - window)
    raise ValueError(f"unknown mask kind {mask_kind}")


def visible_count_per_row(N: int, mask_kind: int, window=None) -> np.ndarray:
    """|V(i)| for every query row i, counted from the visibility definition."""
    i = np.arange(N, dtype=np.int64)
    if mask_kind == MASK_FULL:
        return np.full(N, N, dtype=np.int64)
    if mask_kind == MASK_CAUSAL:
        return i + 1                       # j = 0..i
    if mask_kind == MASK_SLIDING_WINDOW:
        lo = np.maximum(i - window + 1, 0)  # smallest j with j > i - w
        return i - lo + 1
    raise ValueError(f"unknown mask kind {mask_kind}")


def visible_pairs(N: int, mask_kind: int, window=None) -> int:
    """Number of visible (query, key) pairs of one head."""
    return int(visible_count_per_row(N, mask_kind, window).sum())


def attention_flops(B: int, Hq: int, N: int, d: int, mask_kind: int, window=None) -> int:
    """FLOPs of the two matmuls counted over visible pairs only: each pair
    costs d multiply-adds for q.k and d for p*v, i.e. 4*d FLOPs
    (stanleyjacob.dev, "The quadratic wall": 2N^2 d per matmul per head)."""
    return 4 * B * Hq * d * visible_pairs(N, mask_kind, window)


def attention(q, k, v, scale=None, mask_kind: int = MASK_CAUSAL, window=None,
              rows=None, row_chunk: int = 512):
    """Exact masked softmax attention in float64.

    q: [B, Hq, N, d]; k, v: [B, Hkv, N, d] (any real dtype; upcast exactly to
    float64).  ``rows`` (optional, 1-D int array) restricts the query rows
    computed; the result then has that many rows, in the given order.
    Returns (out [B, Hq, R, d] float64, lse [B, Hq, R] float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d) or v.shape != k.shape:
        raise ValueError("q, k, v shapes disagree")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]
    out = np.empty((B, Hq, R, d), dtype=np.float64)
    lse = np.empty((B, Hq, R), dtype=np.float64)
    cols = np.arange(N, dtype=np.int64)
    for b in range(B):
        for hq in range(Hq):
            hk = kv_head_of(hq, Hq, Hkv)
            kh = k[b, hk]
            vh = v[b, hk]
            for r0 in range(0, R, row_chunk):
                ri = rows[r0:r0 + row_chunk]
                s = _scores(q[b, hq, ri], kh, scale)
                allowed = visible(ri[:, None], cols[None, :], mask_kind, window)
                s = np.where(allowed, s, -np.inf)          # -inf before softmax
                e, m, l = _softmax_terms(s)
                out[b, hq, r0:r0 + len(ri)] = _normalised_sum(e, l, vh)
                lse[b, hq, r0:r0 + len(ri)] = _log_sum_exp(m, l)
    return out, lse


def _scores(q_rows, k_head, scale):
    """s_ij = scale * sum_c q[i,c] k[j,c]  (the q k^T product, then the scale)."""
    return (q_rows @ k_head.T) * scale


def _softmax_terms(s):
    """Row maximum m_i, e_ij = exp(s_ij - m_i) (masked -inf entries give 0)
    and the row sum l_i = sum_j e_ij."""
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e, m, l


def _normalised_sum(e, l, v_head):
    """out_i = sum_j e_ij v_j / l_i: softmax weights applied to V."""
    return (e @ v_head) / l


def _log_sum_exp(m, l):
    """lse_i = m_i + ln l_i = ln sum_j exp(s_ij)."""
    return (m + np.log(l))[:, 0]
