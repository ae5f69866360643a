"""fp64 CPU oracle for the gradient of exact attention (the backward pass).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only ``tests/`` (and the benchmark's CPU-baseline leg) use it.  It
shares no code with the CUDA path.

What it computes: for the forward of ``attention_fp64.attention`` (masked
softmax attention, definition and page citations there) and an upstream
gradient dO, the gradients of L = sum(dO * O) with respect to q, k and v.
The pages do not print the backward formulas; "Efficient attention: long
context and sub-quadratic variants" (stanleyjacob.dev, section "Against the
real libraries") names a recompute-based backward pass as part of the
production kernel line, and "Efficient Attention: Flash Attention, Sliding
Window, Sparse" (creativeworksofknowledge.com, section "Flash Attention")
describes FlashAttention as trading recompute for memory traffic.  The
gradient itself is fixed by the forward definition and the chain rule, written
out here on the materialised scores of each (batch, query head):

    S = scale * q k^T, masked entries -inf        P = softmax_rows(S)
    dV_j  = sum_i P_ij dO_i                        (P^T dO)
    dP_ij = dO_i . v_j                             (dO v^T)
    dS_ij = P_ij (dP_ij - D_i),  D_i = sum_l P_il dP_il  (softmax Jacobian)
    dQ_i  = scale * sum_j dS_ij k_j                (dS k)
    dK_j  = scale * sum_i dS_ij q_i                (dS^T q)

With grouped KV heads, dK and dV of a KV head are the sums over the query
heads that read it (the gradient of ``repeat_interleave``).  D_i equals
dO_i . O_i, the form a kernel uses; here it is taken from P and dP.

Parity pins (``tests/oracle_bwd_pins.py``): central finite differences of the
pinned forward oracle, torch's float64 autograd of SDPA on the CPU as a library
special case, and identities the mathematics fixes (shift invariance of the
keys, value shift, all-equal keys, one key, window >= N == causal, GQA ==
repeated-KV MHA).
"""
from __future__ import annotations

import numpy as np

from oracle.attention_fp64 import MASK_CAUSAL, kv_head_of, visible


def attention_bwd(q, k, v, do, scale=None, mask_kind: int = MASK_CAUSAL, window=None):
    """Gradients (dq, dk, dv) of sum(do * attention(q, k, v)) in float64.

    q, do: [B, Hq, N, d]; k, v: [B, Hkv, N, d] (any real dtype, upcast exactly
    to float64).  Returns float64 arrays shaped like q, k and v.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or do.shape != q.shape:
        raise ValueError("q, k, v, do shapes disagree")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    idx = np.arange(N, dtype=np.int64)
    allowed = visible(idx[:, None], idx[None, :], mask_kind, window)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for hq in range(Hq):
            hk = kv_head_of(hq, Hq, Hkv)
            p = _probs(q[b, hq], k[b, hk], scale, allowed)
            dv[b, hk] += _grad_v(p, do[b, hq])
            ds = _grad_scores(p, _grad_probs(do[b, hq], v[b, hk]))
            dq[b, hq] = _grad_q(ds, k[b, hk], scale)
            dk[b, hk] += _grad_k(ds, q[b, hq], scale)
    return dq, dk, dv


def _probs(q_head, k_head, scale, allowed):
    """P = row softmax of S = scale q k^T over the visible keys (masked -> 0)."""
    s = np.where(allowed, (q_head @ k_head.T) * scale, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def _grad_v(p, do_head):
    """dV = P^T dO: value j collects dO_i weighted by how much row i used it."""
    return p.T @ do_head


def _grad_probs(do_head, v_head):
    """dP_ij = dO_i . v_j (the gradient of O = P V with respect to P)."""
    return do_head @ v_head.T


def _grad_scores(p, dp):
    """dS_ij = P_ij (dP_ij - D_i), D_i = sum_l P_il dP_il: the softmax Jacobian
    applied row by row (masked entries have P = 0, so dS = 0 there)."""
    dvec = (p * dp).sum(axis=1, keepdims=True)
    return p * (dp - dvec)


def _grad_q(ds, k_head, scale):
    """dQ = scale dS k (S = scale q k^T is linear in q)."""
    return (ds @ k_head) * scale


def _grad_k(ds, q_head, scale):
    """dK = scale dS^T q (S = scale q k^T is linear in k)."""
    return (ds.T @ q_head) * scale
