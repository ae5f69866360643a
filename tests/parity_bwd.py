"""Element-wise parity of the CUDA backward with the fp64 backward oracle.

Bound (derived from the arithmetic of the CUDA path): the kernels recompute P = exp(S - lse) in fp32, round P and
dS = P (dP - D) to bf16 (relative error <= 2^-9 each, round to nearest) before
the P^T dO, dS K and dS^T Q products (the full-tile kernels of the two-kernel
path form dS from the bf16-rounded P: two roundings, <= 2^-8 relative, which
the factor-of-two margin below covers), take D from the forward's bf16 output O
(|D - D_exact| <= 2^-9 sum_c |dO_c O_c|), accumulate in fp32 and round each
gradient to bf16 once (<= 2^-9 relative).  With a factor-of-two margin on
each term, for every element

    |dV_gpu - dV| <= 2^-7 sum_q P_qk |dO_q|                                  + 2^-8 |dV|
    |dQ_gpu - dQ| <= 2^-7 scale sum_k P_qk (|dP_qk - D_q| + A_q) |K_k|       + 2^-8 |dQ|
    |dK_gpu - dK| <= 2^-7 scale sum_q P_qk (|dP_qk - D_q| + A_q) |Q_q|       + 2^-8 |dK|

with A_q = sum_c |dO_qc O_qc| and the sums taken over the visible pairs (and,
for dK and dV, over the query heads that share the KV head), plus 1e-6 for
the fp32 accumulation.  The magnitudes are computed here in float64 from the
oracle's own P and dP.
"""
from __future__ import annotations

import numpy as np
import torch

from harness.inputs import MASK_NAMES, make_dout, make_qkv
from oracle import attention_bwd_fp64 as G
from oracle import attention_fp64 as F


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bounds(q, k, v, do, scale, mask_kind, window):
    """Per-element error bounds of dq, dk, dv (float64 arrays)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    idx = np.arange(N)
    allowed = F.visible(idx[:, None], idx[None, :], mask_kind, window)
    bq = np.zeros_like(q)
    bk = np.zeros_like(k)
    bv = np.zeros_like(v)
    for b in range(B):
        for hq in range(Hq):
            hk = F.kv_head_of(hq, Hq, Hkv)
            p = G._probs(q[b, hq], k[b, hk], scale, allowed)
            dp = G._grad_probs(do[b, hq], v[b, hk])
            o = p @ v[b, hk]
            dvec = (p * dp).sum(axis=1, keepdims=True)
            a = (np.abs(do[b, hq]) * np.abs(o)).sum(axis=1, keepdims=True)
            w = p * (np.abs(dp - dvec) + a)
            bv[b, hk] += p.T @ np.abs(do[b, hq])
            bq[b, hq] = scale * (w @ np.abs(k[b, hk]))
            bk[b, hk] += scale * (w.T @ np.abs(q[b, hq]))
    return bq, bk, bv


def run_cuda_bwd(q, k, v, do, mask, window=None, scale=None, deterministic=False):
    from exact_io_aware_72_b200 import bwd, fwd
    out, lse = fwd(q, k, v, scale=scale, mask=mask, window=window)
    dq, dk, dv = bwd(q, k, v, out, lse, do, scale=scale, mask=mask, window=window, deterministic=deterministic)
    torch.cuda.synchronize()
    return dq, dk, dv


def check_bwd_case(B, Hq, Hkv, N, d, mask, window=None, seed=0, scale=None, sharp=False, deterministic=False):
    q, k, v = make_qkv(B, Hq, Hkv, N, d, seed, device="cpu", sharp=sharp)
    do = make_dout(B, Hq, N, d, seed)
    got = run_cuda_bwd(q.cuda(), k.cuda(), v.cuda(), do.cuda(), mask, window, scale, deterministic)
    qn, kn, vn, don = to_np(q), to_np(k), to_np(v), to_np(do)
    s = (1.0 / np.sqrt(d)) if scale is None else scale
    kind = MASK_NAMES[mask]
    refs = G.attention_bwd(qn, kn, vn, don, s, kind, window)
    bnds = bounds(qn, kn, vn, don, s, kind, window)
    return compare_bwd(("dq", "dk", "dv"), [to_np(g) for g in got], refs, bnds,
                       (B, Hq, Hkv, N, d, mask, window))


def compare_bwd(names, got, refs, bnds, what):
    """Every element within its bound (module docstring); relative L2 < 1e-2.
    Returns the worst error / bound ratio per gradient."""
    worst = {}
    for name, g, ref, bd in zip(names, got, refs, bnds):
        assert np.isfinite(g).all(), name
        err = np.abs(g - ref)
        tol = 2.0 ** -7 * bd + 2.0 ** -8 * np.abs(ref) + 1e-6
        ratio = float((err / tol).max())
        worst[name] = ratio
        assert ratio <= 1.0, (name, what, ratio, float(err.max()))
        ref_norm = np.linalg.norm(ref)
        if ref_norm > 1e-6:  # (one visible key per row gives dQ = dK = 0 exactly)
            assert np.linalg.norm(g - ref) / ref_norm < 1e-2, (name, np.linalg.norm(g - ref) / ref_norm)
    return worst
