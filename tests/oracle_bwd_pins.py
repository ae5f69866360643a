"""Pins of the fp64 backward oracle to facts that do not come from it.

Each ``pin_*`` takes the backward oracle module (or a patched copy) and raises
AssertionError when its gradients disagree with a fact fixed by the forward
definition and the mathematics.  ``test_oracle_bwd.py`` runs them on the real
module; ``test_oracle_bwd_mutants.py`` plants mistakes and checks each one is
caught.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import attention_fp64 as fwd_oracle

FULL, CAUSAL, WINDOW = 0, 1, 2


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _inputs(B, Hq, Hkv, N, d, seed):
    return (_rand((B, Hq, N, d), seed), _rand((B, Hkv, N, d), seed + 1), _rand((B, Hkv, N, d), seed + 2),
            _rand((B, Hq, N, d), seed + 3))


def pin_finite_differences(orc):
    """Central differences of L = sum(dO * O) through the (separately pinned)
    forward oracle, for every element of q, k and v of tiny cases: all three
    masks, grouped heads, a scale other than 1/sqrt(d)."""
    cases = ((1, 2, 1, 5, 3, FULL, None, None), (1, 2, 2, 6, 3, CAUSAL, None, 0.7),
             (2, 2, 1, 6, 2, WINDOW, 3, None), (1, 3, 3, 4, 2, WINDOW, 1, None))
    h = 1e-6
    for n, (B, Hq, Hkv, N, d, kind, w, scale) in enumerate(cases):
        q, k, v, do = _inputs(B, Hq, Hkv, N, d, 100 + 10 * n)
        dq, dk, dv = orc.attention_bwd(q, k, v, do, scale, kind, w)

        def loss(qq, kk, vv):
            return float((do * fwd_oracle.attention(qq, kk, vv, scale, kind, w)[0]).sum())

        for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                args = [q, k, v]
                xp = x.copy(); xp[idx] += h
                xm = x.copy(); xm[idx] -= h
                args[which] = xp
                lp = loss(*args)
                args[which] = xm
                lm = loss(*args)
                num[idx] = (lp - lm) / (2 * h)
            err = np.abs(num - g).max()
            assert err < 1e-6 * max(1.0, np.abs(num).max()), (n, which, err)


def pin_torch_autograd_fp64(orc):
    """torch's CPU float64 SDPA differentiated by autograd (the library
    special case), causal, windowed (explicit mask) and full, B=1, H=4, T=96."""
    torch.manual_seed(1)
    B, H, T, d = 1, 4, 96, 16
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    for kind, w, kw in ((CAUSAL, None, dict(is_causal=True)),
                        (WINDOW, 17, dict(attn_mask=(j <= i) & (j > i - 17))),
                        (FULL, None, dict())):
        q, k, v, do = torch.randn(4, B, H, T, d, dtype=torch.float64).unbind(0)
        qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
        F.scaled_dot_product_attention(qr, kr, vr, **kw).backward(do)
        dq, dk, dv = orc.attention_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), None, kind, w)
        for g, ref in ((dq, qr.grad), (dk, kr.grad), (dv, vr.grad)):
            assert float((torch.from_numpy(g) - ref).abs().max()) < 1e-11, kind


def pin_shift_identities(orc):
    """Adding one vector to every key adds a per-row constant to the scores, so
    the loss does not change: sum_j dK_j = 0 per KV head.  Adding one vector c
    to every value adds c to every output row: sum_j dV_j = sum of dO over the
    query heads that read the KV head."""
    for kind, w in ((FULL, None), (CAUSAL, None), (WINDOW, 5)):
        B, Hq, Hkv, N, d = 2, 4, 2, 23, 6
        q, k, v, do = _inputs(B, Hq, Hkv, N, d, 7)
        _, dk, dv = orc.attention_bwd(q, k, v, do, None, kind, w)
        assert np.abs(dk.sum(axis=2)).max() < 1e-12, kind
        g = Hq // Hkv
        want = do.reshape(B, Hkv, g, N, d).sum(axis=(2, 3))
        assert np.abs(dv.sum(axis=2) - want).max() < 1e-12, kind


def pin_equal_keys_and_single_key(orc):
    """All keys equal: P is uniform over each visible set and cannot move with
    q, so dQ = 0.  N = 1: the one key gets weight 1, so dV = dO (summed over the
    group) and dQ = dK = 0."""
    B, Hq, Hkv, N, d = 1, 2, 1, 17, 4
    q, k, v, do = _inputs(B, Hq, Hkv, N, d, 11)
    k[:] = _rand((1, 1, 1, d), 12)
    for kind, w in ((FULL, None), (CAUSAL, None), (WINDOW, 4)):
        dq, _, _ = orc.attention_bwd(q, k, v, do, None, kind, w)
        assert np.abs(dq).max() < 1e-13, kind
    q, k, v, do = _inputs(B, Hq, Hkv, 1, d, 13)
    dq, dk, dv = orc.attention_bwd(q, k, v, do, None, CAUSAL, None)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    assert np.abs(dv - do.sum(axis=1, keepdims=True)).max() < 1e-15


def pin_window_ge_N_is_causal(orc):
    """A window covering the whole sequence is the causal mask: same gradients."""
    q, k, v, do = _inputs(1, 2, 1, 19, 5, 21)
    ref = orc.attention_bwd(q, k, v, do, None, CAUSAL, None)
    for w in (19, 20, 1000):
        got = orc.attention_bwd(q, k, v, do, None, WINDOW, w)
        for a, b in zip(got, ref):
            assert np.array_equal(a, b), w


def pin_gqa_is_repeated_mha(orc):
    """Grouped heads read KV head h // g ("Multi-Query and Grouped-Query
    Attention", repeat_interleave): their dQ equals MHA's on the repeated K, V,
    and dK, dV of a KV head are the sums of the repeated heads' gradients."""
    B, Hq, Hkv, N, d = 2, 6, 2, 13, 4
    q, k, v, do = _inputs(B, Hq, Hkv, N, d, 31)
    g = Hq // Hkv
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    for kind, w in ((CAUSAL, None), (WINDOW, 4), (FULL, None)):
        dq, dk, dv = orc.attention_bwd(q, k, v, do, None, kind, w)
        dq2, dk2, dv2 = orc.attention_bwd(q, kr, vr, do, None, kind, w)
        assert np.abs(dq - dq2).max() < 1e-13, kind
        assert np.abs(dk - dk2.reshape(B, Hkv, g, N, d).sum(axis=2)).max() < 1e-12, kind
        assert np.abs(dv - dv2.reshape(B, Hkv, g, N, d).sum(axis=2)).max() < 1e-12, kind


def pin_scale_convention(orc):
    """Scores are scale * q k^T: scaling q by t with scale / t leaves every
    forward quantity unchanged, so dQ scales by 1/t and dK, dV do not change."""
    q, k, v, do = _inputs(1, 2, 2, 11, 4, 41)
    t = 3.0
    dq, dk, dv = orc.attention_bwd(q, k, v, do, 0.5, CAUSAL, None)
    dq2, dk2, dv2 = orc.attention_bwd(q * t, k, v, do, 0.5 / t, CAUSAL, None)
    assert np.abs(dq2 * t - dq).max() < 1e-12
    assert np.abs(dk2 - dk).max() < 1e-12 and np.abs(dv2 - dv).max() < 1e-12
    dq0, _, _ = orc.attention_bwd(q, k, v, do, None, CAUSAL, None)
    dq1, _, _ = orc.attention_bwd(q, k, v, do, 1.0 / math.sqrt(4), CAUSAL, None)
    assert np.array_equal(dq0, dq1)


ALL_PINS = [
    pin_shift_identities, pin_equal_keys_and_single_key, pin_window_ge_N_is_causal,
    pin_gqa_is_repeated_mha, pin_scale_convention, pin_finite_differences, pin_torch_autograd_fp64,
]
