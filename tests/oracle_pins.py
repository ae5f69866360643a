"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each ``pin_*`` takes the oracle module (or a patched copy of it) and raises
AssertionError when the oracle disagrees with a fact fixed by the pages or by
the mathematics.  ``test_oracle.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on oracles with a planted mistake and
checks that every mistake is caught by at least one pin.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

FULL, CAUSAL, WINDOW = 0, 1, 2
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_figures.txt")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# --------------------------------------------------------------------------- masks
def pin_mask_page3_form(orc):
    """The creativeworksofknowledge.com page ("Code", ``sliding_window_mask``)
    returns True where a key is MASKED: (j > i) | (j < i - window + 1).  Its
    negation must be the oracle's visible set for every T <= 40, w in 1..T+1."""
    for T in range(1, 41):
        i = torch.arange(T)[:, None]
        j = torch.arange(T)[None, :]
        for w in range(1, T + 2):
            masked = (j > i) | (j < i - w + 1)
            got = orc.visible(np.arange(T)[:, None], np.arange(T)[None, :], WINDOW, w)
            assert np.array_equal(got, (~masked).numpy()), (T, w)


def pin_mask_row_structure(orc):
    """Sliding window (stanleyjacob.dev, "Sliding-window and local attention"):
    every row sees itself, at most w keys, all of them at or before i, and the
    visible keys are contiguous; causal is the lower triangle incl. diagonal."""
    for T in (1, 2, 7, 33):
        I = np.arange(T)[:, None]
        J = np.arange(T)[None, :]
        causal = orc.visible(I, J, CAUSAL)
        assert np.array_equal(causal, np.tril(np.ones((T, T), dtype=bool)))
        assert orc.visible(I, J, FULL).all()
        for w in range(1, T + 2):
            m = orc.visible(I, J, WINDOW, w)
            for r in range(T):
                cols = np.nonzero(m[r])[0]
                assert cols[-1] == r                     # ends at the diagonal
                assert len(cols) == min(r + 1, w)        # at most w, all of them if possible
                assert np.all(np.diff(cols) == 1)        # contiguous band


def pin_visible_counts(orc):
    """Row counts and pair totals against closed forms: N, i+1, min(i+1, w);
    N^2, N(N+1)/2 and N w - w(w-1)/2 (for w <= N)."""
    for N in (1, 5, 128, 1000):
        assert np.array_equal(orc.visible_count_per_row(N, FULL), np.full(N, N))
        assert np.array_equal(orc.visible_count_per_row(N, CAUSAL), np.arange(1, N + 1))
        assert orc.visible_pairs(N, FULL) == N * N
        assert orc.visible_pairs(N, CAUSAL) == N * (N + 1) // 2
        for w in (1, 2, 3, N // 2 + 1, N, N + 5):
            assert np.array_equal(orc.visible_count_per_row(N, WINDOW, w),
                                  np.minimum(np.arange(1, N + 1), w))
            ww = min(w, N)
            assert orc.visible_pairs(N, WINDOW, w) == N * ww - ww * (ww - 1) // 2
    # the counts agree with the mask itself
    for N, w in ((17, 5), (64, 64), (40, 1)):
        I = np.arange(N)[:, None]
        J = np.arange(N)[None, :]
        for kind in (FULL, CAUSAL, WINDOW):
            assert orc.visible_pairs(N, kind, w) == int(orc.visible(I, J, kind, w).sum())


def pin_page_figures(orc):
    """Counts the pages print (tests/golden/page_figures.txt, each line cited)."""
    kinds = {"full": FULL, "causal": CAUSAL, "sliding_window": WINDOW}
    n = 0
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, qty, N, d, heads, mask, window, printed, check = [x.strip() for x in line.split("|")]
            N, d, heads, printed = int(N), int(d), int(heads), float(printed)
            w = None if window == "-" else int(window)
            kind = kinds[mask]
            pairs = orc.visible_pairs(N, kind, w)
            if qty == "pairs":
                got = pairs * heads
            elif qty == "fp16_bytes":
                got = 2 * pairs * heads
            elif qty == "flops":
                got = orc.attention_flops(1, heads, N, d, kind, w)
            elif qty == "ratio":
                got = orc.visible_pairs(N, FULL) / pairs
            else:
                raise ValueError(qty)
            if check == "gt":
                assert got > printed, (name, got, printed)
            else:
                tol = float(check.split(":")[1])
                assert abs(got / printed - 1.0) <= tol, (name, got, printed)
            n += 1
    assert n == 9


# ------------------------------------------------------------------ exact identities
def pin_window_ge_N_is_causal(orc):
    """window >= N is exactly causal attention (stanleyjacob.dev, "Using it on a
    real shape of problem": w = T and w = T + 1 give identical results)."""
    B, H, N, d = 1, 2, 37, 8
    q, k, v = _rand((B, H, N, d), 1), _rand((B, H, N, d), 2), _rand((B, H, N, d), 3)
    oc, lc = orc.attention(q, k, v, None, CAUSAL)
    for w in (N, N + 1, 10 * N):
        ow, lw = orc.attention(q, k, v, None, WINDOW, w)
        assert np.array_equal(oc, ow) and np.array_equal(lc, lw), w
    # a window shorter than N must differ (the mask is not ignored)
    ow, _ = orc.attention(q, k, v, None, WINDOW, N - 5)
    assert not np.allclose(oc, ow)


def pin_gqa_is_repeated_mha(orc):
    """GQA equals MHA on K/V repeated with ``repeat_interleave(Hq // Hkv, dim=1)``
    (tempatgunting.com, "Multi-Query and Grouped-Query Attention")."""
    B, Hq, N, d = 2, 6, 20, 8
    for Hkv in (1, 2, 3, 6):
        q = _rand((B, Hq, N, d), 10)
        k = _rand((B, Hkv, N, d), 11 + Hkv)
        v = _rand((B, Hkv, N, d), 21 + Hkv)
        kr = torch.from_numpy(k).repeat_interleave(Hq // Hkv, dim=1).numpy()
        vr = torch.from_numpy(v).repeat_interleave(Hq // Hkv, dim=1).numpy()
        for kind, w in ((FULL, None), (CAUSAL, None), (WINDOW, 4)):
            o1, l1 = orc.attention(q, k, v, 0.3, kind, w)
            o2, l2 = orc.attention(q, kr, vr, 0.3, kind, w)
            assert np.array_equal(o1, o2) and np.array_equal(l1, l2), (Hkv, kind)


def pin_rows_subset(orc):
    """Computing only some rows gives exactly those rows of the full result."""
    q, k, v = _rand((1, 3, 50, 8), 4), _rand((1, 1, 50, 8), 5), _rand((1, 1, 50, 8), 6)
    rows = np.array([49, 0, 17, 18, 31])
    for kind, w in ((FULL, None), (CAUSAL, None), (WINDOW, 9)):
        of, lf = orc.attention(q, k, v, None, kind, w)
        orr, lr = orc.attention(q, k, v, None, kind, w, rows=rows)
        assert np.array_equal(of[:, :, rows], orr) and np.array_equal(lf[:, :, rows], lr)


# ---------------------------------------------------------------------- closed forms
def pin_equal_keys_mean(orc):
    """All keys equal: every visible score of row i is the same c_i, so out_i is
    the plain mean of the visible v rows and lse_i = c_i + ln |V(i)|
    (masked entries get zero weight and the row renormalises over its visible
    set; stanleyjacob.dev, ``masked_attention``)."""
    B, H, N, d = 1, 2, 23, 6
    q = _rand((B, H, N, d), 7)
    k = np.broadcast_to(_rand((1, 1, 1, d), 8), (B, H, N, d)).copy()
    v = _rand((B, H, N, d), 9)
    scale = 0.7
    for kind, w in ((FULL, None), (CAUSAL, None), (WINDOW, 5)):
        out, lse = orc.attention(q, k, v, scale, kind, w)
        for h in range(H):
            for i in range(N):
                lo = {FULL: 0, CAUSAL: 0, WINDOW: max(0, i - 4)}[kind]
                hi = N if kind == FULL else i + 1
                c = scale * float(np.dot(q[0, h, i], k[0, h, 0]))
                np.testing.assert_allclose(out[0, h, i], v[0, h, lo:hi].mean(axis=0), rtol=0, atol=1e-12)
                np.testing.assert_allclose(lse[0, h, i], c + math.log(hi - lo), rtol=0, atol=1e-12)


def pin_dominant_key(orc):
    """One key whose score beats every other visible score by >= 100 returns
    its own v row (to within e^-100 * N)."""
    N, d = 16, 4
    q = np.zeros((1, 1, N, d)); q[..., 0] = 12.0
    k = _rand((1, 1, N, d), 30) * 0.01
    jstar = 3
    k[0, 0, jstar, 0] = 12.0
    v = _rand((1, 1, N, d), 31)
    out, lse = orc.attention(q, k, v, 1.0, CAUSAL)
    for i in range(jstar, N):
        np.testing.assert_allclose(out[0, 0, i], v[0, 0, jstar], rtol=0, atol=1e-30 + 1e-40)
        assert abs(lse[0, 0, i] - 144.0) < 1.0
    out, _ = orc.attention(q, k, v, 1.0, FULL)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(v[0, 0, jstar], (N, d)), rtol=0, atol=1e-30)


def pin_causal_row0_and_window1(orc):
    """Causal row 0 sees only key 0: out_0 = v_0, lse_0 = s_00.  A window of 1
    sees only the diagonal: out = V (through the head map), lse_i = s_ii."""
    B, Hq, Hkv, N, d = 2, 4, 2, 19, 8
    q, k, v = _rand((B, Hq, N, d), 40), _rand((B, Hkv, N, d), 41), _rand((B, Hkv, N, d), 42)
    scale = 0.37
    oc, lc = orc.attention(q, k, v, scale, CAUSAL)
    o1, l1 = orc.attention(q, k, v, scale, WINDOW, 1)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            assert np.array_equal(oc[b, h, 0], v[b, g, 0])
            assert abs(lc[b, h, 0] - scale * np.dot(q[b, h, 0], k[b, g, 0])) < 1e-12
            np.testing.assert_array_equal(o1[b, h], v[b, g])
            diag = scale * np.einsum("nd,nd->n", q[b, h], k[b, g])
            np.testing.assert_allclose(l1[b, h], diag, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- independent paths
def _brute(q, k, v, scale, kind, w):
    """Pure-Python restatement: per row, the list of visible keys, math.exp
    weights and math.fsum sums."""
    B, Hq, N, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0])
    out = [[[[0.0] * d for _ in range(N)] for _ in range(Hq)] for _ in range(B)]
    lse = [[[0.0] * N for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(N):
                if kind == FULL:
                    js = list(range(N))
                elif kind == CAUSAL:
                    js = list(range(0, i + 1))
                else:
                    js = [j for j in range(N) if i - w < j <= i]
                s = [scale * math.fsum(q[b][h][i][c] * k[b][g][j][c] for c in range(d)) for j in js]
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                tot = math.fsum(e)
                for c in range(d):
                    out[b][h][i][c] = math.fsum(e[t] * v[b][g][j][c] for t, j in enumerate(js)) / tot
                lse[b][h][i] = mx + math.log(tot)
    return np.array(out), np.array(lse)


def pin_brute_force_tiny(orc):
    """Tiny inputs against the pure-Python restatement, all masks, GQA."""
    for (B, Hq, Hkv, N, d, seed) in ((1, 1, 1, 1, 1, 50), (1, 2, 1, 5, 3, 51), (2, 4, 2, 8, 4, 52), (1, 3, 3, 7, 2, 53)):
        q, k, v = _rand((B, Hq, N, d), seed), _rand((B, Hkv, N, d), seed + 1), _rand((B, Hkv, N, d), seed + 2)
        for kind, w in ((FULL, None), (CAUSAL, None), (WINDOW, 1), (WINDOW, 3), (WINDOW, N + 1)):
            o, l = orc.attention(q, k, v, 0.61, kind, w)
            ob, lb = _brute(q.tolist(), k.tolist(), v.tolist(), 0.61, kind, w)
            np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
            np.testing.assert_allclose(l, lb, rtol=0, atol=1e-13)


def pin_torch_sdpa_fp64(orc):
    """torch's CPU float64 scaled_dot_product_attention with the same mask, and
    torch.logsumexp of the masked score matrix for the LSE: the float64 check of
    stanleyjacob.dev, "Using it on a real shape of problem" (B=2, H=8, T=2048,
    d=64, seed 0; is_causal=True and a window of 256 as an explicit mask)."""
    torch.manual_seed(0)
    B, H, T, d = 2, 8, 2048, 64
    q, k, v = torch.randn(3, B, H, T, d, dtype=torch.float64).unbind(0)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    cases = (
        (CAUSAL, None, dict(is_causal=True), j <= i),
        (WINDOW, 256, dict(attn_mask=(j <= i) & (j > i - 256)), (j <= i) & (j > i - 256)),
        (FULL, None, dict(), None),
    )
    for kind, w, kw, allowed in cases:
        ref = F.scaled_dot_product_attention(q, k, v, **kw)
        out, lse = orc.attention(q.numpy(), k.numpy(), v.numpy(), None, kind, w)
        assert float((torch.from_numpy(out) - ref).abs().max()) < 1e-12, kind
        s = (q @ k.transpose(-2, -1)) / math.sqrt(d)
        if allowed is not None:
            s = s.masked_fill(~allowed, float("-inf"))
        ref_lse = torch.logsumexp(s, dim=-1)
        assert float((torch.from_numpy(lse) - ref_lse).abs().max()) < 1e-11, kind


# ------------------------------------------------------------------------ invariants
def pin_invariants(orc):
    """Weights sum to one (V = 1 gives 1), out is linear in V, and a full mask is
    invariant under a joint permutation of the keys and values."""
    B, H, N, d = 1, 2, 31, 5
    q, k = _rand((B, H, N, d), 60), _rand((B, H, N, d), 61)
    v1, v2 = _rand((B, H, N, d), 62), _rand((B, H, N, d), 63)
    for kind, w in ((FULL, None), (CAUSAL, None), (WINDOW, 6)):
        o, _ = orc.attention(q, k, np.ones_like(v1), None, kind, w)
        np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)
        a, _ = orc.attention(q, k, v1, None, kind, w)
        b_, _ = orc.attention(q, k, v2, None, kind, w)
        c, _ = orc.attention(q, k, v1 + 2.0 * v2, None, kind, w)
        np.testing.assert_allclose(c, a + 2.0 * b_, rtol=0, atol=1e-12)
    perm = np.random.default_rng(64).permutation(N)
    o, l = orc.attention(q, k, v1, None, FULL)
    op, lp = orc.attention(q, k[:, :, perm], v1[:, :, perm], None, FULL)
    np.testing.assert_allclose(o, op, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, lp, rtol=0, atol=1e-12)


def pin_scale_convention(orc):
    """Default scale is 1/sqrt(d) (stanleyjacob.dev, ``masked_attention``), and
    the scale multiplies q.k before the softmax: with keys equal to the query of
    row i, lse carries scale * |q_i|^2."""
    q = _rand((1, 1, 9, 16), 70)
    k, v = q.copy(), _rand((1, 1, 9, 16), 71)
    o1, l1 = orc.attention(q, k, v, None, WINDOW, 1)
    np.testing.assert_allclose(l1[0, 0], (q[0, 0] ** 2).sum(-1) / 4.0, rtol=0, atol=1e-12)
    o2, l2 = orc.attention(q, k, v, 0.5, WINDOW, 1)
    np.testing.assert_allclose(l2[0, 0], (q[0, 0] ** 2).sum(-1) * 0.5, rtol=0, atol=1e-12)


ALL_PINS = [
    pin_mask_page3_form, pin_mask_row_structure, pin_visible_counts, pin_page_figures,
    pin_window_ge_N_is_causal, pin_gqa_is_repeated_mha, pin_rows_subset,
    pin_equal_keys_mean, pin_dominant_key, pin_causal_row0_and_window1,
    pin_brute_force_tiny, pin_torch_sdpa_fp64, pin_invariants, pin_scale_convention,
]
