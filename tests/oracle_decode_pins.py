"""Pins of the fp64 decoding oracle to facts that do not come from it.

Each ``pin_*`` takes the decoding oracle module (or a patched copy) and raises
AssertionError when it disagrees with a fact fixed by the pages or by the
mathematics.  ``test_oracle_decode.py`` runs them on the real module;
``test_oracle_decode_mutants.py`` plants mistakes and checks each is caught.

The caches here are built by this file's own scatter (contiguous K/V cut into
pages and placed at random physical indices), not by the input generators.
"""
from __future__ import annotations

import math

import numpy as np

from oracle import attention_fp64 as fwd_oracle

FULL, CAUSAL, WINDOW = 0, 1, 2


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def scatter_to_pages(kv, lens, page_size, rng, keep_from=None, extra_pages=0, fill=0.0):
    """Cut contiguous per-sequence K (or V) [B, Hkv, Lmax, d] into pages.

    Returns (cache [num_pages, Hkv, page_size, d], table [B, width]) with the
    kept logical pages of every sequence at randomly permuted physical
    indices; slots and pages holding no kept position are set to ``fill``
    and table entries of dropped pages to -1."""
    B, Hkv, Lmax, d = kv.shape
    keep_from = np.zeros(B, dtype=np.int64) if keep_from is None else np.asarray(keep_from)
    first = [int(k) // page_size for k in keep_from]
    last = [(int(L) - 1) // page_size for L in lens]
    n = sum(l - f + 1 for f, l in zip(first, last)) + extra_pages
    perm = rng.permutation(n)
    cache = np.full((n, Hkv, page_size, d), fill, dtype=np.float64)
    width = max(last) + 1
    table = np.full((B, width), -1, dtype=np.int64)
    i = 0
    for b in range(B):
        for lp in range(first[b], last[b] + 1):
            phys = int(perm[i])
            i += 1
            table[b, lp] = phys
            p1 = min(int(lens[b]), (lp + 1) * page_size)
            cache[phys, :, :p1 - lp * page_size, :] = kv[b, :, lp * page_size:p1, :]
    return cache, table, perm


def _case(B, Hq, Hkv, Nq, d, lens, seed):
    rng = np.random.default_rng(seed)
    Lmax = max(lens)
    q_full = _rand((B, Hq, Lmax, d), rng)
    k = _rand((B, Hkv, Lmax, d), rng)
    v = _rand((B, Hkv, Lmax, d), rng)
    q = np.stack([q_full[b, :, lens[b] - Nq:lens[b], :] for b in range(B)])
    return rng, q_full, k, v, q


# (B, Hq, Hkv, Nq, d, lens, page_size, mask, window, scale)
FORWARD_CASES = (
    (2, 2, 2, 1, 8, (37, 5), 4, CAUSAL, None, None),
    (2, 4, 2, 3, 6, (21, 3), 4, CAUSAL, None, 0.37),
    (1, 4, 1, 2, 5, (19,), 2, FULL, None, None),
    (2, 4, 2, 1, 4, (30, 12), 4, WINDOW, 8, None),      # 30-1-8+1 = 22, not page-aligned
    (2, 2, 1, 3, 4, (27, 9), 4, WINDOW, 5, 0.8),        # 27-3-5+1 = 20, page-aligned
    (1, 2, 2, 4, 3, (4,), 2, CAUSAL, None, None),        # only the new tokens are cached
    (1, 2, 1, 1, 3, (1,), 16, WINDOW, 1, None),
)


def pin_matches_forward_last_rows(orc):
    """Decoding the last Nq positions through the page table equals the forward
    oracle's rows L-Nq .. L-1 of the contiguous sequence (the KV cache only
    avoids recomputing past keys and values)."""
    for n, (B, Hq, Hkv, Nq, d, lens, ps, kind, w, scale) in enumerate(FORWARD_CASES):
        rng, q_full, k, v, q = _case(B, Hq, Hkv, Nq, d, lens, 500 + n)
        kc, table, _ = scatter_to_pages(k, lens, ps, np.random.default_rng(600 + n), extra_pages=1)
        vc, table_v, _ = scatter_to_pages(v, lens, ps, np.random.default_rng(600 + n), extra_pages=1)
        assert (table == table_v).all()
        out, lse = orc.decode_attention(q, kc, vc, table, np.array(lens), scale, kind, w)
        for b in range(B):
            L = lens[b]
            ref_o, ref_l = fwd_oracle.attention(q_full[b:b + 1, :, :L], k[b:b + 1, :, :L], v[b:b + 1, :, :L],
                                                scale, kind, w, rows=np.arange(L - Nq, L))
            assert np.abs(out[b] - ref_o[0]).max() < 1e-12, (n, b, "out")
            assert np.abs(lse[b] - ref_l[0]).max() < 1e-12, (n, b, "lse")


def _build(B, Hq, Hkv, Nq, d, lens, ps, seed, keep_from=None, extra_pages=0, fill=0.0):
    rng, q_full, k, v, q = _case(B, Hq, Hkv, Nq, d, lens, seed)
    kc, table, perm = scatter_to_pages(k, lens, ps, np.random.default_rng(seed + 1), keep_from, extra_pages, fill)
    vc, table2, _ = scatter_to_pages(v, lens, ps, np.random.default_rng(seed + 1), keep_from, extra_pages, fill)
    assert (table == table2).all()
    return q, kc, vc, table


def pin_page_permutation_invariance(orc):
    """Where the pages sit in the pool does not change anything: two different
    physical placements give bitwise-identical results."""
    for kind, w in ((CAUSAL, None), (WINDOW, 6), (FULL, None)):
        lens = (29, 13, 8)
        a = _build(3, 4, 2, 2, 4, lens, 4, 700)
        rng, q_full, k, v, q = _case(3, 4, 2, 2, 4, lens, 700)
        kc2, t2, _ = scatter_to_pages(k, lens, 4, np.random.default_rng(999))
        vc2, _, _ = scatter_to_pages(v, lens, 4, np.random.default_rng(999))
        o1, l1 = orc.decode_attention(a[0], a[1], a[2], a[3], np.array(lens), None, kind, w)
        o2, l2 = orc.decode_attention(q, kc2, vc2, t2, np.array(lens), None, kind, w)
        assert not (a[3] == t2).all()
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2), kind


def pin_unread_slots_do_not_matter(orc):
    """NaN in every slot the step must not read (past the end of a sequence's
    last page, unused pool pages, and under a window the pages wholly before
    the oldest visible key, whose table entries are -1) leaves the result
    finite and bitwise equal to the zero-filled cache."""
    # the last window case puts every sequence's oldest visible key (33-2-8+1 = 24,
    # 8, 16) on a page boundary, so the page before it is dropped
    cases = ((CAUSAL, None, (23, 9, 16), 2), (WINDOW, 7, (40, 9, 26), 1), (WINDOW, 4, (24, 5, 12), 3),
             (FULL, None, (11, 3, 8), 1), (WINDOW, 8, (33, 17, 25), 2))
    for kind, w, lens, Nq in cases:
        keep = None
        if kind == WINDOW:
            keep = [max(0, L - Nq - w + 1) for L in lens]
        args = (3, 4, 2, Nq, 4, lens, 4, 800)
        qa, ka, va, ta = _build(*args, keep_from=keep, extra_pages=2, fill=0.0)
        qb, kb, vb, tb = _build(*args, keep_from=keep, extra_pages=2, fill=np.nan)
        assert np.isnan(kb).any()
        o1, l1 = orc.decode_attention(qa, ka, va, ta, np.array(lens), None, kind, w)
        o2, l2 = orc.decode_attention(qb, kb, vb, tb, np.array(lens), None, kind, w)
        assert np.isfinite(o2).all() and np.isfinite(l2).all(), (kind, w)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2), (kind, w)


def pin_single_cached_key(orc):
    """One cached key (L = 1, Nq = 1): out = v_0 and lse = scale * q . k_0."""
    rng = np.random.default_rng(11)
    q = _rand((1, 4, 1, 6), rng)
    k = _rand((1, 2, 1, 6), rng)
    v = _rand((1, 2, 1, 6), rng)
    kc, table, _ = scatter_to_pages(k, [1], 4, rng, extra_pages=3)
    vc = np.zeros_like(kc)
    vc[table[0, 0], :, 0, :] = v[0, :, 0, :]
    for kind, w in ((CAUSAL, None), (FULL, None), (WINDOW, 1)):
        out, lse = orc.decode_attention(q, kc, vc, table, np.array([1]), 0.5, kind, w)
        for h in range(4):
            g = h // 2
            assert np.allclose(out[0, h, 0], v[0, g, 0], rtol=0, atol=1e-15)
            assert abs(lse[0, h, 0] - 0.5 * float(q[0, h, 0] @ k[0, g, 0])) < 1e-13


def pin_equal_keys(orc):
    """All cached keys equal: every visible key gets the same weight, so out is
    the mean of the visible values and lse = s + ln(count)."""
    rng = np.random.default_rng(12)
    L, Nq, d, ps = 19, 3, 5, 4
    q = _rand((1, 2, Nq, d), rng)
    krow = _rand((d,), rng)
    k = np.broadcast_to(krow, (1, 1, L, d)).copy()
    v = _rand((1, 1, L, d), rng)
    kc, table, _ = scatter_to_pages(k, [L], ps, np.random.default_rng(3))
    vc, _, _ = scatter_to_pages(v, [L], ps, np.random.default_rng(3))
    for kind, w in ((CAUSAL, None), (WINDOW, 6), (FULL, None)):
        out, lse = orc.decode_attention(q, kc, vc, table, np.array([L]), None, kind, w)
        for h in range(2):
            for t in range(Nq):
                i = L - Nq + t
                if kind == FULL:
                    js = np.arange(L)
                elif kind == CAUSAL:
                    js = np.arange(i + 1)
                else:
                    js = np.arange(max(0, i - w + 1), i + 1)
                s = float(q[0, h, t] @ krow) / math.sqrt(d)
                assert np.abs(out[0, h, t] - v[0, 0, js].mean(axis=0)).max() < 1e-13, (kind, h, t)
                assert abs(lse[0, h, t] - (s + math.log(len(js)))) < 1e-12, (kind, h, t)


def pin_brute_force_tiny(orc):
    """Pure-Python restatement on tiny inputs: walk the page table by hand,
    score every visible cached key, exponentiate and sum with math.fsum."""
    cases = ((2, 4, 2, 2, 3, (7, 3), 2, CAUSAL, None, 0.9), (1, 2, 1, 3, 2, (6,), 4, WINDOW, 3, None),
             (2, 2, 2, 1, 3, (5, 2), 2, FULL, None, None), (1, 3, 3, 2, 2, (8,), 4, WINDOW, 1, 1.3))
    for n, (B, Hq, Hkv, Nq, d, lens, ps, kind, w, scale) in enumerate(cases):
        rng = np.random.default_rng(900 + n)
        q = _rand((B, Hq, Nq, d), rng)
        npages = sum((L - 1) // ps + 1 for L in lens) + 1
        kc = _rand((npages, Hkv, ps, d), rng)
        vc = _rand((npages, Hkv, ps, d), rng)
        perm = rng.permutation(npages)
        table = np.full((B, max((L - 1) // ps + 1 for L in lens)), -1)
        i = 0
        for b, L in enumerate(lens):
            for lp in range((L - 1) // ps + 1):
                table[b, lp] = perm[i]
                i += 1
        out, lse = orc.decode_attention(q, kc, vc, table, np.array(lens), scale, kind, w)
        sc = scale if scale is not None else 1.0 / math.sqrt(d)
        for b, L in enumerate(lens):
            for h in range(Hq):
                g = h * Hkv // Hq
                for t in range(Nq):
                    i_pos = L - Nq + t
                    terms = []
                    for j in range(L):
                        if kind == CAUSAL and j > i_pos:
                            continue
                        if kind == WINDOW and not (i_pos - w < j <= i_pos):
                            continue
                        page = int(table[b, j // ps])
                        kj = kc[page, g, j % ps]
                        vj = vc[page, g, j % ps]
                        s = sc * math.fsum(float(q[b, h, t, c]) * float(kj[c]) for c in range(d))
                        terms.append((s, vj))
                    mx = max(s for s, _ in terms)
                    ws = [math.exp(s - mx) for s, _ in terms]
                    tot = math.fsum(ws)
                    for c in range(d):
                        ref = math.fsum(wj * float(vj[c]) for wj, (_, vj) in zip(ws, terms)) / tot
                        assert abs(out[b, h, t, c] - ref) < 1e-13, (n, b, h, t, c)
                    assert abs(lse[b, h, t] - (mx + math.log(tot))) < 1e-13, (n, b, h, t)


ALL_PINS = (pin_matches_forward_last_rows, pin_page_permutation_invariance, pin_unread_slots_do_not_matter,
            pin_single_cached_key, pin_equal_keys, pin_brute_force_tiny)
