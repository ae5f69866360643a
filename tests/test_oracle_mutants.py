"""Plant plausible mistakes in the oracle (on the CPU) and check that at least
one pin catches each: the pins are strong enough to trust the oracle."""
import numpy as np
import pytest

import oracle
from oracle import attention_fp64 as A
from tests import oracle_pins

# Cheap pins first; the float64 SDPA pin is the slowest and runs last.
ORDER = [p for p in oracle_pins.ALL_PINS if p is not oracle_pins.pin_torch_sdpa_fp64] + [
    oracle_pins.pin_torch_sdpa_fp64]


def _visible_window_off_by_one(i, j, kind, window=None):
    if kind == A.MASK_SLIDING_WINDOW:
        return (np.asarray(j) <= i) & (np.asarray(j) >= np.asarray(i) - window)
    return _orig_visible(i, j, kind, window)


def _visible_causal_strict(i, j, kind, window=None):
    if kind == A.MASK_CAUSAL:
        return np.asarray(j) < np.asarray(i)
    return _orig_visible(i, j, kind, window)


_orig_visible = A.visible


def _count_off_by_one(N, kind, window=None):
    c = _orig_count(N, kind, window)
    return c - 1 if kind == A.MASK_SLIDING_WINDOW else c


_orig_count = A.visible_count_per_row


def _softmax_mask_dropped(s):
    s = np.where(np.isfinite(s), s, 0.0)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e, m, e.sum(axis=1, keepdims=True)


def _softmax_wrong_axis(s):
    m = s.max(axis=0, keepdims=True)
    e = np.exp(s - m)
    return e, s.max(axis=1, keepdims=True), e.sum(axis=1, keepdims=True)


MUTANTS = {
    "head map modular": ("kv_head_of", lambda hq, Hq, Hkv: hq % Hkv),
    "window edge off by one": ("visible", _visible_window_off_by_one),
    "causal strict": ("visible", _visible_causal_strict),
    "row count off by one": ("visible_count_per_row", _count_off_by_one),
    "scale dropped": ("_scores", lambda qr, kh, scale: qr @ kh.T),
    "scale squared": ("_scores", lambda qr, kh, scale: (qr @ kh.T) * scale * scale),
    "v applied transposed": ("_normalised_sum", lambda e, l, vh: (e.T @ vh) / l if e.shape[0] == e.shape[1] else (e @ vh[::-1]) / l),
    "no normalisation": ("_normalised_sum", lambda e, l, vh: e @ vh),
    "mask dropped in softmax": ("_softmax_terms", _softmax_mask_dropped),
    "max over wrong axis": ("_softmax_terms", _softmax_wrong_axis),
    "lse drops max": ("_log_sum_exp", lambda m, l: np.log(l)[:, 0]),
    "lse base 2": ("_log_sum_exp", lambda m, l: (m + np.log2(l))[:, 0]),
    "flops 2d per pair": ("attention_flops", lambda B, Hq, N, d, k, w=None: 2 * B * Hq * d * A.visible_pairs(N, k, w)),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(A, attr, fn)
    monkeypatch.setattr(oracle, attr, fn, raising=False)
    caught = []
    for pin in ORDER:
        try:
            pin(oracle)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
            break
    assert caught, f"no pin caught the planted mistake '{mutant}'"
