"""Plant plausible mistakes in the decoding oracle (on the CPU) and check that
at least one pin catches each."""
import numpy as np
import pytest

from oracle import attention_decode_fp64 as D
from tests import oracle_decode_pins


def _gather_logical(cache, table_row, page_size, lo, L):
    """Reads logical page p from physical page p (ignores the table)."""
    c = np.asarray(cache)
    out = np.empty((c.shape[1], L - lo, c.shape[3]))
    for pos in range(lo, L):
        out[:, pos - lo, :] = c[pos // page_size, :, pos % page_size, :]
    return out


def _gather_slot_swapped(cache, table_row, page_size, lo, L):
    """Uses the page index as the slot and the slot as the page."""
    c = np.asarray(cache)
    out = np.empty((c.shape[1], L - lo, c.shape[3]))
    for pos in range(lo, L):
        out[:, pos - lo, :] = c[int(table_row[pos % page_size]) % c.shape[0], :, (pos // page_size) % page_size, :]
    return out


def _softmax_no_log(s, v_rows):
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ v_rows) / l, m[:, 0]


def _softmax_unnormalised(s, v_rows):
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e @ v_rows, (m + np.log(l))[:, 0]


MUTANTS = {
    "queries at the first positions": ("query_positions", lambda L, Nq: np.arange(0, Nq)),
    "queries one position late": ("query_positions", lambda L, Nq: np.arange(L - Nq + 1, L + 1)),
    "window start one key late": ("first_needed_position",
                                  lambda L, Nq, kind, w=None: max(0, L - Nq - w + 2) if kind == 2 else 0),
    "window start one key early": ("first_needed_position",
                                   lambda L, Nq, kind, w=None: max(0, L - Nq - w) if kind == 2 else 0),
    "window start from the last query": ("first_needed_position",
                                         lambda L, Nq, kind, w=None: max(0, L - w) if kind == 2 else 0),
    "page table ignored": ("gather_positions", _gather_logical),
    "page and slot swapped": ("gather_positions", _gather_slot_swapped),
    "head map modular": ("kv_head_of", lambda hq, Hq, Hkv: hq % Hkv),
    "scale dropped": ("_scores", lambda qr, kr, scale: qr @ kr.T),
    "keys not transposed": ("_scores", lambda qr, kr, scale: (qr @ kr[::-1].T) * scale),
    "lse without the log-sum": ("_softmax_rows", _softmax_no_log),
    "softmax not normalised": ("_softmax_rows", _softmax_unnormalised),
    "mask ignored": ("visible", lambda i, j, kind, w=None: np.ones(np.broadcast(np.asarray(i), np.asarray(j)).shape,
                                                                  dtype=bool)),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(D, attr, fn)
    caught = False
    for pin in oracle_decode_pins.ALL_PINS:
        try:
            pin(D)
        except (AssertionError, ValueError, IndexError):
            caught = True
            break
    assert caught, f"no pin caught the planted mistake '{mutant}'"
