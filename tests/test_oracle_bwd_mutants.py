"""Plant plausible mistakes in the backward oracle (on the CPU) and check that
at least one pin catches each."""
import numpy as np
import pytest

from oracle import attention_bwd_fp64 as G
from tests import oracle_bwd_pins


def _scores_drop_d(p, dp):
    return p * dp


def _scores_sign(p, dp):
    return p * ((p * dp).sum(axis=1, keepdims=True) - dp)


def _scores_d_over_columns(p, dp):
    return p * (dp - (p * dp).sum(axis=0, keepdims=True))


def _probs_unmasked(q_head, k_head, scale, allowed):
    s = (q_head @ k_head.T) * scale
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def _probs_unnormalised(q_head, k_head, scale, allowed):
    s = np.where(allowed, (q_head @ k_head.T) * scale, -np.inf)
    return np.exp(s - s.max(axis=1, keepdims=True))


MUTANTS = {
    "softmax Jacobian without D": ("_grad_scores", _scores_drop_d),
    "softmax Jacobian sign": ("_grad_scores", _scores_sign),
    "D summed over columns": ("_grad_scores", _scores_d_over_columns),
    "dV without transpose": ("_grad_v", lambda p, do: p @ do),
    "dP from v transposed wrongly": ("_grad_probs", lambda do, vh: do @ vh[::-1].T),
    "dQ without scale": ("_grad_q", lambda ds, kh, scale: ds @ kh),
    "dK without scale": ("_grad_k", lambda ds, qh, scale: ds.T @ qh),
    "dK from dS not transposed": ("_grad_k", lambda ds, qh, scale: (ds @ qh) * scale),
    "mask ignored in P": ("_probs", _probs_unmasked),
    "P not normalised": ("_probs", _probs_unnormalised),
    "head map modular": ("kv_head_of", lambda hq, Hq, Hkv: hq % Hkv),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(G, attr, fn)
    caught = False
    for pin in oracle_bwd_pins.ALL_PINS:
        try:
            pin(G)
        except (AssertionError, ValueError, IndexError):
            caught = True
            break
    assert caught, f"no pin caught the planted mistake '{mutant}'"
