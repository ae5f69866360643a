"""The decoding oracle against its pins (CPU only)."""
import numpy as np
import pytest

from oracle import attention_decode_fp64 as D
from tests import oracle_decode_pins


@pytest.mark.parametrize("pin", oracle_decode_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(D)


def test_rejects_stale_table_entry_inside_the_read_range():
    q = np.zeros((1, 1, 1, 2))
    cache = np.zeros((2, 1, 4, 2))
    table = np.array([[0, -1]])
    with pytest.raises(ValueError):
        D.decode_attention(q, cache, cache, table, np.array([6]))


def test_rejects_more_new_tokens_than_cached_keys():
    q = np.zeros((1, 1, 3, 2))
    cache = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        D.decode_attention(q, cache, cache, np.array([[0]]), np.array([2]))


def test_decode_bytes_counts_window_keys_only():
    # window 4096, one new token: keys L-4096 .. L-1 of each sequence
    n = D.decode_bytes(2, 32, 8, 1, 128, [10000, 300], 2, 4096)
    keys = 4096 + 300
    assert n == 2 * 2 * 128 * 8 * keys + 2 * 32 * 1 * (2 * 2 * 128 + 4)
