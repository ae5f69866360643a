"""Host model of the kernel's static schedule (super-items of row units r and
R-1-r, head unit by head unit, dealt round-robin to the persistent CTAs):
every work item is visited exactly once, and for causal masks every CTA gets
nearly the same number of KV tiles."""
import math

import pytest


def schedule(head_units, R, grid):
    per_head = (R + 1) // 2
    total = head_units * per_head
    rem = total % grid
    split = rem > 0 and 2 * rem <= grid
    split_from = total - rem if split else total
    out = []
    for cta in range(grid):
        items, g = [], cta
        while g < split_from:
            hu, s = divmod(g, per_head)
            items.append((hu, R - 1 - s))
            if R - 1 - s != s:
                items.append((hu, s))
            g += grid
        if split and cta < 2 * rem:
            hu, s = divmod(split_from + cta // 2, per_head)
            if cta % 2 == 0:
                items.append((hu, R - 1 - s))
            elif R - 1 - s != s:
                items.append((hu, s))
        out.append(items)
    return out


@pytest.mark.parametrize("head_units,R,grid", [(64, 32, 148), (32, 128, 148), (16, 512, 148), (3, 5, 4), (1, 1, 1),
                                              (7, 2, 148), (5, 9, 3), (16, 1024, 148), (3, 7, 8), (2, 3, 5)])
def test_every_item_once(head_units, R, grid):
    seen = [it for cta in schedule(head_units, R, grid) for it in cta]
    assert sorted(seen) == [(h, r) for h in range(head_units) for r in range(R)]


@pytest.mark.parametrize("name,head_units,R,cost", [
    ("dense (block pairs)", 64, 32, lambda r: 4 * r + 3),
    ("gqa (head pairs)", 32, 128, lambda r: r + 1),
    ("long (block pairs)", 32, 512, lambda r: 4 * r + 3),
])
def test_causal_balance(name, head_units, R, cost):
    loads = [sum(cost(r) for _, r in cta) for cta in schedule(head_units, R, 148)]
    ideal = sum(loads) / len(loads)
    assert max(loads) / ideal < 1.02, (name, max(loads) / ideal)


@pytest.mark.parametrize("name,head_units,R,cost", [
    ("long (block pairs)", 32, 512, lambda r: 4 * r + 3),
    ("swa (head pairs, equal units)", 16, 1024, lambda r: 33),
])
def test_split_last_round_shortens_the_tail(name, head_units, R, cost):
    # 8192 super-items on 148 CTAs leave 52 for a last round; dealt as 104
    # single row units that round is about half as long.
    loads = [sum(cost(r) for _, r in cta) for cta in schedule(head_units, R, 148)]
    ideal = sum(loads) / len(loads)
    assert max(loads) / ideal < 1.008, (name, max(loads) / ideal)
