"""Bookkeeping of the balanced schedule, on the CPU.

The decode kernel walks each CTA's share of the (sequence, kv head, page)
order and writes a cut unit's partial into slot 2c + k of CTA c (k = 0 for
the first segment of its share, 1 for the last); pa_combine_kernel finds the
slots of a unit from its page offset alone.  Both rules are written out here
from their descriptions in the kernel header, one as a walk and one as the
lookup, and must agree: every cut unit's segments land in distinct slots,
the lookup names exactly those slots, and whole units get none.
"""

import random

import pytest


def pages(lengths, block):
    return [-(-t // block) for t in lengths]


def walk(n_pages, hk, grid):
    """What each CTA writes: {(s, kvh): [("out",) | ("slot", 2c + k, pages)]}."""
    total = hk * sum(n_pages)
    per = max(1, -(-total // grid))
    order = [(s, g) for s, n in enumerate(n_pages) if n for g in range(hk)]
    offsets, off = {}, 0
    for s, n in enumerate(n_pages):
        for g in range(hk):
            offsets[(s, g)] = off
            off += n
    writes = {}
    for c in range(grid):
        x0, x1 = c * per, min(total, (c + 1) * per)
        x = x0
        while x < x1:
            unit = next(u for u in order if offsets[u] <= x < offsets[u] + n_pages[u[0]])
            n = n_pages[unit[0]]
            j0 = x - offsets[unit]
            j1 = min(n, j0 + (x1 - x))
            if j0 == 0 and j1 == n:
                writes.setdefault(unit, []).append(("out",))
            else:
                k = 0 if x == x0 else 1
                writes.setdefault(unit, []).append(("slot", 2 * c + k, j1 - j0))
            x += j1 - j0
    return writes, per


def lookup(n_pages, hk, per, s, g):
    """The combine's view of unit (s, g): None if written directly, else slots."""
    c_s = sum(n_pages[:s])
    n = n_pages[s]
    if n == 0:
        return []
    off = hk * c_s + g * n
    c0, c1 = off // per, (off + n - 1) // per
    if c0 == c1:
        return None
    return [2 * c + (1 if (i == 0 and off != c0 * per) else 0)
            for i, c in enumerate(range(c0, c1 + 1))]


@pytest.mark.parametrize("seed", range(40))
def test_walk_and_lookup_agree(seed):
    r = random.Random(seed)
    block = r.choice([16, 32])
    hk = r.choice([1, 2, 3, 8])
    lengths = [r.choice([0, 1, block, r.randint(1, 40 * block)]) for _ in range(r.randint(1, 12))]
    grid = r.choice([1, 3, 7, 444])
    n_pages = pages(lengths, block)
    writes, per = walk(n_pages, hk, grid)
    used = set()
    for s, n in enumerate(n_pages):
        for g in range(hk):
            w = writes.get((s, g), [])
            want = lookup(n_pages, hk, per, s, g)
            if n == 0:
                assert w == [] and want == []  # a zero row, written by the combine
            elif want is None:
                assert w == [("out",)]
            else:
                slots = [x[1] for x in w]
                assert all(x[0] == "slot" for x in w)
                assert slots == want, (s, g, slots, want)
                assert sum(x[2] for x in w) == n  # the segments cover the unit once
                assert not used & set(slots)
                used |= set(slots)
    assert all(0 <= x < 2 * grid for x in used)
