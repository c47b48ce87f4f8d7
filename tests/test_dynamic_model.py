"""The dynamic schedule's claiming protocol, on the CPU.

The decode kernel's warps claim work through counters in the workspace: a
cursor hands each unit to its owners (partial slots 0 .. owners - 1: four
for a batch with at least half as many units as warps, else one); a unit's
page counter
hands out ranges of its pages, and each warp claims its next range while it
issues the current one; once the cursor is spent, warps join as helpers the
unit with the most pages left (at least two minimum claims) per warp on it,
taking slot owners + (helper counter), and only if that slot is below the
unit's limit K;
a warp that joins a unit with no pages left writes an empty partial.  The
combine then reads slots 0 .. owners + min(helpers, K - owners) - 1 of each
unit.

The protocol is written out here from that description, run with warps
interleaved at random (the order in which their atomics land), and checked:
every page of every unit is read exactly once, every slot the combine reads
was written by exactly one warp, and no warp writes a slot the combine does
not read.
"""

import random

import pytest


class Model:
    def __init__(self, pages, warps, k, owners=1, step_min=4, step_max=32, seed=0):
        self.n = list(pages)
        self.U = len(pages)
        self.W = warps
        self.K = k
        self.O = owners
        self.step_min, self.step_max = step_min, step_max
        self.rng = random.Random(seed)
        self.cursor = 0
        self.page_ctr = [0] * self.U
        self.helpers = [0] * self.U
        self.read = {}      # (unit, page) -> warp
        self.slots = {}     # (unit, slot) -> (warp, pages read)

    def step(self, left):
        st = max(self.step_min, min(self.step_max, left // 4))
        return st

    def warp(self, w):
        """A generator: each yield is one atomic of this warp."""
        cursor_done = False
        attempts = 0  # failed helper attempts since the last join (the kernel gives up at 16)
        empty = 0     # of them, probes that found nothing (the kernel gives up at 4)
        while True:
            joined = None
            while not cursor_done:
                e = self.cursor
                self.cursor += 1
                yield
                if e >= self.U * self.O:
                    cursor_done = True
                    break
                joined = (e // self.O, e % self.O)
                break
            if joined is None:
                best, best_score = None, 0.0
                probe = list(range(self.U))
                self.rng.shuffle(probe)
                for u in probe[:256]:
                    left = self.n[u] - self.page_ctr[u]
                    if left >= 2 * self.step_min and self.O + self.helpers[u] < self.K:
                        score = left / (2 + self.helpers[u])
                        if score > best_score:
                            best, best_score = u, score
                yield
                if best is None:
                    empty += 1
                    if empty == 4:
                        return
                    attempts += 1
                    if attempts == 16:
                        return
                    continue
                hs = self.helpers[best]
                self.helpers[best] += 1
                yield
                if self.O + hs >= self.K:
                    attempts += 1
                    if attempts == 16:
                        return
                    continue  # no slot: probe again
                joined = (best, self.O + hs)
            attempts = empty = 0
            u, slot = joined
            assert (u, slot) not in self.slots
            mine = []
            self.slots[(u, slot)] = (w, mine)
            # first range
            st = self.step(self.n[u])
            v = self.page_ctr[u]
            self.page_ctr[u] += st
            yield
            while v < self.n[u]:
                # claim the next range now, read the current one
                nst = self.step(self.n[u] - (v + st))
                nv = self.page_ctr[u]
                self.page_ctr[u] += nst
                yield
                for j in range(v, min(v + st, self.n[u])):
                    assert (u, j) not in self.read, (u, j)
                    self.read[(u, j)] = w
                    mine.append(j)
                v, st = nv, nst

    def run(self):
        gens = {w: self.warp(w) for w in range(self.W)}
        live = list(gens)
        while live:
            w = self.rng.choice(live)
            try:
                next(gens[w])
            except StopIteration:
                live.remove(w)


CASES = [
    ("many short units", [256] * 40, 32, None),
    ("few long units", [3072] * 8 + [1024] * 2, 64, None),
    ("ragged, empty units", [0, 5, 130, 4096, 1, 0, 77, 900, 33], 48, None),
    ("more units than warps", [64] * 100, 16, None),
    ("slot limit binds", [2000] * 3, 64, 4),
    ("four owners per unit", [256] * 30 + [70] * 10, 48, None),
]


@pytest.mark.parametrize("name,pages,warps,k", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("seed", range(5))
def test_every_page_once_and_every_read_slot_written(name, pages, warps, k, seed):
    units = len(pages)
    owners = 4 if 2 * units >= warps else 1
    if k is None:
        k = min(64, owners + -(-2 * warps // units) + 8)
    m = Model(pages, warps, k, owners=owners, seed=seed)
    m.run()
    # every page of every unit read exactly once
    want = {(u, j) for u, n in enumerate(pages) for j in range(n)}
    assert set(m.read) == want
    # the combine's slots of each unit are exactly the written ones
    for u in range(units):
        count = owners + min(m.helpers[u], k - owners)
        written = {s for (uu, s) in m.slots if uu == u}
        assert written == set(range(count)), (u, written, count)
    # pages of a slot belong to that slot's unit and warp
    for (u, s), (w, mine) in m.slots.items():
        for j in mine:
            assert m.read[(u, j)] == w
