"""The split tail's bookkeeping, on the CPU.

The decode grid of a split-tail plan is n_full whole-unit CTAs followed by
tail_P CTAs per tail unit, partition-major: CTA b >= n_full takes tail unit
t = (b - n_full) mod n_tail, partition (b - n_full) div n_tail, i.e. unit
n_full + t.  Its pages are [part * tail_PP, (part + 1) * tail_PP) of that
unit, and its partial rows are (t * G + g) * tail_P + part.  The unit's
last CTA to count in merges the partitions that have pages.

Written out here from that description and checked over the planner's
actual plans (through the library, no GPU): every unit is covered once, every
page of every unit by exactly one CTA, no two CTAs share a partial row, the
partial rows fit the workspace the plan asks for, and the tail's CTAs all
come after every whole unit's.
"""

import itertools
import random

import pytest

import paged_kv_cache_471_b200 as pa


def _cover(plan, S, Hq, Hk, D, B, T):
    units = S * Hk
    G = Hq // Hk
    n_tail = plan["tail_units"]
    tP, tPP = plan["tail_partitions"], plan["tail_partition_pages"]
    n_full = units - n_tail
    pages = -(-T // B)
    grid = plan["grid_ctas"]
    assert grid == n_full + n_tail * tP
    seen_units, page_owner, rows = {}, {}, set()
    for b in range(grid):
        if b < n_full:
            u, part, lo, hi = b, 0, 0, pages
        else:
            t, part = (b - n_full) % n_tail, (b - n_full) // n_tail
            u = n_full + t
            lo, hi = part * tPP, min(pages, (part + 1) * tPP)
            for g in range(G):
                r = (t * G + g) * tP + part
                assert r not in rows
                rows.add(r)
        seen_units.setdefault(u, []).append(part)
        for j in range(lo, hi):
            assert (u, j) not in page_owner
            page_owner[(u, j)] = b
    assert sorted(seen_units) == list(range(units))
    for u, parts in seen_units.items():
        assert sorted(parts) == (list(range(tP)) if u >= n_full else [0])
    assert len(page_owner) == units * pages
    # tail CTAs follow every whole unit's
    assert all(page_owner[(u, 0)] < n_full for u in range(n_full))
    # partial rows fit the workspace: header, tail counts, (D + 2) floats per row
    need = (pa.WORKSPACE_HEADER_BYTES + pa.WORKSPACE_MERGE_COUNT_BYTES
            + len(rows) * (D + 2) * 4)
    assert max(rows, default=-1) < n_tail * G * tP
    assert plan["workspace_bytes"] >= need
    assert n_tail <= pa.WORKSPACE_MERGE_COUNT_BYTES // 4


SHAPES = [(S, Hq, Hk, D, B, T) for S, (Hq, Hk), D, B, T in itertools.product(
    (16, 37, 64, 128), ((8, 8), (32, 8), (32, 32), (64, 8)), (64, 128), (16, 32),
    (1024, 4096, 5000))]


@pytest.mark.parametrize("sms", [148, 40, 13])
def test_tail_mapping_covers_every_page_once(sms):
    rng = random.Random(sms)
    checked = 0
    for S, Hq, Hk, D, B, T in rng.sample(SHAPES, 60):
        plan = pa.plan(S, Hq, Hk, D, B, T, "bf16", num_sms=sms)
        if plan["tail_units"] == 0:
            continue
        assert plan["num_partitions"] == 1 and plan["prefix_partitions"] == 0
        # the grid less the tail's extra CTAs is one CTA per unit
        assert plan["grid_ctas"] - plan["tail_units"] * (plan["tail_partitions"] - 1) == S * Hk
        _cover(plan, S, Hq, Hk, D, B, T)
        checked += 1
    assert checked > 0


def test_tail_units_are_the_last_partial_wave():
    for sms in (148, 40, 13):
        for S, Hq, Hk, D, B, T in SHAPES[::7]:
            plan = pa.plan(S, Hq, Hk, D, B, T, "bf16", num_sms=sms)
            if plan["tail_units"]:
                per_sm = None
                for k in (1, 2, 3):  # CTA slots per SM the planner used
                    slots = sms * k
                    units = S * Hk
                    paired = B == 16 and D == 64  # bf16 pages that go in pairs
                    waves_ok = 2 * slots <= units and (units < 4 * slots or paired)
                    if waves_ok and units % slots == plan["tail_units"]:
                        per_sm = k
                assert per_sm is not None, (S, Hq, Hk, D, B, T, sms, plan)
