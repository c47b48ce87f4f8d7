"""The host block manager (pa_bm_*) on CPU: blocks on demand, shared blocks
with reference counts, copy on write of a shared partly filled block, and
all-or-nothing failure; plus a randomised comparison with a plain Python model
of the same rules."""

import math

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import paged_kv_cache_471_b200 as pa


def test_blocks_are_allocated_on_demand():
    bm = pa.BlockManager(num_blocks=8, block_size=16, max_blocks_per_seq=4)
    s = bm.add_sequence()
    assert bm.export([s])[0][0].tolist() == [-1, -1, -1, -1]
    assert bm.append(s, 1) is None and bm.num_free_blocks() == 7
    assert bm.append(s, 15) is None and bm.num_free_blocks() == 7  # fills block 0
    assert bm.append(s, 1) is None and bm.num_free_blocks() == 6  # spills into block 1
    bt, sl = bm.export([s])
    assert bt[0].tolist() == [0, 1, -1, -1] and sl.tolist() == [17]


def test_fork_shares_blocks_and_free_returns_them():
    bm = pa.BlockManager(8, 4, 4)
    p = bm.add_sequence()
    bm.append(p, 8)  # two full blocks
    c = bm.fork(p)
    assert [bm.refcount(b) for b in (0, 1)] == [2, 2]
    assert bm.export([p, c])[0].tolist() == [[0, 1, -1, -1], [0, 1, -1, -1]]
    bm.free(p)
    assert [bm.refcount(b) for b in (0, 1)] == [1, 1] and bm.num_free_blocks() == 6
    bm.free(c)
    assert bm.num_free_blocks() == 8 and bm.refcount(0) == 0


def test_copy_on_write_only_for_a_shared_partial_block():
    bm = pa.BlockManager(16, 4, 8)
    p = bm.add_sequence()
    bm.append(p, 6)  # block 0 full, block 1 half full
    c1, c2 = bm.fork(p), bm.fork(p)
    cow = bm.append(c1, 1)
    assert cow == (1, 2)  # private copy of the shared, partly filled block
    assert bm.export([c1])[0][0].tolist()[:2] == [0, 2]
    assert bm.refcount(1) == 2 and bm.refcount(2) == 1
    assert bm.append(c1, 1) is None  # already private
    # a sequence whose last block is full never copies, even when shared
    q = bm.add_sequence()
    bm.append(q, 8)
    r = bm.fork(q)
    assert bm.append(r, 3) is None
    assert bm.export([q, r])[0][:, :2].tolist() == [[3, 4], [3, 4]]
    # once the other sharers are gone the block returns to the pool
    bm.free(p)
    bm.free(c2)
    assert bm.refcount(1) == 0


def test_out_of_blocks_changes_nothing():
    bm = pa.BlockManager(3, 4, 8)
    s = bm.add_sequence()
    bm.append(s, 10)  # 3 blocks
    before = bm.export([s])
    with pytest.raises(pa.PagedAttentionError) as e:
        bm.append(s, 5)
    assert e.value.status == pa.PA_ERR_OUT_OF_BLOCKS
    after = bm.export([s])
    assert np.array_equal(before[0], after[0]) and np.array_equal(before[1], after[1])
    bm2 = pa.BlockManager(100, 4, 2)
    x = bm2.add_sequence()
    with pytest.raises(pa.PagedAttentionError):
        bm2.append(x, 9)  # needs 3 blocks, the row holds 2
    assert bm2.seq_len(x) == 0


def test_bad_arguments():
    bm = pa.BlockManager(4, 4, 4)
    with pytest.raises(pa.PagedAttentionError):
        bm.fork(7)
    with pytest.raises(pa.PagedAttentionError):
        bm.free(0)
    with pytest.raises(pa.PagedAttentionError):
        pa.BlockManager(0, 4, 4)
    assert bm.refcount(99) == -1


class Model:
    """The rules written out plainly: a sequence is a list of block ids plus a
    length; a block's reference count is the number of live sequences listing
    it; growing into a partly filled block listed by another live sequence
    first replaces it with a fresh block."""

    def __init__(self, n, B, maxb):
        self.n, self.B, self.maxb = n, B, maxb
        self.seqs = {}

    def refs(self):
        r = {}
        for blocks, _ in self.seqs.values():
            for b in blocks:
                r[b] = r.get(b, 0) + 1
        return r

    def free_count(self):
        return self.n - len(self.refs())


@settings(max_examples=60, deadline=None)
@given(st.lists(st.tuples(st.sampled_from(["add", "fork", "free", "append"]),
                          st.integers(0, 7), st.integers(0, 40)), min_size=1, max_size=60))
def test_matches_plain_model(ops):
    B, N, MAXB = 4, 24, 6
    bm = pa.BlockManager(N, B, MAXB)
    m = Model(N, B, MAXB)
    live = []
    for op, pick, k in ops:
        if op == "add" or not live:
            s = bm.add_sequence()
            m.seqs[s] = ([], 0)
            live.append(s)
            continue
        s = live[pick % len(live)]
        if op == "fork":
            c = bm.fork(s)
            m.seqs[c] = (list(m.seqs[s][0]), m.seqs[s][1])
            live.append(c)
        elif op == "free":
            bm.free(s)
            del m.seqs[s]
            live.remove(s)
        else:
            blocks, L = m.seqs[s]
            need = math.ceil((L + k) / B)
            shared_partial = L % B != 0 and blocks and m.refs()[blocks[-1]] > 1
            fresh = need - len(blocks) + (1 if (k and shared_partial) else 0)
            expect_fail = k > 0 and (need > MAXB or fresh > m.free_count())
            try:
                cow = bm.append(s, k)
            except pa.PagedAttentionError as e:
                assert expect_fail and e.status == pa.PA_ERR_OUT_OF_BLOCKS
                continue
            assert not expect_fail
            bt, sl = bm.export([s])
            new_blocks = [b for b in bt[0].tolist() if b >= 0]
            if k and shared_partial:
                assert cow is not None and cow[0] == blocks[-1] and new_blocks[len(blocks) - 1] == cow[1]
            else:
                assert cow is None
            assert new_blocks[:len(blocks) - (1 if cow else 0)] == blocks[:len(blocks) - (1 if cow else 0)]
            m.seqs[s] = (new_blocks, L + k)
        # invariants against the model after every step
        refs = m.refs()
        assert bm.num_free_blocks() == m.free_count()
        for b in range(N):
            assert bm.refcount(b) == refs.get(b, 0)
        if live:
            bt, sl = bm.export(live)
            for i, s in enumerate(live):
                blocks, L = m.seqs[s]
                assert sl[i] == L and len(blocks) == math.ceil(L / B)
                assert bt[i].tolist() == blocks + [-1] * (MAXB - len(blocks))
