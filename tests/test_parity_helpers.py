"""The parity tests' host-side oracle drivers (CPU): the chunked whole-batch
run and the sampled-row run copy only the blocks their sequences reference
and renumber them; both must give, bit for bit, the rows of the plain oracle
over the whole batch."""

import numpy as np
import pytest
import torch

from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import REL_ROW_BOUND, compare, run_oracle, run_oracle_all, run_oracle_sampled

CASES = {
    "gqa ragged": W.reduced(3, num_seqs=6, seq_len_hi=900, seq_len_lo=1),
    "fp8": W.reduced(4, num_seqs=3, seq_len_hi=400, seq_len_lo=200),
    "shared prefix b32": W.reduced(5, num_seqs=3, seq_len_hi=1500, seq_len_lo=1100,
                                   shared_prefix_blocks=20),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_chunked_and_sampled_rows_equal_the_whole_batch(name):
    cfg = CASES[name]
    wl = W.make_workload(cfg, "cpu", seq_lens=None)
    whole = run_oracle(wl)
    per_seq = 2 * cfg.num_kv_heads * cfg.page_bytes() * cfg.max_blocks_per_seq
    for budget in (1, per_seq, 2 * per_seq + 1, 1 << 40):  # one sequence per chunk .. one chunk
        assert np.array_equal(run_oracle_all(wl, max_host_bytes=budget), whole), budget
    pairs = [(cfg.num_seqs - 1, 0), (0, cfg.num_heads - 1), (1, 3), (0, 0), (1, 3)]
    got = run_oracle_sampled(wl, pairs)
    for r, (s, h) in enumerate(pairs):
        assert np.array_equal(got[r], whole[s, h]), (s, h)


def test_zero_length_rows_are_checked_exactly():
    cfg = W.reduced(1, num_seqs=3, seq_len_hi=40, seq_len_lo=1)
    wl = W.make_workload(cfg, "cpu", seq_lens=[0, 17, 40])
    ref = run_oracle(wl)
    assert (ref[0] == 0).all()
    good = torch.from_numpy(ref).to(torch.bfloat16)
    compare(good, ref, W.BF16, "bf16 of the oracle itself")
    bad = good.clone()
    bad[0, 0, 0] = 1e-3  # a tiny value in a row that must be zero
    with pytest.raises(AssertionError):
        compare(bad, ref, W.BF16, "nonzero empty row")


def test_relative_bound_catches_a_scaled_long_row():
    """A long sequence's output is small (rms about sqrt(e / T)); a 7% error
    there passes the absolute bounds but not the relative one."""
    cfg = W.reduced(3, num_seqs=1, seq_len_hi=16384, seq_len_lo=16384)
    wl = W.make_workload(cfg, "cpu")
    ref = run_oracle(wl)
    assert np.sqrt(np.mean(ref ** 2)) < 0.02
    off = torch.from_numpy(ref * 1.07).to(torch.bfloat16)
    err = np.abs(off.double().numpy() - ref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3  # inside the absolute bar
    with pytest.raises(AssertionError):
        compare(off, ref, W.BF16, "7% too large")
    assert REL_ROW_BOUND < 0.1
