"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding, run the oracle on the same inputs (whole batch, sampled rows, or
every row of a full-size batch in chunks of sequences, with only the blocks
they reference copied to the host), and compare."""

from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W

# Tolerances of the acceptance bar: bf16 KV max-abs 1e-2 and mean-abs 1e-3
# against the fp64 oracle; FP8 KV max-abs 2e-2 against the oracle fed the same
# dequantised values.
TOL = {W.BF16: dict(max_abs=1e-2, mean_abs=1e-3), W.FP8_E4M3: dict(max_abs=2e-2, mean_abs=2e-3)}

# Relative bound, per output row: max_d |gpu - oracle| <= REL_ROW_BOUND * rms_d(oracle row),
# and the same for the whole output (max-abs over the rms of all rows).  The
# absolute bounds above stop constraining long rows: at 4096 tokens an output
# row's rms is about sqrt(e / T) = 0.026, at 131072 tokens 0.0046.  Where the
# bound comes from (u = 2^-8, the unit roundoff of bf16):
#   * the output is rounded to bf16 once: at most u |o_d|, and |o_d| / rms is
#     below about 5.5 over the millions of elements a full batch has;
#   * the softmax weights enter the P.V product rounded to bf16 (f16 for an
#     e4m3 cache, 2^-11; hi + lo e4m3 codes with FP8 compute, about 2^-8) and
#     the running sum uses the same rounded weights, so the result is an exact
#     weighted mean with each weight off by a relative delta_t, |delta_t| <= u.
#     Its error is sum_t p_t delta_t (v_t - o) / sum_t p_t, whose spread is
#     about (u / sqrt 3) * rms(o) whatever the length; over millions of
#     elements its largest value stays below about 6.5 of those, 3.7 u;
#   * fp32 accumulation and ex2.approx contribute about 2^-22 relative.
# Sum: about 9.2 u = 0.036; the bound leaves a third more for the tails.
REL_ROW_BOUND = 0.05

# Every comparison's statistics, in order; the session summary (conftest.py)
# prints the full-size ones and the worst of the rest.
PARITY_LOG: list = []


def kv_code(cfg):
    return oracle.KV_E4M3 if cfg.kv_dtype == W.FP8_E4M3 else oracle.KV_BF16


def run_gpu(wl: W.Workload, partition_pages=0, out=None, ws=None, stream=None,
            schedule="auto", **kw):
    c = wl.cfg
    if out is None:
        out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, c.num_kv_heads, c.scale,
              wl.block_tables, wl.seq_lens, c.block_size, c.max_seq_len, c.kv_dtype,
              wl.k_scale, wl.v_scale, workspace_tensor=ws, partition_pages=partition_pages,
              stream=stream, schedule=schedule, **kw)
    return out


def run_oracle(wl: W.Workload, pairs=None, threads=0):
    c = wl.cfg
    return oracle.pa_decode(wl.query.cpu(), wl.key_cache.cpu(), wl.value_cache.cpu(),
                            c.num_kv_heads, c.scale, wl.block_tables.cpu(), wl.seq_lens.cpu(),
                            c.block_size, kv_code(c), c.k_scale, c.v_scale, pairs=pairs,
                            threads=threads)


def sub_batch(wl: W.Workload, seqs):
    """Host copies of the inputs of sequences `seqs` only: their queries,
    lengths and block-table rows, and just the blocks those rows reference,
    renumbered densely (the oracle's result does not depend on physical ids)."""
    c = wl.cfg
    bt = wl.block_tables[seqs].cpu()
    ids = bt[bt >= 0].unique()
    remap = torch.full((c.num_blocks,), -1, dtype=torch.int64)
    remap[ids] = torch.arange(ids.numel())
    bt_new = torch.where(bt >= 0, remap[bt.clamp(min=0).long()], torch.tensor(-1)).to(torch.int32)
    ids_d = ids.to(wl.key_cache.device)
    return (wl.query[seqs].cpu(), wl.key_cache[ids_d].cpu(), wl.value_cache[ids_d].cpu(), bt_new,
            wl.seq_lens[seqs].cpu())


def run_oracle_sampled(wl: W.Workload, pairs, threads=0):
    """Oracle rows for (s, h) pairs, through the sub-batch of the sequences
    they name."""
    c = wl.cfg
    seqs = sorted({s for s, _ in pairs})
    q, kc, vc, bt, sl = sub_batch(wl, seqs)
    pos = {s: i for i, s in enumerate(seqs)}
    local = [(pos[s], h) for s, h in pairs]
    return oracle.pa_decode(q, kc, vc, c.num_kv_heads, c.scale, bt, sl, c.block_size,
                            kv_code(c), c.k_scale, c.v_scale, pairs=local, threads=threads)


def run_oracle_all(wl: W.Workload, threads=0, max_host_bytes=1 << 30):
    """Every output row [S, Hq, D] of a batch of any size: the oracle runs on
    consecutive chunks of whole sequences, each chunk's referenced blocks
    (about max_host_bytes of K+V at most, one sequence at least) copied to the
    host at a time."""
    c = wl.cfg
    S = c.num_seqs
    nbs = ((wl.seq_lens.cpu().to(torch.int64).clamp(min=0) + c.block_size - 1)
           // c.block_size).tolist()
    per_block = 2 * c.num_kv_heads * c.page_bytes()
    out = np.zeros((S, c.num_heads, c.head_size), dtype=np.float64)
    s0 = 0
    while s0 < S:
        s1, used = s0, 0
        while s1 < S and (s1 == s0 or used + nbs[s1] * per_block <= max_host_bytes):
            used += nbs[s1] * per_block
            s1 += 1
        seqs = list(range(s0, s1))
        q, kc, vc, bt, sl = sub_batch(wl, seqs)
        out[s0:s1] = oracle.pa_decode(q, kc, vc, c.num_kv_heads, c.scale, bt, sl, c.block_size,
                                      kv_code(c), c.k_scale, c.v_scale, threads=threads)
        s0 = s1
    return out


_ALL_ROWS_CACHE: dict = {}


def oracle_all_rows_cached(wl: W.Workload):
    """run_oracle_all of a seeded workload, kept for the session (the same
    config always draws the same inputs), for tests that do not modify them."""
    key = wl.cfg
    if key not in _ALL_ROWS_CACHE:
        _ALL_ROWS_CACHE[key] = run_oracle_all(wl)
    return _ALL_ROWS_CACHE[key]


def compare(got_bf16, ref64, kv_dtype, what="", full_size=False, rel_bound=REL_ROW_BOUND):
    """Element-by-element comparison with the oracle: max-abs and mean-abs
    against the acceptance bar, and max-abs relative to the rms of the
    oracle's rows (per row and over the whole output) against rel_bound.
    A row whose oracle value is all zeros (an empty sequence) must be exactly
    zero.  Returns the statistics; a passing comparison's are also kept in
    PARITY_LOG (a failing one's are in the assertion message)."""
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    D = ref.shape[-1]
    err = np.abs(got - ref)
    tol = TOL[kv_dtype]
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err_rows = err.reshape(-1, D).max(axis=1)
    rms_rows = np.sqrt(np.mean(ref.reshape(-1, D) ** 2, axis=1))
    live = rms_rows > 0
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                 max_abs_over_rms=float(err.max() / rms) if rms > 0 else 0.0,
                 max_row_rel=float((err_rows[live] / rms_rows[live]).max()) if live.any() else 0.0,
                 rows=int(err_rows.size))
    assert stats["max_abs"] <= tol["max_abs"], f"{what}: {stats}"
    assert stats["mean_abs"] <= tol["mean_abs"], f"{what}: {stats}"
    assert (err_rows[~live] == 0).all(), f"{what}: a zero row of the oracle is not zero: {stats}"
    assert stats["max_abs_over_rms"] <= rel_bound, f"{what}: {stats}"
    assert stats["max_row_rel"] <= rel_bound, f"{what}: {stats}"
    PARITY_LOG.append((what, stats, full_size))
    return stats


def sample_pairs(cfg, n, seed, max_seqs=4):
    """About n (sequence, q head) pairs drawn from at most max_seqs sequences
    (the first and last always among them), first and last head included."""
    g = torch.Generator().manual_seed(seed)
    S = cfg.num_seqs
    seqs = {0, S - 1}
    if S > 2:
        seqs |= set((1 + torch.randperm(S - 2, generator=g)[:max(0, max_seqs - 2)]).tolist())
    seqs = sorted(seqs)
    pairs = {(seqs[0], 0), (seqs[-1], cfg.num_heads - 1)}
    for _ in range(n):
        s = seqs[int(torch.randint(0, len(seqs), (1,), generator=g))]
        h = int(torch.randint(0, cfg.num_heads, (1,), generator=g))
        pairs.add((s, h))
    return sorted(pairs)
