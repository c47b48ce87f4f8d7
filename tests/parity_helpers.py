"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding, run the oracle on the same inputs (whole batch, or sampled rows with
only the blocks they reference copied to the host), and compare."""

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


def kv_code(cfg):
    return oracle.KV_E4M3 if cfg.kv_dtype == W.FP8_E4M3 else oracle.KV_BF16


def run_gpu(wl: W.Workload, partition_pages=0, out=None, ws=None, stream=None,
            schedule="auto"):
    c = wl.cfg
    if out is None:
        out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, c.num_kv_heads, c.scale,
              wl.block_tables, wl.seq_lens, c.block_size, c.max_seq_len, c.kv_dtype,
              wl.k_scale, wl.v_scale, workspace_tensor=ws, partition_pages=partition_pages,
              stream=stream, schedule=schedule)
    return out


def run_oracle(wl: W.Workload, pairs=None, threads=0):
    c = wl.cfg
    return oracle.pa_decode(wl.query.cpu(), wl.key_cache.cpu(), wl.value_cache.cpu(),
                            c.num_kv_heads, c.scale, wl.block_tables.cpu(), wl.seq_lens.cpu(),
                            c.block_size, kv_code(c), c.k_scale, c.v_scale, pairs=pairs,
                            threads=threads)


def run_oracle_sampled(wl: W.Workload, pairs, threads=0):
    """Oracle rows for (s, h) pairs, copying to the host only the blocks the
    sampled sequences reference (renumbered densely; the oracle's result does
    not depend on physical ids)."""
    c = wl.cfg
    seqs = sorted({s for s, _ in pairs})
    bt = wl.block_tables[seqs].cpu()
    ids = bt[bt >= 0].unique()
    remap = torch.full((c.num_blocks,), -1, dtype=torch.int64)
    remap[ids] = torch.arange(ids.numel())
    bt_new = torch.where(bt >= 0, remap[bt.clamp(min=0).long()], torch.tensor(-1)).to(torch.int32)
    ids_d = ids.to(wl.key_cache.device)
    kc = wl.key_cache[ids_d].cpu()
    vc = wl.value_cache[ids_d].cpu()
    q = wl.query[seqs].cpu()
    sl = wl.seq_lens[seqs].cpu()
    pos = {s: i for i, s in enumerate(seqs)}
    local = [(pos[s], h) for s, h in pairs]
    return oracle.pa_decode(q, kc, vc, c.num_kv_heads, c.scale, bt_new, sl, c.block_size,
                            kv_code(c), c.k_scale, c.v_scale, pairs=local, threads=threads)


def compare(got_bf16, ref64, kv_dtype, what=""):
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = TOL[kv_dtype]
    rms = float(np.sqrt(np.mean(ref ** 2))) or 1.0
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                 max_rel_rms=float(err.max() / rms))
    assert stats["max_abs"] <= tol["max_abs"], f"{what}: {stats}"
    assert stats["mean_abs"] <= tol["mean_abs"], f"{what}: {stats}"
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
