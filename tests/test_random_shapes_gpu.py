"""Seeded random problems, CUDA path vs the fp64 oracle (GPU).

Each case draws its own head size, block size, group size (any divisor
structure up to 16 query heads per kv head), kv head count, cache type,
sequence lengths (zero, one token, ragged tails, block multiples), a forced
or planned split, and at most one of a declared shared prefix or ALiBi
slopes.  Every case is fixed by its seed, so a failure reproduces exactly.
"""

import random

import pytest
import torch

import oracle
import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, kv_code

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
N_CASES = 60


def _draw(seed):
    r = random.Random(seed)
    D = r.choice([64, 128])
    B = r.choice([16, 32])
    G = r.choice([1, 2, 3, 4, 5, 6, 7, 8, 12, 16])
    Hk = r.choice([1, 2, 3])
    kv = r.choice([W.BF16, W.FP8_E4M3])
    fp8_compute = kv == W.FP8_E4M3 and r.random() < 0.5
    S = r.randint(1, 9)
    mode = r.choice(["plain", "plain", "prefix", "alibi"])
    prefix = r.randint(1, 6) if mode == "prefix" else 0
    lens = []
    for _ in range(S):
        kind = r.random()
        if kind < 0.1 and not prefix:
            t = 0
        elif kind < 0.2:
            t = r.choice([1, B - 1, B, B + 1])
        elif kind < 0.35:
            t = B * r.randint(1, 40)
        else:
            t = r.randint(1, 60 * B)
        lens.append(max(t, prefix * B + r.randint(0, 2 * B)) if prefix else t)
    pp = r.choice([0, 0, 1, 2, 5, 13])
    return dict(D=D, B=B, G=G, Hk=Hk, kv=kv, fp8_compute=fp8_compute, lens=lens, pp=pp,
                prefix=prefix, alibi=mode == "alibi")


@pytest.mark.parametrize("seed", range(9000, 9000 + N_CASES))
def test_random_problem(seed):
    d = _draw(seed)
    lens = d["lens"]
    fp8 = d["kv"] == W.FP8_E4M3
    hi = max(max(lens), 1)
    cfg = W.PagedConfig(f"random seed={seed}", num_seqs=len(lens), num_heads=d["Hk"] * d["G"],
                        num_kv_heads=d["Hk"], head_size=d["D"], block_size=d["B"],
                        num_blocks=sum(-(-t // d["B"]) for t in lens) + 6, seq_len_lo=0,
                        seq_len_hi=hi, kv_dtype=d["kv"], k_scale=0.05 if fp8 else 1.0,
                        v_scale=0.04 if fp8 else 1.0, shared_prefix_blocks=d["prefix"],
                        seed=seed)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    slopes = None
    if d["alibi"]:
        g = torch.Generator().manual_seed(seed)
        slopes = torch.rand(cfg.num_heads, generator=g, dtype=torch.float32) * 0.5
    kw = dict(partition_pages=d["pp"], shared_prefix_blocks=d["prefix"])
    ws = torch.zeros(pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                       cfg.head_size, cfg.block_size, cfg.max_seq_len,
                                       cfg.kv_dtype, **kw), dtype=torch.uint8, device=DEV)
    out = torch.full_like(wl.query, float("nan"))
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, cfg.num_kv_heads, cfg.scale,
              wl.block_tables, wl.seq_lens, cfg.block_size, cfg.max_seq_len, cfg.kv_dtype,
              wl.k_scale, wl.v_scale, workspace_tensor=ws,
              alibi_slopes=None if slopes is None else slopes.to(DEV),
              **kw, **({"fp8_compute": True} if d["fp8_compute"] else {}))
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0, d
    ref = oracle.pa_decode(wl.query.cpu(), wl.key_cache.cpu(), wl.value_cache.cpu(),
                           cfg.num_kv_heads, cfg.scale, wl.block_tables.cpu(),
                           wl.seq_lens.cpu(), cfg.block_size, kv_code(cfg), cfg.k_scale,
                           cfg.v_scale, alibi_slopes=slopes)
    compare(out, ref, cfg.kv_dtype, str(d))
