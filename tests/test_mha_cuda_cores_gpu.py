"""The CUDA-core form for one query head per kv head (pa_options
.mha_cuda_cores: q.K and P.V as fp32 FMAs instead of tensor-core tiles with
one real row) against the fp64 oracle (GPU), under the partitioned and the
dynamic schedules."""

import itertools

import pytest
import torch

import oracle
import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, kv_code, oracle_all_rows_cached, run_gpu, run_oracle
from test_parity import REDUCED

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SCHEDULES = ["partitioned", "dynamic"]


def _ws(c, schedule, **kw):
    n = pa.workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                          c.max_seq_len, c.kv_dtype, schedule=schedule, **kw)
    return torch.zeros(n, dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("idx,pp", [(1, 0), (1, 3), (2, 0), (2, 5)])
def test_reduced_mha_workloads(idx, pp, schedule):
    if schedule == "dynamic" and pp:
        pytest.skip("the dynamic schedule takes no forced partitions")
    cfg = REDUCED[idx]
    wl = W.make_workload(cfg, DEV)
    ws = _ws(cfg, schedule, partition_pages=pp)
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, ws=ws, partition_pages=pp, schedule=schedule, mha_cuda_cores=True)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, run_oracle(wl), cfg.kv_dtype, f"cuda cores cfg{idx} pp={pp} {schedule}")


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("D,B", list(itertools.product([64, 128], [16, 32])))
@pytest.mark.parametrize("alibi", [False, True], ids=["plain", "alibi"])
def test_shapes(D, B, schedule, alibi):
    Hk = 3
    lens = [1, B - 1, B, B + 1, 3 * B + 5, 17 * B - 1, 40 * B + 3, 0]
    cfg = W.PagedConfig(f"cuda cores D={D} B={B}", num_seqs=len(lens), num_heads=Hk,
                        num_kv_heads=Hk, head_size=D, block_size=B,
                        num_blocks=sum(-(-t // B) for t in lens) + 9, seq_len_lo=0,
                        seq_len_hi=max(lens), seed=5150 + D + B)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    slopes = torch.tensor([0.05, 0.2, 0.7], dtype=torch.float32) if alibi else None
    ref = oracle.pa_decode(wl.query.cpu(), wl.key_cache.cpu(), wl.value_cache.cpu(),
                           cfg.num_kv_heads, cfg.scale, wl.block_tables.cpu(),
                           wl.seq_lens.cpu(), cfg.block_size, kv_code(cfg), alibi_slopes=slopes)
    for pp in ((0, 4) if schedule == "partitioned" else (0,)):
        out = torch.full_like(wl.query, float("nan"))
        run_gpu(wl, out=out, partition_pages=pp, schedule=schedule, mha_cuda_cores=True,
                alibi_slopes=None if slopes is None else slopes.to(DEV))
        torch.cuda.synchronize()
        compare(out, ref, cfg.kv_dtype, f"{cfg.name} pp={pp} {schedule} alibi={alibi}")


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_full_size_llama_mha_all_rows(schedule):
    cfg = W.WORKLOADS[2]
    wl = W.make_workload(cfg, DEV)
    ws = _ws(cfg, schedule)
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, ws=ws, schedule=schedule, mha_cuda_cores=True)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, oracle_all_rows_cached(wl), cfg.kv_dtype,
            f"cuda cores full cfg2 all rows {schedule}", full_size=True)
    del wl, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("D,B", [(128, 16), (64, 16), (128, 32)])
def test_one_hot_probe_bit_exact(D, B, schedule):
    lens = (3 * B + 5, B, 1, 7 * B - 1)
    cfg = W.PagedConfig(f"cuda cores probe D={D} B={B}", num_seqs=len(lens), num_heads=2,
                        num_kv_heads=2, head_size=D, block_size=B,
                        num_blocks=sum(-(-t // B) for t in lens) + 7, seq_len_lo=1,
                        seq_len_hi=max(lens), seed=78)
    wl = W.make_workload(cfg, DEV, seq_lens=list(lens))
    kc = wl.key_cache

    def slot(s, t):
        return int(wl.block_tables[s, t // B]), t % B

    for s, T in enumerate(lens):
        for t in range(T):
            pb, o = slot(s, t)
            kc[pb, :, 0, o, 0] = 0
    q = torch.zeros_like(wl.query)
    q[:, :, 0] = 4096.0
    wl.query = q
    for s, T in enumerate(lens):
        for t_star in sorted({0, T // 2, T - 1, min(B, T - 1)}):
            pb, o = slot(s, t_star)
            old = kc[pb, :, 0, o, 0].clone()
            kc[pb, :, 0, o, 0] = 1.0
            out = run_gpu(wl, partition_pages=2 if schedule == "partitioned" else 0,
                          schedule=schedule, mha_cuda_cores=True)
            torch.cuda.synchronize()
            for h in range(2):
                want = wl.value_cache[pb, h, :, o]
                assert torch.equal(out[s, h].view(torch.int16), want.view(torch.int16)), \
                    (s, t_star, h)
            kc[pb, :, 0, o, 0] = old


def test_option_leaves_grouped_and_fp8_caches_on_the_tensor_cores():
    """The option applies to bf16 caches with one query head per kv head; a
    grouped or FP8 batch decodes as usual."""
    for idx in (3, 4):
        cfg = REDUCED[idx]
        wl = W.make_workload(cfg, DEV)
        out = run_gpu(wl, mha_cuda_cores=True)
        torch.cuda.synchronize()
        compare(out, run_oracle(wl), cfg.kv_dtype, f"option on cfg{idx}")
