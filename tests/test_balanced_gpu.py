"""The balanced schedule (one wave of CTAs over equal page ranges; units cut
at range ends are merged by the combine kernel) against the fp64 oracle and
against the partitioned schedule (GPU)."""

import pytest
import torch

import oracle
import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, kv_code, oracle_all_rows_cached, run_gpu, run_oracle
from test_parity import REDUCED
from test_random_shapes_gpu import _draw

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _ws(c, schedule="balanced", **kw):
    n = pa.workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                          c.max_seq_len, c.kv_dtype, schedule=schedule, **kw)
    return torch.zeros(n, dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_reduced_workloads(idx):
    cfg = REDUCED[idx]
    if cfg.shared_prefix_blocks:  # same sizes, no prefix declared: a pool for it
        cfg = W.reduced(idx, num_seqs=cfg.num_seqs, seq_len_hi=cfg.seq_len_hi,
                        seq_len_lo=cfg.seq_len_lo, shared_prefix_blocks=0)
    wl = W.make_workload(cfg, DEV)
    ws = _ws(cfg)
    out = run_gpu(wl, ws=ws, schedule="balanced")
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, run_oracle(wl), cfg.kv_dtype, f"balanced cfg{idx}")


@pytest.mark.parametrize("idx", [2, 4])
def test_full_size_all_rows(idx):
    cfg = W.WORKLOADS[idx]
    wl = W.make_workload(cfg, DEV)
    ws = _ws(cfg)
    out = run_gpu(wl, ws=ws, schedule="balanced")
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, oracle_all_rows_cached(wl), cfg.kv_dtype, f"balanced full cfg{idx} all rows",
            full_size=True)
    del wl, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("seed", range(9000, 9060))
def test_random_problem(seed):
    """The random problems of test_random_shapes_gpu that allow the balanced
    schedule (no shared prefix, no forced split)."""
    d = _draw(seed)
    if d["prefix"]:
        pytest.skip("shared prefix: partitioned only")
    lens = d["lens"]
    fp8 = d["kv"] == W.FP8_E4M3
    cfg = W.PagedConfig(f"random seed={seed}", num_seqs=len(lens), num_heads=d["Hk"] * d["G"],
                        num_kv_heads=d["Hk"], head_size=d["D"], block_size=d["B"],
                        num_blocks=sum(-(-t // d["B"]) for t in lens) + 6, seq_len_lo=0,
                        seq_len_hi=max(max(lens), 1), kv_dtype=d["kv"],
                        k_scale=0.05 if fp8 else 1.0, v_scale=0.04 if fp8 else 1.0, seed=seed)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    slopes = None
    if d["alibi"]:
        g = torch.Generator().manual_seed(seed)
        slopes = torch.rand(cfg.num_heads, generator=g, dtype=torch.float32) * 0.5
    ws = _ws(cfg, fp8_compute=d["fp8_compute"])
    out = torch.full_like(wl.query, float("nan"))
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, cfg.num_kv_heads, cfg.scale,
              wl.block_tables, wl.seq_lens, cfg.block_size, cfg.max_seq_len, cfg.kv_dtype,
              wl.k_scale, wl.v_scale, workspace_tensor=ws, schedule="balanced",
              alibi_slopes=None if slopes is None else slopes.to(DEV),
              **({"fp8_compute": True} if d["fp8_compute"] else {}))
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0, d
    ref = oracle.pa_decode(wl.query.cpu(), wl.key_cache.cpu(), wl.value_cache.cpu(),
                           cfg.num_kv_heads, cfg.scale, wl.block_tables.cpu(),
                           wl.seq_lens.cpu(), cfg.block_size, kv_code(cfg), cfg.k_scale,
                           cfg.v_scale, alibi_slopes=slopes)
    compare(out, ref, cfg.kv_dtype, str(d))


def test_zero_length_rows_and_agreement_with_partitions():
    lens = [0, 300, 0, 4096, 5, 0]
    cfg = W.PagedConfig("balanced zero rows", num_seqs=len(lens), num_heads=8, num_kv_heads=2,
                        head_size=128, block_size=16,
                        num_blocks=sum(-(-t // 16) for t in lens) + 4, seq_len_lo=0,
                        seq_len_hi=max(lens), seed=71)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ref = run_oracle(wl)
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, ws=_ws(cfg), schedule="balanced")
    other = run_gpu(wl, schedule="partitioned")
    torch.cuda.synchronize()
    compare(out, ref, cfg.kv_dtype, "balanced")
    for s in (0, 2, 5):
        assert (out[s] == 0).all()
    d = (out.float() - other.float()).abs()
    assert d.max().item() <= 2e-3 and d.mean().item() <= 1e-4


def test_length_flags():
    lens = [100, 64]
    cfg = W.PagedConfig("balanced flags", num_seqs=2, num_heads=4, num_kv_heads=2, head_size=64,
                        block_size=16, num_blocks=16, seq_len_lo=1, seq_len_hi=100, seed=73)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    wl.seq_lens[1] = -5
    ws = _ws(cfg)
    run_gpu(wl, ws=ws, schedule="balanced")
    torch.cuda.synchronize()
    assert pa.read_status(ws) & pa.PA_DEV_SEQ_LEN_OUT_OF_RANGE


def test_guard_bands_and_back_to_back_calls():
    """Sentinels around out and the workspace survive; calls queued back to
    back with one workspace (and replayed from a CUDA graph) match calls
    separated by a synchronisation, bit for bit."""
    lens = [1000, 37, 700, 2000]
    cfgs = [W.PagedConfig(f"balanced b2b {i}", num_seqs=4, num_heads=8, num_kv_heads=2,
                          head_size=128, block_size=16,
                          num_blocks=sum(-(-t // 16) for t in lens) + 4, seq_len_lo=1,
                          seq_len_hi=max(lens), seed=81 + i) for i in range(2)]
    wls = [W.make_workload(c, DEV, seq_lens=lens) for c in cfgs]
    need = pa.workspace_size(4, 8, 2, 128, 16, max(lens), schedule="balanced")
    wbuf = torch.full((need + 512,), 0xA5, dtype=torch.uint8, device=DEV)
    wbuf[256:256 + need].zero_()
    ws = wbuf[256:256 + need]
    n = wls[0].query.numel()
    obuf = torch.full((n + 128,), -12288.0, dtype=torch.bfloat16, device=DEV)
    out = obuf[64:64 + n].view(wls[0].query.shape)
    run_gpu(wls[0], out=out, ws=ws, schedule="balanced")
    torch.cuda.synchronize()
    assert (obuf[:64] == -12288.0).all() and (obuf[-64:] == -12288.0).all()
    assert (wbuf[:256] == 0xA5).all() and (wbuf[-256:] == 0xA5).all()
    compare(out, run_oracle(wls[0]), W.BF16, "balanced guard bands")
    alone = []
    for wl in wls:
        alone.append(run_gpu(wl, ws=ws, schedule="balanced"))
        torch.cuda.synchronize()
    outs = [torch.empty_like(out) for _ in range(4)]
    for i, o in enumerate(outs):
        run_gpu(wls[i % 2], ws=ws, out=o, schedule="balanced")
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        assert torch.equal(o, alone[i % 2]), f"queued call {i}"
    st = torch.cuda.Stream(DEV)
    st.wait_stream(torch.cuda.current_stream(DEV))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(graph, stream=st):
            for i, o in enumerate(outs):
                run_gpu(wls[i % 2], ws=ws, out=o, stream=st, schedule="balanced")
    torch.cuda.current_stream(DEV).wait_stream(st)
    for o in outs:
        o.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        assert torch.equal(o, alone[i % 2]), f"graph call {i}"
    del graph
