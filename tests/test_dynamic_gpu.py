"""The dynamic schedule (persistent warps claiming pages from per-unit
counters, partials merged by the combine kernel) against the fp64 oracle
(GPU).

Which warp reads which pages depends on timing, so two calls may split a
unit differently and round differently: results are compared with the
oracle (and the bit-exact one-hot probe, which no split changes), not with
each other bit for bit.
"""

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


def _ws(c, shared_prefix_blocks=0, **kw):
    n = pa.workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                          c.max_seq_len, c.kv_dtype, schedule="dynamic",
                          shared_prefix_blocks=shared_prefix_blocks, **kw)
    return torch.zeros(n, dtype=torch.uint8, device=DEV)


def _decode(wl, ws, out=None, prefix=0, stream=None, **kw):
    return run_gpu(wl, out=out, ws=ws, stream=stream, schedule="dynamic",
                   shared_prefix_blocks=prefix, **kw)


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("prefix", [False, True], ids=["plain", "prefix"])
def test_reduced_workloads(idx, prefix):
    cfg = REDUCED[idx]
    if prefix and not cfg.shared_prefix_blocks:
        pytest.skip("no shared prefix in this workload")
    wl = W.make_workload(cfg, DEV)
    ws = _ws(cfg, cfg.shared_prefix_blocks if prefix else 0)
    out = torch.full_like(wl.query, float("nan"))
    _decode(wl, ws, out=out, prefix=cfg.shared_prefix_blocks if prefix else 0)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, run_oracle(wl), cfg.kv_dtype, f"dynamic cfg{idx} prefix={prefix}")


@pytest.mark.parametrize("idx", [2, 3, 4, 5])
def test_full_size_all_rows(idx):
    """Full workloads, in the bench's launch configuration apart from the
    schedule (config 5 with its shared prefix declared)."""
    cfg = W.WORKLOADS[idx]
    wl = W.make_workload(cfg, DEV)
    ws = _ws(cfg, cfg.shared_prefix_blocks)
    out = torch.full_like(wl.query, float("nan"))
    _decode(wl, ws, out=out, prefix=cfg.shared_prefix_blocks)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, oracle_all_rows_cached(wl), cfg.kv_dtype, f"dynamic full cfg{idx} all rows",
            full_size=True)
    del wl, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("seed", range(9000, 9060))
def test_random_problem(seed):
    """The seeded random problems of test_random_shapes_gpu (shared prefix,
    ALiBi and FP8 compute included; a forced split does not apply)."""
    d = _draw(seed)
    lens = d["lens"]
    fp8 = d["kv"] == W.FP8_E4M3
    cfg = W.PagedConfig(f"random seed={seed}", num_seqs=len(lens), num_heads=d["Hk"] * d["G"],
                        num_kv_heads=d["Hk"], head_size=d["D"], block_size=d["B"],
                        num_blocks=d["prefix"] + sum(max(-(-t // d["B"]) - d["prefix"], 0)
                                                     for t in lens) + 6,
                        seq_len_lo=0, seq_len_hi=max(max(lens), 1), kv_dtype=d["kv"],
                        k_scale=0.05 if fp8 else 1.0, v_scale=0.04 if fp8 else 1.0,
                        shared_prefix_blocks=d["prefix"], seed=seed)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    slopes = None
    if d["alibi"]:
        g = torch.Generator().manual_seed(seed)
        slopes = torch.rand(cfg.num_heads, generator=g, dtype=torch.float32) * 0.5
    ws = _ws(cfg, d["prefix"], fp8_compute=d["fp8_compute"])
    out = torch.full_like(wl.query, float("nan"))
    _decode(wl, ws, out=out, prefix=d["prefix"],
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
    cfg = W.PagedConfig("dynamic zero rows", num_seqs=len(lens), num_heads=8, num_kv_heads=2,
                        head_size=128, block_size=16,
                        num_blocks=sum(-(-t // 16) for t in lens) + 4, seq_len_lo=0,
                        seq_len_hi=max(lens), seed=71)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ref = run_oracle(wl)
    out = torch.full_like(wl.query, float("nan"))
    _decode(wl, _ws(cfg), out=out)
    other = run_gpu(wl, schedule="partitioned")
    torch.cuda.synchronize()
    compare(out, ref, cfg.kv_dtype, "dynamic zero rows")
    for s in (0, 2, 5):
        assert (out[s] == 0).all()
    d = (out.float() - other.float()).abs()
    assert d.max().item() <= 2e-3 and d.mean().item() <= 1e-4


def test_many_calls_in_a_row_with_one_workspace():
    """Each call's counters carry the workspace's generation number, which
    the last warp of the call moves on: calls queued back to back (two
    workloads of one shape, alternating) and the same calls replayed from a
    CUDA graph all match the oracle, and the guard bands around out and the
    workspace keep their sentinels."""
    lens = [1000, 37, 700, 2000]
    cfgs = [W.PagedConfig(f"dynamic b2b {i}", num_seqs=4, num_heads=8, num_kv_heads=2,
                          head_size=128, block_size=16,
                          num_blocks=sum(-(-t // 16) for t in lens) + 4, seq_len_lo=1,
                          seq_len_hi=max(lens), seed=81 + i) for i in range(2)]
    wls = [W.make_workload(c, DEV, seq_lens=lens) for c in cfgs]
    refs = [run_oracle(wl) for wl in wls]
    need = pa.workspace_size(4, 8, 2, 128, 16, max(lens), schedule="dynamic")
    wbuf = torch.full((need + 512,), 0xA5, dtype=torch.uint8, device=DEV)
    wbuf[256:256 + need].zero_()
    ws = wbuf[256:256 + need]
    n = wls[0].query.numel()
    obuf = torch.full((n + 128,), -12288.0, dtype=torch.bfloat16, device=DEV)
    out = obuf[64:64 + n].view(wls[0].query.shape)
    _decode(wls[0], ws, out=out)
    torch.cuda.synchronize()
    assert (obuf[:64] == -12288.0).all() and (obuf[-64:] == -12288.0).all()
    assert (wbuf[:256] == 0xA5).all() and (wbuf[-256:] == 0xA5).all()
    compare(out, refs[0], W.BF16, "dynamic guard bands")
    outs = [torch.full_like(out, float("nan")) for _ in range(6)]
    for i, o in enumerate(outs):
        _decode(wls[i % 2], ws, out=o)
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        compare(o, refs[i % 2], W.BF16, f"queued dynamic call {i}")
    st = torch.cuda.Stream(DEV)
    st.wait_stream(torch.cuda.current_stream(DEV))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(graph, stream=st):
            for i, o in enumerate(outs):
                _decode(wls[i % 2], ws, out=o, stream=st)
    torch.cuda.current_stream(DEV).wait_stream(st)
    for rep in range(2):
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for i, o in enumerate(outs):
            compare(o, refs[i % 2], W.BF16, f"graph replay {rep} call {i}")
    del graph
    assert (wbuf[:256] == 0xA5).all() and (wbuf[-256:] == 0xA5).all()
    assert pa.read_status(ws) == 0


@pytest.mark.parametrize("kv", [W.BF16, W.FP8_E4M3, "fp8_compute"])
@pytest.mark.parametrize("D,B", [(128, 16), (64, 32)])
def test_one_hot_probe_bit_exact(kv, D, B):
    """A single dominant token: its V row comes out bit for bit, however the
    warps split the unit (every other weight underflows to exactly 0)."""
    f8c = kv == "fp8_compute"
    if f8c:
        kv = W.FP8_E4M3
    lens = (3 * B + 5, B, 1, 7 * B - 1, 40 * B + 3)
    cfg = W.PagedConfig(f"dynamic probe D={D} B={B} {kv}", num_seqs=len(lens), num_heads=8,
                        num_kv_heads=2, head_size=D, block_size=B,
                        num_blocks=sum(-(-t // B) for t in lens) + 7, seq_len_lo=1,
                        seq_len_hi=max(lens), kv_dtype=kv,
                        k_scale=0.05 if kv == W.FP8_E4M3 else 1.0,
                        v_scale=0.05 if kv == W.FP8_E4M3 else 1.0, seed=77)
    wl = W.make_workload(cfg, DEV, seq_lens=list(lens))
    kc = wl.key_cache
    ws = _ws(cfg, fp8_compute=f8c)

    def slot(s, t):
        return int(wl.block_tables[s, t // B]), t % B

    for s, T in enumerate(lens):
        for t in range(T):
            pb, o = slot(s, t)
            kc[pb, :, 0, o, 0] = 0
    q = torch.zeros_like(wl.query)
    q[:, :, 0] = 4096.0
    wl.query = q
    one = 1.0 if kv == W.BF16 else 0x7E
    for s, T in enumerate(lens):
        for t_star in sorted({0, T // 2, T - 1, min(B, T - 1), min(9 * B + 2, T - 1)}):
            pb, o = slot(s, t_star)
            old = kc[pb, :, 0, o, 0].clone()
            kc[pb, :, 0, o, 0] = one if kv == W.BF16 else torch.full_like(old, one)
            out = torch.empty_like(wl.query)
            _decode(wl, ws, out=out, **({"fp8_compute": True} if f8c else {}))
            torch.cuda.synchronize()
            for g in range(cfg.num_kv_heads):
                v = wl.value_cache[pb, g, :, o]
                want = v if kv == W.BF16 else \
                    (v.view(torch.float8_e4m3fn).float() * cfg.v_scale).to(torch.bfloat16)
                for h in range(g * cfg.group, (g + 1) * cfg.group):
                    assert torch.equal(out[s, h].view(torch.int16), want.view(torch.int16)), \
                        (s, t_star, h)
            kc[pb, :, 0, o, 0] = old
    assert pa.read_status(ws) == 0


def test_flags():
    """Bad block ids, lengths beyond the block table and a broken shared
    prefix set their status bits, without any out-of-range read."""
    lens = [100, 64, 300]
    cfg = W.PagedConfig("dynamic flags", num_seqs=3, num_heads=8, num_kv_heads=2, head_size=128,
                        block_size=16, num_blocks=40, seq_len_lo=1, seq_len_hi=300, seed=73)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ref = run_oracle(wl)
    ws = _ws(cfg)
    compare(_decode(wl, ws), ref, W.BF16, "dynamic before the flags")
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    bt = wl.block_tables.clone()
    wl.block_tables[0, 2] = cfg.num_blocks + 1000
    wl.block_tables[1, 1] = -1
    out = _decode(wl, ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    wl.block_tables = bt
    wl.seq_lens[1] = 10 ** 6
    out = _decode(wl, ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_SEQ_LEN_OUT_OF_RANGE
    assert torch.isfinite(out.float()).all()
    compare(out[0:1], ref[0:1], W.BF16, "rows of a good sequence beside a bad one")
    wl.seq_lens[1] = -5
    _decode(wl, ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_SEQ_LEN_OUT_OF_RANGE

    pref = 3
    lens = [pref * 16 + 40, pref * 16 + 9, pref * 16 + 100]
    pc = W.PagedConfig("dynamic prefix flags", num_seqs=3, num_heads=8, num_kv_heads=2,
                       head_size=128, block_size=16,
                       num_blocks=pref + sum(-(-t // 16) - pref for t in lens) + 4, seq_len_lo=1,
                       seq_len_hi=max(lens), shared_prefix_blocks=pref, seed=74)
    wp = W.make_workload(pc, DEV, seq_lens=lens)
    wsp = _ws(pc, pref)
    wp.block_tables[2, 1] = wp.block_tables[2, pref]  # row 2's prefix differs from row 0's
    _decode(wp, wsp, prefix=pref)
    torch.cuda.synchronize()
    assert pa.read_status(wsp, clear=True) & pa.PA_DEV_PREFIX_MISMATCH


def test_wait_give_up_path_sets_status_and_leaves_context_usable():
    """With test_stall_copies every page barrier waits for bytes no copy
    sends (every copy still lands) and each wait gives up after ~20 ms: the
    warps drain, flag PA_DEV_WAIT_TIMEOUT and return, and the counters are
    left for the next call, which is correct."""
    lens = [80, 40]
    cfg = W.PagedConfig("dynamic give-up", num_seqs=2, num_heads=4, num_kv_heads=1,
                        head_size=128, block_size=16, num_blocks=12, seq_len_lo=1,
                        seq_len_hi=80, seed=75)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ws = _ws(cfg)
    out = torch.empty_like(wl.query)
    _decode(wl, ws, out=out, test_stall_copies=True)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_WAIT_TIMEOUT
    assert torch.isfinite(out.float()).all()
    for _ in range(2):
        good = _decode(wl, ws)
        torch.cuda.synchronize()
        assert pa.read_status(ws) == 0
        compare(good, run_oracle(wl), cfg.kv_dtype, "dynamic after a give-up")
