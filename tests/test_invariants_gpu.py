"""Bit-exact and structural checks of the CUDA path (GPU):

* one-hot probe: a single token dominates every other logit by ~500 in log2
  units, so every other weight underflows to exactly 0 in fp32 and the output
  is that token's V row -- bit-exact, swept over every position, across block
  and partition boundaries (this pins the block-table gather and the K/V page
  indexing bit for bit);
* relabelling physical blocks (moving their data) leaves the output bit-identical;
* uniform logits give the mean of V; seq_len 0 gives a zero row;
* illegal block ids / lengths set status bits without any out-of-range read.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _cfg(D=128, B=16, G=4, kv=W.BF16, lens=(37, 200, 16, 1), Hk=2, extra_blocks=7, seed=77):
    return W.PagedConfig(f"probe D={D} B={B} G={G} {kv}", num_seqs=len(lens), num_heads=Hk * G,
                         num_kv_heads=Hk, head_size=D, block_size=B,
                         num_blocks=sum(-(-t // B) for t in lens) + extra_blocks, seq_len_lo=1,
                         seq_len_hi=max(lens), kv_dtype=kv,
                         k_scale=0.05 if kv == W.FP8_E4M3 else 1.0,
                         v_scale=0.05 if kv == W.FP8_E4M3 else 1.0, seed=seed)


def _token_slot(wl, s, t):
    B = wl.cfg.block_size
    return int(wl.block_tables[s, t // B]), t % B


@pytest.mark.parametrize("kv", [W.BF16, W.FP8_E4M3, "fp8_compute"])
@pytest.mark.parametrize("D,B", [(128, 16), (64, 32), (128, 32)])
@pytest.mark.parametrize("pp", [0, 2, "balanced"])
def test_one_hot_probe_bit_exact(kv, D, B, pp):
    f8c = kv == "fp8_compute"
    if f8c:
        kv = W.FP8_E4M3
    # "balanced": one wave of CTAs over equal page ranges; this tiny batch gets
    # about one page per CTA, so every unit is cut and merged by the combine.
    schedule = "balanced" if pp == "balanced" else "auto"
    pp = 0 if pp == "balanced" else pp
    lens = (3 * B + 5, B, 1, 7 * B - 1)
    cfg = _cfg(D=D, B=B, G=4, kv=kv, lens=lens)
    wl = W.make_workload(cfg, DEV, seq_lens=list(lens))
    kc, vc = wl.key_cache, wl.value_cache
    x = cfg.x
    # zero the d=0 column of every referenced K slot (NaN poison elsewhere stays)
    for s, T in enumerate(lens):
        for t in range(T):
            pb, o = _token_slot(wl, s, t)
            kc[pb, :, 0, o, 0] = 0
    q = torch.zeros_like(wl.query)
    q[:, :, 0] = 4096.0
    wl.query = q
    one = 1.0 if kv == W.BF16 else 0x7E  # bf16 1.0 / e4m3 code of 448
    for s, T in enumerate(lens):
        for t_star in sorted({0, T // 2, T - 1, min(B, T - 1), min(2 * B - 1, T - 1)}):
            pb, o = _token_slot(wl, s, t_star)
            old = kc[pb, :, 0, o, 0].clone()
            kc[pb, :, 0, o, 0] = one if kv == W.BF16 else torch.full_like(old, one)
            if f8c:
                out = torch.empty_like(wl.query)
                pa.decode(out, wl.query, kc, wl.value_cache, cfg.num_kv_heads, cfg.scale,
                          wl.block_tables, wl.seq_lens, B, cfg.max_seq_len, kv, wl.k_scale,
                          wl.v_scale, partition_pages=pp, fp8_compute=True, schedule=schedule)
            else:
                out = run_gpu(wl, partition_pages=pp, schedule=schedule)
            torch.cuda.synchronize()
            for g in range(cfg.num_kv_heads):
                v = wl.value_cache[pb, g, :, o]
                if kv == W.BF16:
                    want = v
                else:
                    want = (v.view(torch.float8_e4m3fn).float() * cfg.v_scale).to(torch.bfloat16)
                for h in range(g * cfg.group, (g + 1) * cfg.group):
                    got = out[s, h]
                    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), \
                        (s, t_star, h, got[:4], want[:4])
            kc[pb, :, 0, o, 0] = old


@pytest.mark.parametrize("kv", [W.BF16, W.FP8_E4M3])
def test_block_relabelling_bit_identical(kv):
    lens = [500, 33, 129]
    cfg = _cfg(kv=kv, lens=lens, extra_blocks=20, G=8)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    a = run_gpu(wl).clone()
    g = torch.Generator().manual_seed(5)
    perm = torch.randperm(cfg.num_blocks, generator=g).to(DEV)
    kc2 = torch.empty_like(wl.key_cache)
    vc2 = torch.empty_like(wl.value_cache)
    kc2[perm] = wl.key_cache
    vc2[perm] = wl.value_cache
    bt = wl.block_tables.long()
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32)
    wl.key_cache, wl.value_cache, wl.block_tables = kc2, vc2, bt2.contiguous()
    b = run_gpu(wl)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_uniform_logits_mean():
    lens = [1000, 17]
    cfg = _cfg(lens=lens, G=8)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    wl.query = torch.zeros_like(wl.query)
    out = run_gpu(wl)
    torch.cuda.synchronize()
    ref = run_oracle(wl)
    compare(out, ref, cfg.kv_dtype, "uniform logits")


def test_zero_length_sequence_and_split_agreement():
    lens = [0, 300, 0, 4096, 5]
    cfg = _cfg(lens=lens, G=4)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ref = run_oracle(wl)
    outs = []
    for pp in (0, 1, 2, 7, 1000):
        o = run_gpu(wl, partition_pages=pp)
        torch.cuda.synchronize()
        compare(o, ref, cfg.kv_dtype, f"pp={pp}")
        assert (o[0] == 0).all() and (o[2] == 0).all()
        outs.append(o.float())
    for o in outs[1:]:
        # Each partitioning rounds the softmax weights to bf16 against its own
        # running max, so results differ by O(2^-9 / sqrt(T)) absolute, not by
        # a relative bf16 ulp; they must agree far inside the oracle tolerance.
        d = (o - outs[0]).abs()
        assert d.max().item() <= 2e-3 and d.mean().item() <= 1e-4, (d.max(), d.mean())


def test_non_default_stream():
    cfg = W.reduced(3, num_seqs=3, seq_len_hi=900, seq_len_lo=100)
    wl = W.make_workload(cfg, DEV)
    st = torch.cuda.Stream(DEV)
    out = torch.empty_like(wl.query)
    st.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(st):
        run_gpu(wl, out=out, stream=st)
    st.synchronize()
    compare(out, run_oracle(wl), cfg.kv_dtype, "side stream")


def _split_pair():
    """Two batches of the same shape and different data, decoded with forced
    partitions so that every call runs the decode and the combine kernel."""
    lens = [1000, 37, 700, 2000]
    wa = W.make_workload(_cfg(lens=lens, G=4, seed=301), DEV, seq_lens=lens)
    wb = W.make_workload(_cfg(lens=lens, G=4, seed=302), DEV, seq_lens=lens)
    return wa, wb


def test_back_to_back_calls_sharing_a_workspace():
    """Calls queued back to back on one stream with one workspace: each
    kernel is launched while the one ahead of it drains (dependent launch) and
    must still see the inputs and partials in stream order.  The outputs equal
    those of calls separated by a device synchronisation, bit for bit."""
    wa, wb = _split_pair()
    c = wa.cfg
    ws = torch.zeros(pa.workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size,
                                       c.block_size, c.max_seq_len, c.kv_dtype,
                                       partition_pages=3), dtype=torch.uint8, device=DEV)
    alone = []
    for wl in (wa, wb):
        alone.append(run_gpu(wl, partition_pages=3, ws=ws))
        torch.cuda.synchronize()
    outs = [torch.empty_like(wa.query) for _ in range(6)]
    for i, o in enumerate(outs):
        run_gpu((wa, wb)[i % 2], partition_pages=3, ws=ws, out=o)
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        assert torch.equal(o, alone[i % 2]), f"call {i}"
    compare(alone[1], run_oracle(wb), c.kv_dtype, "second batch")
    _merge_counts_are_zero(ws)


def _merge_counts_are_zero(ws):
    """The in-kernel merge leaves every unit's count at 0 after a call."""
    lo = pa.WORKSPACE_HEADER_BYTES
    assert not ws[lo:lo + pa.WORKSPACE_MERGE_COUNT_BYTES].any()


def test_calls_captured_in_a_cuda_graph():
    """The same sequence of calls captured in a CUDA graph (the dependent
    launches become graph edges) and replayed: bit-identical outputs."""
    wa, wb = _split_pair()
    c = wa.cfg
    ws = torch.zeros(pa.workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size,
                                       c.block_size, c.max_seq_len, c.kv_dtype,
                                       partition_pages=3), dtype=torch.uint8, device=DEV)
    alone = [run_gpu(wl, partition_pages=3, ws=ws) for wl in (wa, wb)]
    torch.cuda.synchronize()
    outs = [torch.zeros_like(wa.query) for _ in range(4)]
    st = torch.cuda.Stream(DEV)
    st.wait_stream(torch.cuda.current_stream(DEV))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(graph, stream=st):
            for i, o in enumerate(outs):
                run_gpu((wa, wb)[i % 2], partition_pages=3, ws=ws, out=o, stream=st)
    torch.cuda.current_stream(DEV).wait_stream(st)
    for _ in range(2):
        for o in outs:
            o.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for i, o in enumerate(outs):
            assert torch.equal(o, alone[i % 2]), f"graph call {i}"
        _merge_counts_are_zero(ws)
    del graph


@pytest.mark.parametrize("case", ["direct", "split", "cascade", "fp8_split"])
def test_writes_stay_inside_out_and_workspace(case):
    """Guard bands on both sides of `out` and of the workspace keep their
    sentinel values through a call that writes outputs (and, split or
    cascade, partials): no kernel writes outside the buffers it was given."""
    lens = [300, 37, 1000, 520]
    kv = W.FP8_E4M3 if case == "fp8_split" else W.BF16
    pref = 2 if case == "cascade" else 0
    cfg = _cfg(lens=lens, G=4, kv=kv, seed=411)
    if pref:
        cfg = cfg.replace(shared_prefix_blocks=pref)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    pp = 0 if case in ("direct", "cascade") else 3
    c = wl.cfg
    need = pa.workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                             c.max_seq_len, c.kv_dtype, partition_pages=pp,
                             shared_prefix_blocks=pref)
    G_WS = 256
    wbuf = torch.full((need + 2 * G_WS,), 0xA5, dtype=torch.uint8, device=DEV)
    wbuf[G_WS:G_WS + need].zero_()
    ws = wbuf[G_WS:G_WS + need]
    G_OUT = 64
    n = wl.query.numel()
    sentinel = -12288.0  # exact in bf16
    obuf = torch.full((n + 2 * G_OUT,), sentinel, dtype=torch.bfloat16, device=DEV)
    out = obuf[G_OUT:G_OUT + n].view(wl.query.shape)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, c.num_kv_heads, c.scale,
              wl.block_tables, wl.seq_lens, c.block_size, c.max_seq_len, c.kv_dtype,
              wl.k_scale, wl.v_scale, workspace_tensor=ws, partition_pages=pp,
              shared_prefix_blocks=pref)
    torch.cuda.synchronize()
    assert (obuf[:G_OUT] == sentinel).all() and (obuf[-G_OUT:] == sentinel).all()
    assert (wbuf[:G_WS] == 0xA5).all() and (wbuf[-G_WS:] == 0xA5).all()
    assert pa.read_status(ws) == 0
    if need > pa.WORKSPACE_HEADER_BYTES:
        _merge_counts_are_zero(ws)
    compare(out, run_oracle(wl), c.kv_dtype, case)


@pytest.mark.parametrize("kv", [W.FP8_E4M3, "fp8_compute", "bf16_d64"])
@pytest.mark.parametrize("bad,hot", [(2, 3), (3, 2), (4, 1)])
def test_bad_block_in_a_paired_stage(kv, bad, hot):
    """Small pages travel in pairs (logical blocks 0+1, 2+3, 4 of a 5-block
    sequence).  A bad block id in one page of a pair skips that page only:
    with a one-hot query on a token of another page, the output stays that
    token's V row bit for bit, and the bad-id flag is set."""
    f8c = kv == "fp8_compute"
    D = 64 if kv == "bf16_d64" else 128
    kv = W.BF16 if kv == "bf16_d64" else W.FP8_E4M3
    B = 16
    lens = [5 * B]
    cfg = _cfg(D=D, B=B, G=4, kv=kv, lens=lens, extra_blocks=4, seed=91)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    kc = wl.key_cache
    for t in range(lens[0]):
        pb, o = _token_slot(wl, 0, t)
        kc[pb, :, 0, o, 0] = 0
    q = torch.zeros_like(wl.query)
    q[:, :, 0] = 4096.0
    wl.query = q
    t_star = hot * B + 5
    pb, o = _token_slot(wl, 0, t_star)
    kc[pb, :, 0, o, 0] = 1.0 if kv == W.BF16 else torch.full_like(kc[pb, :, 0, o, 0], 0x7E)
    wl.block_tables[0, bad] = cfg.num_blocks + 7  # out of range
    ws = torch.zeros(pa.workspace_size(1, cfg.num_heads, cfg.num_kv_heads, D, B, lens[0], kv,
                                       fp8_compute=f8c), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, kc, wl.value_cache, cfg.num_kv_heads, cfg.scale, wl.block_tables,
              wl.seq_lens, B, cfg.max_seq_len, kv, wl.k_scale, wl.v_scale, workspace_tensor=ws,
              **({"fp8_compute": True} if f8c else {}))
    torch.cuda.synchronize()
    assert pa.read_status(ws) & pa.PA_DEV_BAD_BLOCK_ID
    for g in range(cfg.num_kv_heads):
        v = wl.value_cache[pb, g, :, o]
        if kv == W.BF16:
            want = v
        else:
            want = (v.view(torch.float8_e4m3fn).float() * cfg.v_scale).to(torch.bfloat16)
        for h in range(g * cfg.group, (g + 1) * cfg.group):
            assert torch.equal(out[0, h].view(torch.int16), want.view(torch.int16)), (g, h)


def test_bad_block_id_and_length_flags():
    lens = [100, 64]
    cfg = _cfg(lens=lens)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ws = torch.zeros(pa.workspace_size(2, cfg.num_heads, 2, 128, 16, 100), dtype=torch.uint8,
                     device=DEV)
    good = run_gpu(wl, ws=ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    bt = wl.block_tables.clone()
    wl.block_tables[0, 2] = cfg.num_blocks + 1000  # out of range
    wl.block_tables[1, 1] = -1
    out = run_gpu(wl, ws=ws)
    torch.cuda.synchronize()
    st = pa.read_status(ws, clear=True)
    assert st & pa.PA_DEV_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    # the skipped block's tokens drop out; other rows are untouched
    wl.block_tables = bt
    wl.seq_lens[1] = 10 ** 6  # longer than the block table row
    out = run_gpu(wl, ws=ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_SEQ_LEN_OUT_OF_RANGE
    assert torch.isfinite(out[0].float()).all()
    assert torch.equal(out[0], good[0])
    assert pa.read_status(ws) == 0


@pytest.mark.parametrize("nseq", [3, 17])
@pytest.mark.parametrize("kv", [W.BF16, W.FP8_E4M3])
@pytest.mark.parametrize("B", [16, 32])
def test_one_hot_probe_bit_exact_with_shared_prefix(kv, B, nseq):
    """Cascade decode: the probe token sits in the shared prefix (a shared
    block, so every sequence sees it) or in a sequence's own pages.  With 3
    sequences a kv head has one 16-row group (a prefix CTA per group); with
    17, five (prefix CTAs whose warps share one page ring, the last CTA's
    partly idle)."""
    pref = 5
    lens = ([pref * B + 3, pref * B, 9 * B + 1] * 6)[:nseq]
    cfg = W.PagedConfig(f"probe prefix B={B} {kv}", num_seqs=nseq, num_heads=8, num_kv_heads=2,
                        head_size=128, block_size=B,
                        num_blocks=pref + sum(-(-t // B) - pref for t in lens) + 6,
                        seq_len_lo=1, seq_len_hi=max(lens), kv_dtype=kv,
                        k_scale=0.05 if kv == W.FP8_E4M3 else 1.0,
                        v_scale=0.05 if kv == W.FP8_E4M3 else 1.0, shared_prefix_blocks=pref,
                        seed=91)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    kc = wl.key_cache
    for s, T in enumerate(lens):
        for t in range(T):
            pb, o = _token_slot(wl, s, t)
            kc[pb, :, 0, o, 0] = 0
    q = torch.zeros_like(wl.query)
    q[:, :, 0] = 4096.0
    wl.query = q
    one = 1.0 if kv == W.BF16 else 0x7E
    ws = torch.zeros(pa.workspace_size(nseq, 8, 2, 128, B, max(lens), kv, 2,
                                       shared_prefix_blocks=pref), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(wl.query)
    every = list(range(nseq))
    for t_star, seqs in [(0, every), (pref * B - 1, every), (2 * B + 3, every),
                         (pref * B + 2, [0]), (9 * B, [2])]:
        marks = []
        for s in seqs:
            pb, o = _token_slot(wl, s, t_star)
            marks.append((pb, o, kc[pb, :, 0, o, 0].clone()))
            kc[pb, :, 0, o, 0] = one if kv == W.BF16 else torch.full_like(marks[-1][2], one)
        pa.decode(out, wl.query, kc, wl.value_cache, 2, cfg.scale, wl.block_tables, wl.seq_lens,
                  B, max(lens), kv, wl.k_scale, wl.v_scale, workspace_tensor=ws,
                  partition_pages=2, shared_prefix_blocks=pref)
        torch.cuda.synchronize()
        assert pa.read_status(ws) == 0
        for s in seqs:
            pb, o = _token_slot(wl, s, t_star)
            for h in range(8):
                v = wl.value_cache[pb, h // 4, :, o]
                want = v if kv == W.BF16 else \
                    (v.view(torch.float8_e4m3fn).float() * cfg.v_scale).to(torch.bfloat16)
                assert torch.equal(out[s, h].view(torch.int16), want.view(torch.int16)), \
                    (s, t_star, h)
        for pb, o, old in reversed(marks):  # shared slots appear once per sequence
            kc[pb, :, 0, o, 0] = old


def test_wait_give_up_path_sets_status_and_leaves_context_usable():
    """With test_stall_copies every page barrier waits for bytes no copy sends
    (the copies themselves all land) and each wait gives up after ~20 ms: the
    kernel must drain, flag PA_DEV_WAIT_TIMEOUT and return; afterwards a normal
    decode on the same context is correct."""
    lens = [80]
    cfg = _cfg(lens=lens, G=4, Hk=1)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ws = torch.zeros(pa.workspace_size(1, 4, 1, 128, 16, 80), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, 1, cfg.scale, wl.block_tables,
              wl.seq_lens, 16, 80, workspace_tensor=ws, test_stall_copies=True)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_WAIT_TIMEOUT
    assert torch.isfinite(out.float()).all()
    good = run_gpu(wl, ws=ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(good, run_oracle(wl), cfg.kv_dtype, "after a give-up")


def test_wait_give_up_path_with_a_shared_prefix():
    """The prefix units' shared page ring under test_stall_copies: its waits
    give up too, the call ends with PA_DEV_WAIT_TIMEOUT and a finite output,
    and a normal call afterwards is correct."""
    lens = [700, 650, 900, 520, 610]
    cfg = _cfg(lens=lens, G=4, Hk=2, seed=515).replace(shared_prefix_blocks=20)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    c = wl.cfg
    ws = torch.zeros(pa.workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size,
                                       c.block_size, c.max_seq_len, c.kv_dtype,
                                       shared_prefix_blocks=20), dtype=torch.uint8, device=DEV)
    out = torch.full_like(wl.query, float("nan"))
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, c.num_kv_heads, c.scale,
              wl.block_tables, wl.seq_lens, c.block_size, c.max_seq_len, c.kv_dtype,
              wl.k_scale, wl.v_scale, workspace_tensor=ws, shared_prefix_blocks=20,
              test_stall_copies=True)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_WAIT_TIMEOUT
    assert torch.isfinite(out.float()).all()
    good = run_gpu(wl, ws=ws, shared_prefix_blocks=20)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(good, run_oracle(wl), c.kv_dtype, "prefix after a give-up")
