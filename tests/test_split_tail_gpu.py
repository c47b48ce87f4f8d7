"""The split tail (GPU): when (sequence, kv head) units are not split and fill
two or more waves of CTA slots, the units of the last, partial wave are cut
into partitions whose CTAs follow every whole unit's, and the last CTA of
each such unit merges its rows.  Checked against the fp64 oracle on reduced
batches planned for a smaller SM count (so that a small batch has a tail),
with mixed lengths (ranked longest first, so the tail holds the shortest
units), empty sequences, sequences within one tail partition, and one
workspace reused from a longer batch; and on the full-size workloads that
take it, through the allocation-free entry point as well."""

import ctypes

import pytest
import torch

import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, run_gpu, run_oracle
from test_parity import REDUCED

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _plan(cfg, sms, **kw):
    return pa.plan(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size,
                   cfg.block_size, cfg.max_seq_len, cfg.kv_dtype, num_sms=sms, **kw)


def _ws(cfg, sms, **kw):
    n = pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size,
                          cfg.block_size, cfg.max_seq_len, cfg.kv_dtype, num_sms=sms, **kw)
    return torch.zeros(n, dtype=torch.uint8, device=DEV)


# (workload, SM count to plan for): each plan has two or three waves of whole
# units and a tail
CASES = [(2, 9), (3, 5), (4, 3), (4, 4)]


@pytest.mark.parametrize("idx,sms", CASES)
def test_reduced_workloads_with_a_tail(idx, sms):
    cfg = REDUCED[idx]
    p = _plan(cfg, sms)
    units = cfg.num_seqs * cfg.num_kv_heads
    assert p["num_partitions"] == 1 and 0 < p["tail_units"] < units, p
    wl = W.make_workload(cfg, DEV)
    ws = _ws(cfg, sms)
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, ws=ws, num_sms=sms)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    ref = run_oracle(wl)
    compare(out, ref, cfg.kv_dtype, f"split tail cfg{idx} sms={sms}")
    # the partitioned schedule (no tail) on the same batch agrees too
    out2 = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out2, num_sms=sms, schedule="partitioned")
    torch.cuda.synchronize()
    compare(out2, ref, cfg.kv_dtype, f"no tail cfg{idx} sms={sms}")


def _mixed(B, lens, Hk=4, G=2, D=128, seed=0):
    return W.PagedConfig(f"split tail lengths B={B}", num_seqs=len(lens), num_heads=Hk * G,
                         num_kv_heads=Hk, head_size=D, block_size=B,
                         num_blocks=sum(-(-t // B) for t in lens) + 11, seq_len_lo=0,
                         seq_len_hi=max(lens), seed=seed)


@pytest.mark.parametrize("B", [16, 32])
def test_mixed_lengths_empty_and_short_units(B):
    # 40 sequences x 4 kv heads = 160 units for 16 SMs (48 slots): 16 tail
    # units, the shortest by rank -- empty ones, ones within one tail
    # partition, and ones spanning several.
    T = 64 * B  # 64 pages: tail partitions of 16 pages
    lens = [T, T - 1, 5, 0, 16 * B, 16 * B + 1, 3 * B + 7, T // 2] * 5
    cfg = _mixed(B, lens, seed=700 + B)
    sms = 16
    p = _plan(cfg, sms)
    assert p["tail_units"] == 160 % 48 and p["tail_partition_pages"] == 16, p
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ws = _ws(cfg, sms)
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, ws=ws, num_sms=sms)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, run_oracle(wl), cfg.kv_dtype, f"split tail mixed B={B}")


def test_equal_lengths_tail_of_index_order():
    # equal lengths keep index order: the tail is the last units by index
    lens = [64 * 16] * 37
    cfg = _mixed(16, lens, Hk=3, G=4, seed=77)
    sms = 12  # 36 slots; 111 units -> 3 in the tail
    p = _plan(cfg, sms)
    assert p["tail_units"] == 111 % 36
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    out = run_gpu(wl, num_sms=sms)
    torch.cuda.synchronize()
    compare(out, run_oracle(wl), cfg.kv_dtype, "split tail equal lengths")


def test_one_workspace_long_then_short():
    """A long batch fills every tail partition's slots; the same shape with
    short sequences then writes fewer, and must not read the stale ones."""
    T = 64 * 16
    long_lens = [T] * 40
    short_lens = [0, 1, 17, 16 * 16, 16 * 16 + 1, T, 5, 33] * 5
    cfg = _mixed(16, [T] * 40, seed=91)
    sms = 16
    ws = _ws(cfg, sms)
    for lens in (long_lens, short_lens):
        wl = W.make_workload(cfg, DEV, seq_lens=lens)
        out = torch.full_like(wl.query, float("nan"))
        run_gpu(wl, out=out, ws=ws, num_sms=sms)
        torch.cuda.synchronize()
        compare(out, run_oracle(wl), cfg.kv_dtype, f"split tail reuse {lens[:4]}")


@pytest.mark.parametrize("idx", [3, 4])
def test_full_size_noalloc_matches_workspace_call(idx):
    """The full GQA batch (1024 units) and the FP8 batch (2048 units of paired
    pages) take the split tail on this GPU; the allocation-free entry point
    (same plan, scratch in the library's own array) gives the same bits as a
    call with a caller workspace."""
    cfg = W.WORKLOADS[idx]
    p = pa.plan(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size, cfg.block_size,
                cfg.max_seq_len, cfg.kv_dtype)
    if p["tail_units"] == 0:
        pytest.skip("this GPU's CTA slots divide the batch's units")
    assert p["workspace_bytes"] <= pa.NOALLOC_SCRATCH_BYTES
    wl = W.make_workload(cfg, DEV)
    ref = run_gpu(wl)
    out = torch.full_like(wl.query, float("nan"))
    code = pa.kv_dtype_code(cfg.kv_dtype)
    fp8 = code == pa.PA_KV_FP8_E4M3
    L = pa.lib()
    rc = L.pa_decode_noalloc(
        out.data_ptr(), wl.query.data_ptr(), wl.key_cache.data_ptr(), wl.value_cache.data_ptr(),
        cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size, ctypes.c_float(cfg.scale),
        wl.block_tables.data_ptr(), wl.block_tables.shape[1], wl.seq_lens.data_ptr(),
        cfg.block_size, cfg.max_seq_len, cfg.num_blocks, code,
        wl.k_scale.data_ptr() if fp8 else None, wl.v_scale.data_ptr() if fp8 else None,
        torch.cuda.current_stream(DEV).cuda_stream)
    assert rc == pa.PA_OK, L.pa_last_error_detail()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    del wl, out, ref
    torch.cuda.empty_cache()


def _tail_counts(ws):
    lo = pa.WORKSPACE_HEADER_BYTES
    return ws[lo:lo + pa.WORKSPACE_MERGE_COUNT_BYTES]


def test_back_to_back_calls_graph_and_guard_bands():
    """Calls queued back to back on one workspace, and replayed twice from a
    CUDA graph, match calls separated by a synchronisation bit for bit; no
    byte outside out and the workspace changes; the split-tail counts are 0
    again after every call."""
    T = 64 * 16
    sms = 16
    lens_a = [T] * 40
    lens_b = [T, 5, 0, 17 * 16, T - 3, 33, 16 * 16, T] * 5
    cfg = _mixed(16, lens_a, seed=123)
    wls = [W.make_workload(cfg, DEV, seq_lens=l) for l in (lens_a, lens_b)]
    need = pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size,
                             cfg.block_size, cfg.max_seq_len, cfg.kv_dtype, num_sms=sms)
    wbuf = torch.full((need + 512,), 0xA5, dtype=torch.uint8, device=DEV)
    wbuf[256:256 + need].zero_()
    ws = wbuf[256:256 + need]
    n = wls[0].query.numel()
    obuf = torch.full((n + 128,), -12288.0, dtype=torch.bfloat16, device=DEV)
    out = obuf[64:64 + n].view(wls[0].query.shape)
    run_gpu(wls[1], out=out, ws=ws, num_sms=sms)
    torch.cuda.synchronize()
    assert (obuf[:64] == -12288.0).all() and (obuf[-64:] == -12288.0).all()
    assert (wbuf[:256] == 0xA5).all() and (wbuf[-256:] == 0xA5).all()
    assert not _tail_counts(ws).any()
    compare(out, run_oracle(wls[1]), cfg.kv_dtype, "split tail guard bands")
    alone = []
    for wl in wls:
        alone.append(run_gpu(wl, ws=ws, num_sms=sms))
        torch.cuda.synchronize()
    outs = [torch.empty_like(out) for _ in range(6)]
    for i, o in enumerate(outs):
        run_gpu(wls[i % 2], ws=ws, out=o, num_sms=sms)
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        assert torch.equal(o.view(torch.int16), alone[i % 2].view(torch.int16)), f"queued {i}"
    assert not _tail_counts(ws).any()
    st = torch.cuda.Stream(DEV)
    st.wait_stream(torch.cuda.current_stream(DEV))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(graph, stream=st):
            for i, o in enumerate(outs):
                run_gpu(wls[i % 2], ws=ws, out=o, stream=st, num_sms=sms)
    torch.cuda.current_stream(DEV).wait_stream(st)
    for _ in range(2):
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for i, o in enumerate(outs):
            assert torch.equal(o.view(torch.int16), alone[i % 2].view(torch.int16)), f"graph {i}"
        assert not _tail_counts(ws).any()
    del graph
    assert pa.read_status(ws) == 0


def test_workspace_shared_with_split_and_unsplit_plans():
    """One workspace for a batch split into partitions (its partials start
    after the split-tail counts) and then for a split-tail plan: the counts
    stay 0 and both match the oracle."""
    T = 64 * 16
    sms = 16
    cfg = _mixed(16, [T] * 40, seed=321)
    wl = W.make_workload(cfg, DEV, seq_lens=[T, T - 1, 40, 0, 16 * 16 + 1] * 8)
    ref = run_oracle(wl)
    need = max(pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size,
                                 cfg.block_size, cfg.max_seq_len, cfg.kv_dtype, num_sms=sms,
                                 partition_pages=pp) for pp in (0, 5))
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for pp in (5, 0, 5, 0):
        out = torch.full_like(wl.query, float("nan"))
        run_gpu(wl, out=out, ws=ws, num_sms=sms, partition_pages=pp)
        torch.cuda.synchronize()
        assert not _tail_counts(ws).any()
        compare(out, ref, cfg.kv_dtype, f"shared workspace pp={pp}")


def test_wait_give_up_path_with_a_tail():
    """With test_stall_copies every page wait gives up after ~20 ms: every
    tail CTA still counts in once, so the call ends with the counts at 0,
    a finite output and PA_DEV_WAIT_TIMEOUT set; a normal call on the same
    workspace afterwards is correct."""
    T = 64 * 16
    sms = 16
    lens = [T, 5, 0, 17 * 16, T - 3, 33, 16 * 16, T] * 5
    cfg = _mixed(16, lens, seed=55)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    assert _plan(cfg, sms)["tail_units"] > 0
    ws = _ws(cfg, sms)
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, ws=ws, num_sms=sms, test_stall_copies=True)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_WAIT_TIMEOUT
    assert torch.isfinite(out.float()).all()
    assert not _tail_counts(ws).any()
    good = run_gpu(wl, ws=ws, num_sms=sms)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(good, run_oracle(wl), cfg.kv_dtype, "split tail after a give-up")


def test_small_last_wave_gets_more_partitions():
    """A last wave of few units is cut into more partitions (up to 16), so
    that the tail's CTAs about fill the CTA slots; a row then merges up to 16
    partials."""
    T = 256 * 16
    lens = [T, T - 7, 3000, T, 0, 1, 17 * 16 + 3, T] * 5
    cfg = _mixed(16, lens, seed=808)
    sms = 26  # 78 slots; 160 units -> 4 in the tail
    p = _plan(cfg, sms)
    assert p["tail_units"] == 4 and p["tail_partitions"] == 16, p
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ws = _ws(cfg, sms)
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, ws=ws, num_sms=sms)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    assert not _tail_counts(ws).any()
    compare(out, run_oracle(wl), cfg.kv_dtype, "split tail, 16 partitions")
