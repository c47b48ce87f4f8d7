"""CUDA path vs the fp64 oracle, element by element (GPU)."""

import itertools

import pytest
import torch

import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, oracle_all_rows_cached, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    pa.lib()  # fails loudly when the library is missing


# Reduced versions of the five workloads: same heads, head size, block size,
# dtype and length mix; sizes the oracle finishes in seconds, still many
# pages per (sequence, kv head) and ragged last blocks.
REDUCED = {
    1: W.WORKLOADS[1],  # already tiny
    2: W.reduced(2, num_seqs=3, seq_len_hi=1000, seq_len_lo=700),
    3: W.reduced(3, num_seqs=6, seq_len_hi=2100, seq_len_lo=100),
    4: W.reduced(4, num_seqs=4, seq_len_hi=1500, seq_len_lo=900),
    5: W.reduced(5, num_seqs=3, seq_len_hi=5000, seq_len_lo=4100, shared_prefix_blocks=40),
}


@pytest.mark.parametrize("idx", sorted(REDUCED))
@pytest.mark.parametrize("partition_pages", [0, 3, 16])
def test_reduced_workloads(idx, partition_pages):
    cfg = REDUCED[idx]
    wl = W.make_workload(cfg, DEV)
    out = run_gpu(wl, partition_pages=partition_pages)
    torch.cuda.synchronize()
    ref = run_oracle(wl)
    compare(out, ref, cfg.kv_dtype, f"cfg{idx} pp={partition_pages}")
    assert pa.read_status(device=DEV) == 0


# Partition sizes that put a row's slot count (prefix partitions plus the
# sequence's own) in each regime of the combine kernel: at most 16 (one batch
# of partial rows), 17..32 (a second batch), exactly 32, and more than 32 (the
# slots read 32 at a time), on the reduced workloads and on a batch of 1040
# (sequence, kv head) units.
SLOT_REGIMES = {
    3: [(9, "<=16"), (5, "17..32"), (4, ">32")],
    5: [(64, "<=16"), (8, "17..32"), (5, "32"), (4, ">32")],
    "many units": [(3, "<=16"), (2, "17..32"), (1, ">32")],
    "many units, prefix": [(4, "<=16"), (2, "17..32"), (1, ">32")],
}
MANY_UNITS = W.PagedConfig("1040 units", num_seqs=260, num_heads=8, num_kv_heads=4, head_size=64,
                           block_size=16, num_blocks=260 * 38 + 16, seq_len_lo=300,
                           seq_len_hi=600, seed=4242)
MANY_UNITS_PREFIX = MANY_UNITS.replace(name="1040 units, prefix", shared_prefix_blocks=8,
                                       seq_len_lo=400)


@pytest.mark.parametrize("idx", list(SLOT_REGIMES), ids=str)
def test_combine_slot_count_regimes(idx):
    cfg = {"many units": MANY_UNITS, "many units, prefix": MANY_UNITS_PREFIX}.get(idx)
    cfg = cfg if cfg is not None else REDUCED[idx]
    wl = W.make_workload(cfg, DEV)
    ref = run_oracle(wl)
    for pp, regime in SLOT_REGIMES[idx]:
        plan = pa.plan(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size,
                       cfg.block_size, cfg.max_seq_len, cfg.kv_dtype,
                       shared_prefix_blocks=cfg.shared_prefix_blocks, partition_pages=pp)
        slots = plan["num_partitions"] + plan["prefix_partitions"]
        ok = {"<=16": slots <= 16, "17..32": 16 < slots < 32, "32": slots == 32,
              ">32": slots > 32}[regime]
        assert ok, (pp, regime, slots)
        assert plan["combine"] == 1
        out = torch.full_like(wl.query, float("nan"))
        run_gpu(wl, out=out, partition_pages=pp, shared_prefix_blocks=cfg.shared_prefix_blocks)
        torch.cuda.synchronize()
        compare(out, ref, cfg.kv_dtype, f"cfg{idx} pp={pp} ({slots} slots)")
        assert pa.read_status(device=DEV) == 0


@pytest.mark.parametrize("schedule", ["auto", "partitioned"])
def test_longest_first_ranking_with_ties(schedule):
    """Planned for 2 SMs, the reduced GQA batch (48 units) takes several waves
    of CTAs, so CTAs take its sequences longest first, ranked on the device;
    lengths with ties and an empty sequence."""
    cfg = REDUCED[3]
    lens = [2100, 100, 2100, 0, 1500, 100]
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    p = pa.plan(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size, cfg.block_size,
                cfg.max_seq_len, cfg.kv_dtype, num_sms=2, schedule=schedule)
    assert p["longest_first"] == 1 and p["num_partitions"] == 1
    out = torch.full_like(wl.query, float("nan"))
    run_gpu(wl, out=out, num_sms=2, schedule=schedule)
    torch.cuda.synchronize()
    compare(out, run_oracle(wl), cfg.kv_dtype, f"longest first {schedule}")


@pytest.mark.parametrize("idx", [1, 3, 4, 5])
def test_pa_decode_symbol_through_ctypes(idx):
    """The boundary call itself, pa_decode (no options), called through
    ctypes in the pages' argument order with a caller-allocated workspace;
    config 5 reduced is split by the planner, so the combine runs too."""
    import ctypes
    cfg = REDUCED[idx]
    if cfg.shared_prefix_blocks:  # same sizes, no prefix declared: a pool for it
        cfg = W.reduced(idx, num_seqs=cfg.num_seqs, seq_len_hi=cfg.seq_len_hi,
                        seq_len_lo=cfg.seq_len_lo, shared_prefix_blocks=0)
    wl = W.make_workload(cfg, DEV)
    L = pa.lib()
    code = pa.kv_dtype_code(cfg.kv_dtype)
    fp8 = code == pa.PA_KV_FP8_E4M3
    ws = torch.zeros(pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                       cfg.head_size, cfg.block_size, cfg.max_seq_len,
                                       cfg.kv_dtype), dtype=torch.uint8, device=DEV)
    out = torch.full_like(wl.query, float("nan"))
    rc = L.pa_decode(out.data_ptr(), wl.query.data_ptr(), wl.key_cache.data_ptr(),
                     wl.value_cache.data_ptr(), cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                     cfg.head_size, ctypes.c_float(cfg.scale), wl.block_tables.data_ptr(),
                     wl.block_tables.shape[1], wl.seq_lens.data_ptr(), cfg.block_size,
                     cfg.max_seq_len, cfg.num_blocks, code,
                     wl.k_scale.data_ptr() if fp8 else None, wl.v_scale.data_ptr() if fp8 else None,
                     ws.data_ptr(), ws.numel(), torch.cuda.current_stream(DEV).cuda_stream)
    assert rc == pa.PA_OK, L.pa_last_error_detail()
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, run_oracle(wl), cfg.kv_dtype, f"pa_decode symbol cfg{idx}")


SHAPES = list(itertools.product([64, 128], [16, 32], [1, 4, 8, 16], [W.BF16, W.FP8_E4M3]))


@pytest.mark.parametrize("D,B,G,kv", SHAPES, ids=lambda v: str(v))
def test_shapes(D, B, G, kv):
    Hk = 2
    lens = [1, B - 1, B, B + 1, 3 * B + 5, 17 * B - 1, 40 * B + 3]
    cfg = W.PagedConfig(f"shape D={D} B={B} G={G} {kv}", num_seqs=len(lens), num_heads=Hk * G,
                        num_kv_heads=Hk, head_size=D, block_size=B,
                        num_blocks=sum(-(-t // B) for t in lens) + 9, seq_len_lo=1,
                        seq_len_hi=max(lens), kv_dtype=kv,
                        k_scale=0.05 if kv == W.FP8_E4M3 else 1.0,
                        v_scale=0.04 if kv == W.FP8_E4M3 else 1.0, seed=4242 + D + B + G)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ref = run_oracle(wl)
    for pp in (0, 4):
        out = run_gpu(wl, partition_pages=pp)
        torch.cuda.synchronize()
        compare(out, ref, kv, f"{cfg.name} pp={pp}")


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_full_size_all_rows(idx):
    """Full workload in the launch configuration the bench times (config 5's
    shared prefix declared, as the bench does), every (sequence, query head)
    row against the oracle, which runs on chunks of whole sequences."""
    cfg = W.WORKLOADS[idx]
    wl = W.make_workload(cfg, DEV)
    ws = torch.zeros(pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                       cfg.head_size, cfg.block_size, cfg.max_seq_len,
                                       cfg.kv_dtype,
                                       shared_prefix_blocks=cfg.shared_prefix_blocks),
                     dtype=torch.uint8, device=DEV)
    out = run_gpu(wl, ws=ws, shared_prefix_blocks=cfg.shared_prefix_blocks)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    ref = oracle_all_rows_cached(wl)
    compare(out, ref, cfg.kv_dtype, f"full cfg{idx} all rows", full_size=True)
    del wl, out
    torch.cuda.empty_cache()


SMALL_LONG = {
    "1 x 32768, B=16": W.PagedConfig("1 x 32768", num_seqs=1, num_heads=32, num_kv_heads=8,
                                     head_size=128, block_size=16, num_blocks=2048 + 40,
                                     seq_len_lo=32768, seq_len_hi=32768, seed=501),
    "2 x 32768, B=16, ragged": W.PagedConfig("2 x 32768", num_seqs=2, num_heads=32,
                                             num_kv_heads=8, head_size=128, block_size=16,
                                             num_blocks=2 * 2048 + 40, seq_len_lo=20001,
                                             seq_len_hi=32768, seed=502),
    "2 x 131072, B=32, shared prefix": W.reduced(5, num_seqs=2),
    # a handful of units: about 128 CTAs, up to 128 / units partials per row
    "1 x 32768, 1 kv head": W.PagedConfig("1 x 32768, 8/1", num_seqs=1, num_heads=8,
                                          num_kv_heads=1, head_size=128, block_size=16,
                                          num_blocks=2048 + 40, seq_len_lo=32768,
                                          seq_len_hi=32768, seed=503),
    "1 x 20000, 2 kv heads, B=32": W.PagedConfig("1 x 20000, 16/2", num_seqs=1, num_heads=16,
                                                 num_kv_heads=2, head_size=128, block_size=32,
                                                 num_blocks=625 + 40, seq_len_lo=20000,
                                                 seq_len_hi=20000, seed=504),
}


@pytest.mark.parametrize("name", sorted(SMALL_LONG))
def test_small_long_context_batches_all_rows(name):
    """One or two long sequences: the planner takes one partial wave of CTAs
    with at most 32 partials per row (or, for a handful of units, about 128
    CTAs with up to 128 / units partials per row, merged in several batches of
    loads); every row against the oracle."""
    cfg = SMALL_LONG[name]
    plan = pa.plan(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size,
                   cfg.block_size, cfg.max_seq_len, cfg.kv_dtype,
                   shared_prefix_blocks=cfg.shared_prefix_blocks)
    units = cfg.num_seqs * cfg.num_kv_heads
    assert plan["num_partitions"] + plan["prefix_partitions"] <= max(32, -(-128 // units)), plan
    wl = W.make_workload(cfg, DEV)
    out = run_gpu(wl, shared_prefix_blocks=cfg.shared_prefix_blocks)
    torch.cuda.synchronize()
    assert pa.read_status(device=DEV) == 0
    compare(out, run_oracle(wl), cfg.kv_dtype, f"{name} all rows", full_size=True)


def test_full_size_cfg5_without_prefix_declaration():
    """Config 5 decoded as plain per-sequence units (the shared prefix not
    declared: every sequence streams its own copy of the prefix pages)."""
    cfg = W.WORKLOADS[5]
    wl = W.make_workload(cfg, DEV)
    out = run_gpu(wl)
    torch.cuda.synchronize()
    assert pa.read_status(device=DEV) == 0
    compare(out, oracle_all_rows_cached(wl), cfg.kv_dtype, "full cfg5 all rows, no prefix",
            full_size=True)
    del wl, out
    torch.cuda.empty_cache()


# ----------------------------------------------------------------- shared prefix
PREFIX_CASES = {
    "b32_bf16_g4": W.reduced(5, num_seqs=3, seq_len_hi=5000, seq_len_lo=4100,
                             shared_prefix_blocks=40),
    "b16_bf16_g8": W.reduced(3, num_seqs=5, seq_len_hi=3000, seq_len_lo=1000).replace(
        shared_prefix_blocks=50, num_blocks=50 + 5 * 188 + 16),
    "b16_fp8_g4": W.reduced(4, num_seqs=6, seq_len_hi=2500, seq_len_lo=800).replace(
        shared_prefix_blocks=33, num_blocks=33 + 6 * 157 + 16),
    "b16_bf16_g16": W.PagedConfig("prefix G=16", num_seqs=3, num_heads=32, num_kv_heads=2,
                                  head_size=64, block_size=16, num_blocks=20 + 3 * 40 + 8,
                                  seq_len_lo=400, seq_len_hi=640, shared_prefix_blocks=20,
                                  seed=31),
    # group sizes that do not divide 16: a sequence's rows fall in two 16-row
    # prefix groups
    "b32_bf16_g5": W.PagedConfig("prefix G=5", num_seqs=7, num_heads=10, num_kv_heads=2,
                                 head_size=128, block_size=32, num_blocks=3 + 7 * 48 + 8,
                                 seq_len_lo=100, seq_len_hi=1500, shared_prefix_blocks=3,
                                 seed=32),
    "b16_bf16_g3": W.PagedConfig("prefix G=3", num_seqs=11, num_heads=6, num_kv_heads=2,
                                 head_size=64, block_size=16, num_blocks=12 + 11 * 60 + 8,
                                 seq_len_lo=200, seq_len_hi=950, shared_prefix_blocks=12,
                                 seed=33),
    # at least as many 16-row groups per kv head as warps per CTA: the prefix
    # CTAs' warps share one page ring (4 groups on 4 warps; 5 groups, the last
    # CTA with one)
    "b16_bf16_g8_ring": W.PagedConfig("prefix G=8, shared ring", num_seqs=8, num_heads=16,
                                      num_kv_heads=2, head_size=128, block_size=16,
                                      num_blocks=37 + 8 * 70 + 8, seq_len_lo=600,
                                      seq_len_hi=1100, shared_prefix_blocks=37, seed=34),
    "b16_fp8_g8_ring": W.PagedConfig("prefix G=8 e4m3, shared ring", num_seqs=9, num_heads=16,
                                     num_kv_heads=2, head_size=128, block_size=16,
                                     num_blocks=21 + 9 * 60 + 8, seq_len_lo=400,
                                     seq_len_hi=950, shared_prefix_blocks=21,
                                     kv_dtype=W.FP8_E4M3, k_scale=0.05, v_scale=0.05, seed=35),
}


@pytest.mark.parametrize("name", sorted(PREFIX_CASES))
@pytest.mark.parametrize("partition_pages", [0, 7])
def test_shared_prefix_cascade(name, partition_pages):
    cfg = PREFIX_CASES[name]
    wl = W.make_workload(cfg, DEV)
    ws = torch.zeros(pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                       cfg.head_size, cfg.block_size, cfg.max_seq_len,
                                       cfg.kv_dtype, partition_pages,
                                       shared_prefix_blocks=cfg.shared_prefix_blocks),
                     dtype=torch.uint8, device=DEV)
    out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, cfg.num_kv_heads, cfg.scale,
              wl.block_tables, wl.seq_lens, cfg.block_size, cfg.max_seq_len, cfg.kv_dtype,
              wl.k_scale, wl.v_scale, workspace_tensor=ws, partition_pages=partition_pages,
              shared_prefix_blocks=cfg.shared_prefix_blocks)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0
    compare(out, run_oracle(wl), cfg.kv_dtype, f"prefix {name} pp={partition_pages}")


def test_shared_prefix_mismatch_is_flagged():
    cfg = PREFIX_CASES["b16_bf16_g8"]
    wl = W.make_workload(cfg, DEV)
    ws = torch.zeros(pa.workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                       cfg.head_size, cfg.block_size, cfg.max_seq_len,
                                       shared_prefix_blocks=cfg.shared_prefix_blocks),
                     dtype=torch.uint8, device=DEV)
    out = torch.empty_like(wl.query)
    bt = wl.block_tables
    bt[2, 7] = bt[2, cfg.shared_prefix_blocks]  # row 2's prefix now differs from row 0's
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, cfg.num_kv_heads, cfg.scale, bt,
              wl.seq_lens, cfg.block_size, cfg.max_seq_len, workspace_tensor=ws,
              shared_prefix_blocks=cfg.shared_prefix_blocks)
    torch.cuda.synchronize()
    assert pa.read_status(ws, clear=True) & pa.PA_DEV_PREFIX_MISMATCH
    wl.seq_lens[1] = cfg.shared_prefix_blocks * cfg.block_size - 3  # shorter than the prefix
    bt[2, 7] = bt[0, 7]
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, cfg.num_kv_heads, cfg.scale, bt,
              wl.seq_lens, cfg.block_size, cfg.max_seq_len, workspace_tensor=ws,
              shared_prefix_blocks=cfg.shared_prefix_blocks)
    torch.cuda.synchronize()
    assert pa.read_status(ws) & pa.PA_DEV_PREFIX_MISMATCH


# ----------------------------------------------------------------------- ALiBi
def alibi_slopes(n):
    """Geometric slopes 2^(-8 i / n), i = 1..n (the usual ALiBi choice)."""
    return torch.tensor([2.0 ** (-8.0 * (i + 1) / n) for i in range(n)], dtype=torch.float32)


@pytest.mark.parametrize("idx", [1, 3, 4])
@pytest.mark.parametrize("partition_pages", [0, 5])
def test_alibi(idx, partition_pages):
    cfg = REDUCED[idx]
    wl = W.make_workload(cfg, DEV)
    sl = alibi_slopes(cfg.num_heads)
    out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, cfg.num_kv_heads, cfg.scale,
              wl.block_tables, wl.seq_lens, cfg.block_size, cfg.max_seq_len, cfg.kv_dtype,
              wl.k_scale, wl.v_scale, partition_pages=partition_pages,
              alibi_slopes=sl.to(DEV))
    torch.cuda.synchronize()
    c = wl.cfg
    from parity_helpers import kv_code
    import oracle
    ref = oracle.pa_decode(wl.query.cpu(), wl.key_cache.cpu(), wl.value_cache.cpu(),
                           c.num_kv_heads, c.scale, wl.block_tables.cpu(), wl.seq_lens.cpu(),
                           c.block_size, kv_code(c), c.k_scale, c.v_scale, alibi_slopes=sl)
    compare(out, ref, cfg.kv_dtype, f"alibi cfg{idx} pp={partition_pages}")
    # the bias matters: the plain result is far from the biased one
    plain = run_gpu(wl)
    torch.cuda.synchronize()
    assert (plain.float() - out.float()).abs().max().item() > 0.05


# ---------------------------------------------------------- FP8 tensor-core compute
def _decode_fp8_compute(wl, partition_pages=0):
    c = wl.cfg
    out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, c.num_kv_heads, c.scale,
              wl.block_tables, wl.seq_lens, c.block_size, c.max_seq_len, c.kv_dtype,
              wl.k_scale, wl.v_scale, partition_pages=partition_pages, fp8_compute=True)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("D,B,G", list(itertools.product([64, 128], [16, 32], [1, 4, 8, 16])),
                         ids=lambda v: str(v))
def test_fp8_compute_shapes(D, B, G):
    Hk = 2
    lens = [1, B - 1, B, B + 1, 3 * B + 5, 17 * B - 1, 40 * B + 3]
    cfg = W.PagedConfig(f"fp8 compute D={D} B={B} G={G}", num_seqs=len(lens), num_heads=Hk * G,
                        num_kv_heads=Hk, head_size=D, block_size=B,
                        num_blocks=sum(-(-t // B) for t in lens) + 9, seq_len_lo=1,
                        seq_len_hi=max(lens), kv_dtype=W.FP8_E4M3, k_scale=0.05, v_scale=0.04,
                        seed=777 + D + B + G)
    wl = W.make_workload(cfg, DEV, seq_lens=lens)
    ref = run_oracle(wl)
    for pp in (0, 4):
        compare(_decode_fp8_compute(wl, pp), ref, W.FP8_E4M3, f"{cfg.name} pp={pp}")


def test_fp8_compute_reduced_and_full_size():
    cfg = REDUCED[4]
    wl = W.make_workload(cfg, DEV)
    compare(_decode_fp8_compute(wl), run_oracle(wl), cfg.kv_dtype, "fp8 compute reduced cfg4")
    cfg = W.WORKLOADS[4]
    wl = W.make_workload(cfg, DEV)
    out = _decode_fp8_compute(wl)
    compare(out, oracle_all_rows_cached(wl), cfg.kv_dtype, "fp8 compute full cfg4 all rows",
            full_size=True)
    del wl, out
    torch.cuda.empty_cache()


def test_fp8_compute_needs_fp8_cache():
    cfg = REDUCED[1]
    wl = W.make_workload(cfg, DEV)
    with pytest.raises(pa.PagedAttentionError):
        pa.decode(torch.empty_like(wl.query), wl.query, wl.key_cache, wl.value_cache,
                  cfg.num_kv_heads, cfg.scale, wl.block_tables, wl.seq_lens, cfg.block_size,
                  cfg.max_seq_len, fp8_compute=True)
