"""The C ABI without a GPU: the library loads, exports every declared entry
point, rejects bad arguments before any CUDA call, and plans the split."""

import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import build as pbuild
from paged_kv_cache_471_b200 import workloads as W

HEADER = os.path.join(pbuild.INCLUDE, "pagedattn.h")


@pytest.fixture(scope="module")
def L():
    pbuild.build()
    return pa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("pa_decode", "pa_decode_ex", "pa_decode_workspace_size", "pa_plan_decode",
              "pa_status_string", "pa_read_device_status", "pa_last_error_detail", "pa_version"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, flags=re.M))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(L, n)


def test_no_cuda_link_to_oracle():
    # The product library must not carry any oracle symbol.
    out = subprocess.run(["nm", "-D", pa.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in out


def test_version_and_strings(L):
    assert pa.version() >= 10000
    for code in range(5):
        assert L.pa_status_string(code).decode().startswith("PA_")
    assert b"unknown" in L.pa_status_string(77)


def _decode(L, **over):
    args = dict(out=0x10000, query=0x20000, key_cache=0x30000, value_cache=0x40000, num_seqs=2,
                num_heads=8, num_kv_heads=2, head_size=128, scale=0.088, block_tables=0x50000,
                max_blocks_per_seq=4, seq_lens=0x60000, block_size=16, max_seq_len=64,
                num_blocks=64, kv_dtype=0, k_scale=None, v_scale=None, workspace=0x70000,
                workspace_bytes=1 << 20, stream=None, opts=ctypes.byref(pa.Options(0, 148, 0, 0, None, 0, 0)))
    args.update(over)
    return L.pa_decode_ex(*args.values())


@pytest.mark.parametrize("over,code", [
    (dict(out=None), pa.PA_ERR_INVALID_ARG),
    (dict(query=0x20002), pa.PA_ERR_INVALID_ARG),
    (dict(key_cache=None), pa.PA_ERR_INVALID_ARG),
    (dict(value_cache=0x40008), pa.PA_ERR_INVALID_ARG),
    (dict(block_tables=0x50002), pa.PA_ERR_INVALID_ARG),
    (dict(seq_lens=None), pa.PA_ERR_INVALID_ARG),
    (dict(workspace=None), pa.PA_ERR_INVALID_ARG),
    (dict(num_heads=9), pa.PA_ERR_INVALID_ARG),
    (dict(num_heads=34, num_kv_heads=2), pa.PA_ERR_UNSUPPORTED),
    (dict(head_size=96), pa.PA_ERR_UNSUPPORTED),
    (dict(block_size=8), pa.PA_ERR_UNSUPPORTED),
    (dict(kv_dtype=5), pa.PA_ERR_UNSUPPORTED),
    (dict(max_seq_len=65), pa.PA_ERR_INVALID_ARG),
    (dict(max_seq_len=-1), pa.PA_ERR_INVALID_ARG),
    (dict(num_blocks=0), pa.PA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), pa.PA_ERR_INVALID_ARG),
    (dict(kv_dtype=1), pa.PA_ERR_INVALID_ARG),  # fp8 without scales
    (dict(workspace_bytes=16), pa.PA_ERR_WORKSPACE_TOO_SMALL),
    (dict(num_seqs=-1), pa.PA_ERR_INVALID_ARG),
    (dict(max_blocks_per_seq=0), pa.PA_ERR_INVALID_ARG),
])
def test_rejects_before_launch(L, over, code):
    assert _decode(L, **over) == code
    assert L.pa_last_error_detail().decode() != ""


def test_zero_sequences_is_a_no_op(L):
    assert _decode(L, num_seqs=0, out=None, query=None) == pa.PA_OK


def test_workspace_size_header_only_without_split():
    n = pa.workspace_size(64, 32, 32, 128, 16, 4096, "bf16", num_sms=148,
                          schedule="partitioned")
    assert n == pa.WORKSPACE_HEADER_BYTES


def test_split_tail_plan_and_workspace():
    """Whole units in two or three waves (or more, for paired pages): the
    last wave's units (units mod CTA slots) are cut into 4 partitions whose
    CTAs follow the whole units; the workspace holds, after the header and the
    split-tail counts, their partials ((D + 2) floats per row and partition),
    256-byte aligned."""
    S, Hq, Hk, D, B, T = 32, 32, 32, 128, 16, 8192
    p = pa.plan(S, Hq, Hk, D, B, T, "bf16", num_sms=148)
    units, slots = S * Hk, 3 * 148
    tail = units % slots
    assert (p["num_partitions"], p["tail_units"], p["tail_partitions"]) == (1, tail, 4)
    assert p["tail_partition_pages"] == -(-(T // B) // 4)
    assert p["grid_ctas"] == units - tail + 4 * tail
    body0 = pa.WORKSPACE_HEADER_BYTES + pa.WORKSPACE_MERGE_COUNT_BYTES
    body = tail * (Hq // Hk) * 4 * (D + 2) * 4
    assert p["workspace_bytes"] == body0 + -(-body // 256) * 256
    assert pa.workspace_size(S, Hq, Hk, D, B, T, "bf16", num_sms=148) == p["workspace_bytes"]
    # GQA: G rows per tail unit
    q = pa.plan(128, 32, 8, 128, 16, 16384, "fp8_e4m3", num_sms=148)
    tail = (128 * 8) % slots
    assert (q["tail_units"], q["tail_partitions"], q["tail_partition_pages"]) == (tail, 4, 256)
    body = tail * 4 * 4 * (128 + 2) * 4
    assert q["workspace_bytes"] == body0 + -(-body // 256) * 256


def test_split_tail_only_where_it_applies():
    base = dict(num_sms=148)
    # 1024 units (2.3 waves of 444 CTA slots) get one
    assert pa.plan(32, 32, 32, 128, 16, 4096, "bf16", **base)["tail_units"] == 1024 % 444
    # the partitioned schedule, forced partitions, a shared prefix, fewer than
    # two or four and more waves of units, or units filling whole waves: none
    assert pa.plan(32, 32, 32, 128, 16, 4096, "bf16", schedule="partitioned",
                   **base)["tail_units"] == 0
    assert pa.plan(32, 32, 32, 128, 16, 4096, "bf16", partition_pages=64,
                   **base)["tail_units"] == 0
    assert pa.plan(32, 32, 32, 128, 16, 4096, "bf16", shared_prefix_blocks=16,
                   **base)["tail_units"] == 0
    assert pa.plan(16, 32, 32, 128, 16, 4096, "bf16", **base)["tail_units"] == 0
    assert pa.plan(64, 32, 32, 128, 16, 4096, "bf16", **base)["tail_units"] == 0  # 4.6 waves
    # ... but pages that go in pairs are split from four waves up too
    assert pa.plan(64, 32, 32, 64, 16, 4096, "bf16", **base)["tail_units"] == 2048 % 444
    assert pa.plan(256, 32, 8, 128, 16, 16384, "fp8_e4m3", **base)["tail_units"] == 2048 % 444
    assert pa.plan(256, 32, 8, 128, 32, 16384, "fp8_e4m3", **base)["tail_units"] == 0
    assert pa.plan(111, 12, 3, 128, 16, 4096, "bf16", num_sms=37)["tail_units"] == 0  # 3 x 111
    # a small last wave gets more partitions (enough to about fill the slots,
    # at most 16, none under 16 pages)
    p = pa.plan(224, 32, 8, 128, 16, 16384, "fp8_e4m3", **base)
    assert (p["tail_units"], p["tail_partitions"], p["tail_partition_pages"]) == (16, 16, 64)
    p = pa.plan(224, 32, 8, 128, 16, 2048, "fp8_e4m3", **base)  # 128 pages: at most 8
    assert (p["tail_units"], p["tail_partitions"], p["tail_partition_pages"]) == (16, 8, 16)
    # tail partitions of fewer than 16 pages are not made
    assert pa.plan(32, 32, 32, 128, 16, 960, "bf16", **base)["tail_units"] == 0
    assert pa.plan(32, 32, 32, 128, 16, 1024, "bf16", **base)["tail_units"] > 0


def test_longest_first_only_for_more_than_one_wave():
    # ranked when the grid takes more than one wave of 444 CTA slots
    p1, p2, p3, p5 = (_plan(i) for i in (1, 2, 3, 5))
    assert p1["grid_ctas"] <= 444 and p1["longest_first"] == 0
    assert p2["longest_first"] == 1 and p3["longest_first"] == 1 and p5["longest_first"] == 1
    # one sequence, more than 256 sequences, or the balanced schedule: never
    assert pa.plan(1, 32, 8, 128, 16, 131072, "bf16", num_sms=148)["longest_first"] == 0
    assert pa.plan(300, 32, 8, 128, 16, 4096, "bf16", num_sms=148)["longest_first"] == 0
    assert pa.plan(64, 32, 8, 128, 16, 4096, "bf16", num_sms=148,
                   schedule="balanced")["longest_first"] == 0


def test_where_the_split_partials_are_merged():
    """By the combine kernel for split partitions, a shared prefix and the
    balanced and dynamic schedules; a split tail's inside the decode kernel
    (no combine launch); whole units need no merge."""
    base = dict(num_sms=148)
    assert pa.plan(8, 32, 8, 128, 32, 131072, "bf16", shared_prefix_blocks=1024,
                   **base)["combine"] == 1
    assert pa.plan(64, 32, 16, 128, 16, 4096, "bf16", partition_pages=64,
                   **base)["combine"] == 1
    assert pa.plan(32, 32, 32, 128, 16, 8192, "bf16", **base)["combine"] == 0  # split tail
    assert pa.plan(64, 32, 32, 128, 16, 4096, "bf16", **base)["combine"] == 0  # whole units
    assert pa.plan(64, 32, 8, 128, 16, 4096, "bf16", schedule="balanced",
                   **base)["combine"] == 1
    assert pa.plan(64, 32, 8, 128, 16, 4096, "bf16", schedule="dynamic",
                   **base)["combine"] == 1


def test_balanced_workspace_layout():
    # header, the per-sequence page scan (S + 2 ints, 256-byte aligned), then
    # two slots of G rows of (D + 2) floats per CTA slot.
    p = pa.plan(64, 32, 8, 128, 16, 4096, "bf16", num_sms=148, schedule="balanced")
    assert p["balanced"] == 1 and p["num_partitions"] == 0 and p["grid_ctas"] == 3 * 148
    scan = -(-(64 + 2) * 4 // 256) * 256
    rows = 2 * p["grid_ctas"] * 4
    expect = -(-(256 + 4096 + scan + rows * 130 * 4) // 256) * 256
    assert p["workspace_bytes"] == expect


def _plan(idx, **kw):
    c = W.WORKLOADS[idx]
    return pa.plan(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                   c.max_seq_len, c.kv_dtype, num_sms=148, **kw)


def test_planner_on_the_five_workloads():
    p1, p2, p3, p4, p5 = (_plan(i) for i in range(1, 6))
    assert all(p["balanced"] == 0 for p in (p1, p2, p3, p4, p5))
    assert p1["num_partitions"] == 1 and p1["partition_pages"] == 16
    # whole units; in two or three waves (or more, for paired pages) the last
    # wave's units in 4 partitions
    assert p2["num_partitions"] == 1 and p2["grid_ctas"] == 64 * 32 and p2["tail_units"] == 0
    assert p3["num_partitions"] == 1  # two waves of units; longest-first order
    assert p3["tail_units"] == 128 * 8 % 444
    assert p4["num_partitions"] == 1 and p4["tail_units"] == 256 * 8 % 444  # paired e4m3
    assert p4["grid_ctas"] == 256 * 8 + 3 * p4["tail_units"]
    assert p1["tail_units"] == 0 and p5["tail_units"] == 0
    assert p5["num_partitions"] >= 4  # 64 (seq, kv head) units cannot fill 148 SMs
    # balanced ranges on request: one wave of CTAs
    q2, q3, q4 = (_plan(i, schedule="balanced") for i in (2, 3, 4))
    for q in (q2, q3, q4):
        assert q["balanced"] == 1 and q["grid_ctas"] == 3 * 148 and q["num_partitions"] == 0
    for p in (p1, p2, p3, p4, p5, q2, q3, q4):
        assert p["smem_bytes"] <= 227 * 1024 and 2 <= p["stages"] <= 8
        P, PP = p["num_partitions"], p["partition_pages"]
    c5 = W.WORKLOADS[5]
    assert p5["num_partitions"] * p5["partition_pages"] >= c5.max_blocks_per_seq
    ws = pa.workspace_size(c5.num_seqs, c5.num_heads, c5.num_kv_heads, 128, 32, c5.max_seq_len,
                           num_sms=148)
    assert ws >= 256 + 4096 + 8 * 32 * p5["num_partitions"] * 130 * 4


def test_planner_splits_between_one_and_two_waves():
    # 64 sequences x 8 kv heads = 512 units for 148 x 3 CTA slots: unsplit, a
    # last wave of 68 full-length units would run alone.
    p = pa.plan(64, 32, 8, 128, 16, 16384, "bf16", num_sms=148)
    assert p["num_partitions"] >= 2
    # 1024 units (more than two waves) are not split, apart from the split
    # tail under the auto schedule, which the partitioned schedule leaves out.
    p = pa.plan(128, 32, 8, 128, 16, 16384, "bf16", num_sms=148)
    assert p["num_partitions"] == 1 and p["tail_units"] == 1024 % 444
    q = pa.plan(128, 32, 8, 128, 16, 16384, "bf16", num_sms=148, schedule="partitioned")
    assert q["num_partitions"] == 1 and q["tail_units"] == 0
    assert q["grid_ctas"] == 1024 and p["grid_ctas"] == 1024 + 3 * p["tail_units"]


def test_split_count_fills_the_last_wave():
    """Split plans take a partition count whose last wave of CTAs is about
    62% full (55-70% measured best), among half to twice the count long
    partitions would give."""
    slots = 3 * 148
    for args, kw in [((8, 32, 8, 128, 32, 131072), dict(shared_prefix_blocks=1024)),
                     ((8, 32, 8, 128, 32, 131072), {}),
                     ((8, 32, 8, 128, 16, 131072), {}),
                     ((16, 32, 8, 128, 16, 16384), {})]:
        p = pa.plan(*args, "bf16", num_sms=148, **kw)
        w = p["grid_ctas"] / slots
        assert p["num_partitions"] > 1 and w >= 1.4, (args, p)
        assert 0.5 <= w - int(w) <= 0.75, (args, p, w)


def test_split_plans_keep_to_one_combine_load_batch():
    """At most 32 partials per query row (one batch of loads in the combine)
    where a grid of 1.4 waves or more allows it; batches too small for that
    take one partial wave, at least half the CTA slots and nearest 75% full;
    a handful of units (too few for half a wave within the limit) takes about
    128 CTAs, with up to max(32, 128 / units) partials per row."""
    slots = 3 * 148

    def per_row(p):
        return p["num_partitions"] + p["prefix_partitions"]

    # multi-wave grids within the limit (4 and 6 x 131072 tokens, 8 kv heads)
    for S in (4, 6):
        p = pa.plan(S, 32, 8, 128, 16, 131072, "bf16", num_sms=148)
        assert per_row(p) <= 32 and p["grid_ctas"] / slots >= 1.4, (S, p)
    # one or two long sequences of 8 kv heads: one partial wave
    for S, T, B, pre in ((1, 32768, 16, 0), (2, 32768, 16, 0), (1, 16384, 16, 0),
                         (1, 131072, 32, 1024), (2, 131072, 32, 1024)):
        p = pa.plan(S, 32, 8, 128, B, T, "bf16", num_sms=148, shared_prefix_blocks=pre)
        w = p["grid_ctas"] / slots
        assert per_row(p) <= 32 and 0.5 <= w < 1.0, (S, T, p, w)
    # 1, 2 and 4 units of one long sequence: 128 CTAs
    for Hk, rows in ((1, 128), (2, 64), (4, 32)):
        p = pa.plan(1, 8 * Hk, Hk, 128, 16, 131072, "bf16", num_sms=148)
        assert per_row(p) == rows and p["grid_ctas"] == 128, (Hk, p)


def test_split_plans_cover_every_page_over_many_shapes():
    """Invariants of every split plan the planner picks, over a grid of batch
    shapes: the partitions cover each sequence's own pages (after a shared
    prefix) and the prefix, none of them is empty at max_seq_len, the sizes are
    even (less than a page of slack per partition), the grid is the per-sequence CTAs plus the prefix CTAs, and the
    partials per row stay within max(32, 128 / units)."""
    n_split = 0
    for S in (1, 2, 3, 5, 8, 13):
        for Hk, G in ((1, 8), (2, 4), (4, 8), (8, 4), (32, 1)):
            for B, T in ((16, 2048), (16, 32768), (32, 131072), (16, 100000)):
                for pre_frac in (0, 4):
                    pages = -(-T // B)
                    prefix = pages // pre_frac if pre_frac else 0
                    p = pa.plan(S, Hk * G, Hk, 128, B, T, "bf16", num_sms=148,
                                shared_prefix_blocks=prefix)
                    P, pp, ppre = p["num_partitions"], p["partition_pages"], p["prefix_partitions"]
                    own = pages - prefix
                    units = S * Hk
                    if P <= 1 and not prefix:
                        continue  # whole units (or the split tail, checked elsewhere)
                    n_split += 1
                    what = (S, Hk, G, B, T, prefix, p)
                    assert P >= 1 and pp >= 1, what
                    assert P * pp >= own and (P - 1) * pp < own, what  # covers, none empty
                    assert P * pp - own < P, what  # even: under a page of slack per partition
                    assert ppre * pp >= prefix and (ppre == 0 or (ppre - 1) * pp < prefix), what
                    groups = -(-S * G // 16)
                    W = p["warps_per_cta"]
                    cta_groups = -(-groups // W) if groups >= W else groups
                    assert p["grid_ctas"] == units * P + Hk * cta_groups * ppre, what
                    assert P + ppre <= max(32, -(-128 // units)), what
    assert n_split > 100


def test_balanced_schedule_limits():
    # forced partitions or a shared prefix rule balanced ranges out
    with pytest.raises(pa.PagedAttentionError):
        pa.plan(64, 32, 8, 128, 16, 4096, "bf16", num_sms=148, schedule="balanced",
                partition_pages=8)
    with pytest.raises(pa.PagedAttentionError):
        pa.plan(64, 32, 8, 128, 16, 4096, "bf16", num_sms=148, schedule="balanced",
                shared_prefix_blocks=4)
    # a tiny batch may ask for them
    p = pa.plan(2, 8, 2, 64, 16, 40, "bf16", num_sms=148, schedule="balanced")
    assert p["balanced"] == 1 and p["grid_ctas"] == 3 * 148
    # e4m3 MMAs: two CTAs per SM
    p = pa.plan(256, 32, 8, 128, 16, 16384, "fp8_e4m3", num_sms=148, fp8_compute=True,
                schedule="balanced")
    assert p["balanced"] == 1 and p["grid_ctas"] == 2 * 148
    with pytest.raises(ValueError):
        pa.plan(4, 8, 2, 64, 16, 40, "bf16", num_sms=148, schedule="sometimes")


def test_paired_small_pages_fill_the_stage_memory():
    # 16-token e4m3 pages, and bf16 pages of head size 64, go two per stage:
    # the same 64 KiB of stages per CTA (4 warps x 2 stages x 8 KiB) as bf16
    # pages of head size 128, with 3 CTAs per SM.
    for kv, D in (("fp8_e4m3", 128), ("bf16", 64), ("bf16", 128)):
        p = pa.plan(256, 32, 8, D, 16, 16384, kv, num_sms=148)
        assert p["warps_per_cta"] == 4 and p["stages"] == 2, (kv, D, p)
        assert p["smem_bytes"] == 4 * 2 * 8192 + 4 * 2 * 8, (kv, D, p)
    # e4m3 with FP8 MMAs pairs too; 2 CTAs per SM for its larger register use
    p = pa.plan(256, 32, 8, 128, 16, 16384, "fp8_e4m3", num_sms=148, fp8_compute=True,
                schedule="balanced")
    assert p["smem_bytes"] == 4 * 2 * 8192 + 4 * 2 * 8 and p["grid_ctas"] == 2 * 148
    # pages of 4 KiB or more are not paired
    p = pa.plan(256, 32, 8, 128, 32, 16384, "fp8_e4m3", num_sms=148)
    assert p["smem_bytes"] == 4 * 2 * 8192 + 4 * 2 * 8
    p = pa.plan(256, 32, 8, 64, 16, 16384, "fp8_e4m3", num_sms=148)
    assert p["smem_bytes"] == 4 * 2 * 4096 + 4 * 2 * 8


def test_forced_partitions():
    p = _plan(2, partition_pages=7)
    assert p["partition_pages"] == 7 and p["num_partitions"] == -(-256 // 7)
    p = _plan(2, partition_pages=10000)
    assert p["num_partitions"] == 1


def test_two_ctas_per_sm_fit_for_the_bf16_b16_pages():
    p = _plan(2)
    assert 2 * (p["smem_bytes"] + 1024) <= 228 * 1024


def test_every_plan_fits_shared_memory():
    # Every supported shape and forced split stays inside the 227 KiB opt-in
    # limit of one CTA (a plan above it would fail to launch).
    for D in (64, 128):
        for B in (16, 32):
            for kv in ("bf16", "fp8_e4m3"):
                for G in (1, 4, 8, 16):
                    for T in (1, 15, 17, 100, 1000, 20000, 131072):
                        for pp in (0, 1, 2, 3, 5, 16, 64):
                            p = pa.plan(4, 2 * G, 2, D, B, T, kv, partition_pages=pp, num_sms=148)
                            assert p["smem_bytes"] <= 227 * 1024 - 256, (D, B, kv, G, T, pp)
                        p = pa.plan(4, 2 * G, 2, D, B, T, kv, num_sms=148, schedule="balanced")
                        assert p["smem_bytes"] <= 227 * 1024 - 256, (D, B, kv, G, T)


def test_alibi_with_shared_prefix_is_refused(L):
    slopes = ctypes.c_void_p(0x80000)
    rc = _decode(L, opts=ctypes.byref(pa.Options(0, 148, 0, 2, slopes)))
    assert rc == pa.PA_ERR_UNSUPPORTED
    rc = _decode(L, opts=ctypes.byref(pa.Options(0, 148, 0, 0, ctypes.c_void_p(0x80002))))
    assert rc == pa.PA_ERR_INVALID_ARG  # misaligned slopes


def _noalloc(L, **over):
    args = dict(out=0x10000, query=0x20000, key_cache=0x30000, value_cache=0x40000,
                num_seqs=64, num_heads=128, num_kv_heads=8, head_size=128, scale=0.088,
                block_tables=0x50000, max_blocks_per_seq=32768, seq_lens=0x60000,
                block_size=16, max_seq_len=524288, num_blocks=1 << 20, kv_dtype=0,
                k_scale=None, v_scale=None, stream=None)
    args.update(over)
    return L.pa_decode_noalloc(*args.values())


@pytest.mark.parametrize("over", [dict(out=None), dict(query=0x20002), dict(seq_lens=None),
                                  dict(scale=float("inf")), dict(num_blocks=0),
                                  dict(kv_dtype=1), dict(max_seq_len=524289)])
def test_noalloc_reports_argument_errors_before_the_scratch_size(L, over):
    # A problem far beyond the built-in scratch, with one bad argument: the
    # argument is what is reported (the checks run before planning, so no
    # CUDA call is needed to get there).
    assert _noalloc(L, **over) == pa.PA_ERR_INVALID_ARG
    assert L.pa_last_error_detail().decode() != ""


def test_noalloc_zero_sequences_is_a_no_op(L):
    assert _noalloc(L, num_seqs=0, out=None, query=None) == pa.PA_OK


def test_dynamic_schedule_plan_and_workspace():
    # One wave of CTAs; slots per row and unit kind from warps per unit; the
    # workspace holds the header, 16 bytes of counters per unit (256-aligned),
    # then the partials of every query row's slots.
    for idx in (2, 3, 4, 5):
        c = W.WORKLOADS[idx]
        pref = c.shared_prefix_blocks
        p = pa.plan(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                    c.max_seq_len, c.kv_dtype, num_sms=148, schedule="dynamic",
                    shared_prefix_blocks=pref)
        assert p["balanced"] == 0 and p["partition_pages"] == 0
        assert p["grid_ctas"] == 148 * 3
        warps = p["grid_ctas"] * p["warps_per_cta"]
        groups = -(-(c.num_seqs * c.group) // 16) if pref else 0
        units = c.num_kv_heads * groups + c.num_seqs * c.num_kv_heads
        owners = 4 if 2 * units >= warps else 1
        assert p["dynamic"] == owners
        k = min(64, owners + -(-2 * warps // units) + 8)
        assert p["num_partitions"] == k and p["prefix_partitions"] == (k if pref else 0)
        assert p["prefix_groups"] == groups
        k_total = k * (2 if pref else 1)
        expect = 256 + 4096 + -(-units * 16 // 256) * 256 + c.num_seqs * c.num_heads * k_total * \
            (c.head_size + 2) * 4
        assert p["workspace_bytes"] == -(-expect // 256) * 256
        assert p["smem_bytes"] == p["warps_per_cta"] * p["stages"] * (
            2 * c.head_size * c.block_size * c.elem_bytes *
            (2 if (c.block_size == 16 and (c.kv_dtype == "fp8_e4m3" or c.head_size == 64)) else 1)
            + 24)
    with pytest.raises(pa.PagedAttentionError):  # no forced partitions
        pa.plan(64, 32, 8, 128, 16, 4096, "bf16", num_sms=148, schedule="dynamic",
                partition_pages=8)
