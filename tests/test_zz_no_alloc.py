"""The allocation-free entry point, pa_decode_noalloc (GPU).

Some callers cannot allocate device memory at the moment they decode (code
running inside an allocator callback, a runtime whose memory pool is owned by
someone else, a plugin whose host forbids allocations after start-up).  For
them the library keeps its split-KV scratch in one fixed device array.  These
checks call that entry point through the C ABI and compare it with pa_decode
given a caller-allocated workspace, on two calls in a row whose plans both
use the scratch, and check that a problem needing more scratch than the
array holds is refused before any launch.

The file is named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import TOL, run_gpu, run_oracle, compare

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _noalloc(L, wl, out):
    c = wl.cfg
    code = pa.kv_dtype_code(c.kv_dtype)
    fp8 = code == pa.PA_KV_FP8_E4M3
    return L.pa_decode_noalloc(
        out.data_ptr(), wl.query.data_ptr(), wl.key_cache.data_ptr(), wl.value_cache.data_ptr(),
        c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, ctypes.c_float(c.scale),
        wl.block_tables.data_ptr(), wl.block_tables.shape[1], wl.seq_lens.data_ptr(),
        c.block_size, c.max_seq_len, c.num_blocks, code,
        wl.k_scale.data_ptr() if fp8 else None, wl.v_scale.data_ptr() if fp8 else None,
        torch.cuda.current_stream(DEV).cuda_stream)


def _uses_scratch(c):
    p = pa.plan(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                c.max_seq_len, c.kv_dtype)
    return p["num_partitions"] > 1 and p["workspace_bytes"] <= pa.NOALLOC_SCRATCH_BYTES


def test_noalloc_matches_workspace_entry_point_twice():
    L = pa.lib()
    cases = [W.reduced(5, num_seqs=3, seq_len_hi=5000, seq_len_lo=4100, shared_prefix_blocks=40),
             W.reduced(4, num_seqs=2, seq_len_hi=6000, seq_len_lo=3000)]
    for cfg in cases:
        assert _uses_scratch(cfg), cfg.name
    tol = {W.BF16: TOL[W.BF16]["max_abs"], W.FP8_E4M3: TOL[W.FP8_E4M3]["max_abs"]}
    for cfg in cases:  # two calls in a row, each with a different split
        wl = W.make_workload(cfg, DEV)
        ref = run_gpu(wl)  # pa_decode with a caller-allocated workspace
        out = torch.full_like(wl.query, float("nan"))
        assert _noalloc(L, wl, out) == pa.PA_OK, L.pa_last_error_detail()
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        diff = (out.float() - ref.float()).abs().max().item()
        assert diff <= tol[cfg.kv_dtype], (cfg.name, diff)
        compare(out, run_oracle(wl), cfg.kv_dtype, "noalloc vs oracle")


def test_noalloc_rejects_problems_beyond_its_scratch():
    L = pa.lib()
    cfg = W.reduced(3, num_seqs=4, seq_len_hi=600, seq_len_lo=500)
    wl = W.make_workload(cfg, DEV)
    # A size whose plan needs more scratch than the array holds, on this GPU.
    big = None
    for S, Hk, T in [(55, 8, 262144), (54, 8, 262144), (53, 8, 262144), (44, 8, 262144),
                     (43, 8, 262144), (64, 8, 65536), (16, 8, 131072), (5, 2, 524288)]:
        need = pa.workspace_size(S, 16 * Hk, Hk, 128, 16, T, "bf16")
        if need > pa.NOALLOC_SCRATCH_BYTES:
            big = (S, Hk, T)
            break
    assert big is not None, "no candidate size exceeds the built-in scratch on this GPU"
    S, Hk, T = big
    # The scratch size is checked on the host before any launch or device
    # access, so the small buffers passed below are never touched.
    out = torch.empty_like(wl.query)
    rc = L.pa_decode_noalloc(
        out.data_ptr(), wl.query.data_ptr(), wl.key_cache.data_ptr(), wl.value_cache.data_ptr(),
        S, 16 * Hk, Hk, 128, ctypes.c_float(cfg.scale), wl.block_tables.data_ptr(), T // 16,
        wl.seq_lens.data_ptr(), 16, T, cfg.num_blocks, 0, None, None,
        torch.cuda.current_stream(DEV).cuda_stream)
    assert rc == pa.PA_ERR_WORKSPACE_TOO_SMALL
    assert b"built-in scratch" in L.pa_last_error_detail()


def test_noalloc_same_shape_long_then_short():
    """One shape called twice: first with long sequences (every partition of
    every row written), then with short ones -- empty, under one partition,
    just over one -- so the scratch still holds the first call's partials in
    slots the second call does not write.  The second output must match the
    oracle: a call reads only partials it wrote itself."""
    L = pa.lib()
    cfg = W.reduced(4, num_seqs=4, seq_len_hi=6000, seq_len_lo=5000)
    p = pa.plan(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_size, cfg.block_size,
                cfg.max_seq_len, cfg.kv_dtype)
    assert p["num_partitions"] > 2 and p["workspace_bytes"] <= pa.NOALLOC_SCRATCH_BYTES
    span = p["partition_pages"] * cfg.block_size  # tokens per partition
    long_wl = W.make_workload(cfg, DEV, seq_lens=[6000, 5999, 5500, 6000])
    short_wl = W.make_workload(cfg, DEV, seq_lens=[0, 7, span - 1, span + 5])
    for wl in (long_wl, short_wl):
        out = torch.full_like(wl.query, float("nan"))
        assert _noalloc(L, wl, out) == pa.PA_OK, L.pa_last_error_detail()
        torch.cuda.synchronize()
        compare(out, run_oracle(wl), cfg.kv_dtype, f"noalloc {wl.seq_lens.tolist()}")
