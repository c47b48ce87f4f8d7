"""CUDA path vs the fp64 oracle on value ranges and sizes at the edges of
what the kernels handle (GPU): near-argmax softmax, queries beyond the f16
range (the FP8 path's power-of-two prescale), saturated and subnormal e4m3
codes, and one sequence of half a million tokens split into many partitions."""

import pytest
import torch

import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, run_oracle, run_oracle_all

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LENS = [1, 15, 16, 17, 100, 777, 2049]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    pa.lib()


def _workload(kv, seed, k_scale=0.05, v_scale=0.04, D=128, B=16, G=4, Hk=2, lens=LENS):
    fp8 = kv == W.FP8_E4M3
    cfg = W.PagedConfig(f"extremes {kv} seed={seed}", num_seqs=len(lens), num_heads=Hk * G,
                        num_kv_heads=Hk, head_size=D, block_size=B,
                        num_blocks=sum(-(-t // B) for t in lens) + 5, seq_len_lo=1,
                        seq_len_hi=max(lens), kv_dtype=kv, k_scale=k_scale if fp8 else 1.0,
                        v_scale=v_scale if fp8 else 1.0, seed=seed)
    return W.make_workload(cfg, DEV, seq_lens=lens)


def _decode(wl, fp8_compute=False, partition_pages=0):
    c = wl.cfg
    out = torch.empty_like(wl.query)
    pa.decode(out, wl.query, wl.key_cache, wl.value_cache, c.num_kv_heads, c.scale,
              wl.block_tables, wl.seq_lens, c.block_size, c.max_seq_len, c.kv_dtype,
              wl.k_scale, wl.v_scale, partition_pages=partition_pages,
              **({"fp8_compute": True} if fp8_compute else {}))
    torch.cuda.synchronize()
    return out


PATHS = [(W.BF16, False), (W.FP8_E4M3, False), (W.FP8_E4M3, True)]
PATH_IDS = ["bf16", "fp8", "fp8_compute"]


@pytest.mark.parametrize("kv,f8c", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("pp", [0, 5])
def test_sharp_softmax(kv, f8c, pp):
    """Query scaled by 16: logits spread over hundreds of units, so a handful
    of tokens hold nearly all the weight and the running maximum moves often
    across pages and partitions."""
    wl = _workload(kv, seed=501)
    wl.query.mul_(16)
    ref = run_oracle(wl)
    compare(_decode(wl, f8c, pp), ref, kv, f"sharp softmax {kv} f8c={f8c} pp={pp}")
    assert pa.read_status(device=DEV) == 0


@pytest.mark.parametrize("pp", [0, 5])
def test_query_beyond_f16_range(pp):
    """FP8 cache, f16 MMAs: head-dim component 0 of every query row is about
    +-1e5, past the f16 limit, so the kernel's power-of-two prescale of q is
    taken (without it that component would become inf).  Component 0 of every
    key is set to code 0, so the spike adds nothing to the logits and the
    result tests that the prescale is undone exactly in the logit multiplier."""
    wl = _workload(W.FP8_E4M3, seed=502)
    g = torch.Generator(device="cpu").manual_seed(502)
    sign = torch.randint(0, 2, wl.query.shape[:2], generator=g).float() * 2 - 1
    wl.query[:, :, 0] = (1e5 * sign).to(wl.query.dtype).to(DEV)
    assert wl.query.float().abs().max().item() > 65504
    wl.key_cache.view(torch.uint8)[:, :, 0, :, 0] = 0  # d = 0 is chunk 0, lane 0
    ref = run_oracle(wl)
    compare(_decode(wl, False, pp), ref, W.FP8_E4M3, f"|q| > f16 max pp={pp}")


@pytest.mark.parametrize("f8c", [False, True], ids=["fp8", "fp8_compute"])
@pytest.mark.parametrize("scales,what", [((0.002, 0.002), "saturated"), ((64.0, 64.0), "subnormal")],
                         ids=["saturated", "subnormal"])
def test_e4m3_code_ranges(f8c, scales, what):
    """Scales that push about a third of the codes to +-448 (saturated), or
    about two thirds of them into the e4m3 subnormal range (exponent field 0)."""
    wl = _workload(W.FP8_E4M3, seed=503, k_scale=scales[0], v_scale=scales[1])
    codes = wl.key_cache.view(torch.uint8)[wl.key_cache.view(torch.uint8) != W.E4M3_NAN_CODE]
    mag = codes & 0x7F
    if what == "saturated":
        assert (mag == 0x7E).float().mean().item() > 0.2  # 0x7E = 448
    else:
        assert (mag < 0x08).float().mean().item() > 0.5  # exponent field 0
    ref = run_oracle(wl)
    compare(_decode(wl, f8c), ref, W.FP8_E4M3, f"{what} codes f8c={f8c}")


def test_half_million_token_sequence():
    """One sequence of 2^19 tokens beside a short one (8 kv heads, block size
    32, bf16): the planner splits the long sequence into many partitions (up
    to the 32 the combine merges in one batch of loads), and a forced partition
    size splits it into 64; the combine merges them.  Every row against the
    oracle, both ways."""
    lens = [1 << 19, 1000]
    wl = _workload(W.BF16, seed=504, D=128, B=32, G=4, Hk=8, lens=lens)
    c = wl.cfg
    p = pa.plan(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_size, c.block_size,
                c.max_seq_len, c.kv_dtype)
    assert 16 <= p["num_partitions"] <= 32, p
    ref = run_oracle_all(wl)
    for pp, what in ((0, "planned"), (256, "64 partitions")):
        out = _decode(wl, partition_pages=pp)
        assert torch.isfinite(out.float()).all()
        compare(out, ref, W.BF16, f"2^19-token sequence all rows, {what}", full_size=True)
        assert pa.read_status(device=DEV) == 0
    del wl, out
    torch.cuda.empty_cache()
