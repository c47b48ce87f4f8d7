"""Block copies on the GPU (pa_copy_blocks) and decode over block tables the
block manager built, with copy on write (GPU)."""

import numpy as np
import pytest
import torch

import paged_kv_cache_471_b200 as pa
from paged_kv_cache_471_b200 import workloads as W
from parity_helpers import compare, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("kv,D,B,Hk", [(W.BF16, 128, 16, 8), (W.FP8_E4M3, 128, 16, 4),
                                       (W.BF16, 64, 32, 2), (W.BF16, 128, 32, 32)])
def test_copy_blocks_bit_exact(kv, D, B, Hk):
    cfg = W.PagedConfig("copy", num_seqs=1, num_heads=Hk, num_kv_heads=Hk, head_size=D,
                        block_size=B, num_blocks=300, seq_len_lo=1, seq_len_hi=B, kv_dtype=kv)
    g = torch.Generator(device=DEV).manual_seed(3)
    if kv == W.BF16:
        kc = torch.randn(cfg.key_cache_shape(), generator=g, device=DEV).to(torch.bfloat16)
        vc = torch.randn(cfg.value_cache_shape(), generator=g, device=DEV).to(torch.bfloat16)
    else:
        kc = torch.randint(0, 255, cfg.key_cache_shape(), generator=g, device=DEV, dtype=torch.uint8)
        vc = torch.randint(0, 255, cfg.value_cache_shape(), generator=g, device=DEV, dtype=torch.uint8)
    perm = torch.randperm(300, generator=torch.Generator().manual_seed(4))
    src, dst = perm[:100].to(DEV), perm[100:200].to(DEV)
    want_k, want_v = kc.clone(), vc.clone()
    want_k[dst] = kc[src]
    want_v[dst] = vc[src]
    pa.copy_blocks(kc, vc, src, dst, kv)
    torch.cuda.synchronize()
    assert torch.equal(kc.view(torch.uint8), want_k.view(torch.uint8))
    assert torch.equal(vc.view(torch.uint8), want_v.view(torch.uint8))


def test_copy_blocks_skips_bad_ids():
    kc = torch.zeros((10, 2, 8, 16, 8), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros((10, 2, 64, 16), dtype=torch.bfloat16, device=DEV)
    kc[3] = 1
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pa.copy_blocks(kc, vc, torch.tensor([3, 12], device=DEV), torch.tensor([4, 5], device=DEV),
                   status=status)
    torch.cuda.synchronize()
    assert (kc[4] == 1).all() and (kc[5] == 0).all()
    assert int(status.item()) & pa.PA_DEV_BAD_BLOCK_ID


def _write_tokens(kc, vc, bm, seq, start, vals_k, vals_v, B, x):
    """Store new tokens' K/V at their slots (test-side cache write)."""
    bt, _ = bm.export([seq])
    for i in range(vals_k.shape[1]):
        t = start + i
        pb, o = int(bt[0, t // B]), t % B
        kc[pb, :, :, o, :] = vals_k[:, i].reshape(kc.shape[1], -1, x)
        vc[pb, :, :, o] = vals_v[:, i]


@pytest.mark.parametrize("kv", [W.BF16, W.FP8_E4M3])
def test_decode_over_block_manager_tables_with_copy_on_write(kv):
    B, Hk, G, D = 16, 2, 4, 128
    x = 8 if kv == W.BF16 else 16
    NB, MAXB = 64, 12
    bm = pa.BlockManager(NB, B, MAXB)
    shape_k, shape_v = (NB, Hk, D // x, B, x), (NB, Hk, D, B)
    if kv == W.BF16:
        kc = torch.full(shape_k, float("nan"), dtype=torch.bfloat16, device=DEV)
        vc = torch.full(shape_v, float("nan"), dtype=torch.bfloat16, device=DEV)
    else:
        kc = torch.full(shape_k, 0x7F, dtype=torch.uint8, device=DEV)
        vc = torch.full(shape_v, 0x7F, dtype=torch.uint8, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(7)

    def draw(n):
        a = torch.randn((Hk, n, D), generator=g, device=DEV)
        b = torch.randn((Hk, n, D), generator=g, device=DEV)
        if kv == W.BF16:
            return a.to(torch.bfloat16), b.to(torch.bfloat16)
        enc = lambda t: (t / 0.05).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        return enc(a), enc(b)

    prompt = bm.add_sequence()
    bm.append(prompt, 70)  # 4 full blocks + 6 tokens in a fifth
    k, v = draw(70)
    _write_tokens(kc, vc, bm, prompt, 0, k, v, B, x)
    kids = [bm.fork(prompt) for _ in range(3)]
    for n_new, kid in zip((1, 9, 40), kids):
        start = bm.seq_len(kid)
        cow = bm.append(kid, n_new)
        assert cow is not None  # the shared fifth block is partly filled
        pa.copy_blocks(kc, vc, torch.tensor([cow[0]], device=DEV),
                       torch.tensor([cow[1]], device=DEV), kv)
        k, v = draw(n_new)
        _write_tokens(kc, vc, bm, kid, start, k, v, B, x)
    seqs = [prompt] + kids
    bt, sl = bm.export(seqs)
    cfg = W.PagedConfig("bm", num_seqs=4, num_heads=Hk * G, num_kv_heads=Hk, head_size=D,
                        block_size=B, num_blocks=NB, seq_len_lo=1, seq_len_hi=MAXB * B,
                        kv_dtype=kv, k_scale=0.05, v_scale=0.05)
    q = torch.randn((4, Hk * G, D), generator=g, device=DEV).to(torch.bfloat16)
    ks = torch.tensor([0.05], device=DEV)
    wl = W.Workload(cfg, q, kc, vc, torch.from_numpy(bt).to(DEV), torch.from_numpy(sl).to(DEV),
                    ks, ks.clone())
    out = torch.empty_like(q)
    pa.decode(out, q, kc, vc, Hk, cfg.scale, wl.block_tables, wl.seq_lens, B, cfg.max_seq_len,
              kv, wl.k_scale, wl.v_scale)
    torch.cuda.synchronize()
    compare(out, run_oracle(wl), kv, "block-manager tables")
    # the prompt kept its own tokens: its row equals a decode over its table alone
    assert sl.tolist() == [70, 71, 79, 110]
