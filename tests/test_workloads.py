"""The seeded input generator: shapes, determinism, poison, block-id structure."""

import torch

from paged_kv_cache_471_b200 import workloads as W


def test_configs_match_stated_sizes():
    c = W.WORKLOADS
    assert (c[1].num_seqs, c[1].num_heads, c[1].num_kv_heads, c[1].head_size,
            c[1].block_size, c[1].num_blocks) == (4, 8, 8, 64, 16, 128)
    assert (c[2].num_seqs, c[2].num_heads, c[2].head_size, c[2].seq_len_hi) == (64, 32, 128, 4096)
    assert (c[3].num_heads, c[3].num_kv_heads, c[3].seq_len_lo, c[3].seq_len_hi) == (64, 8, 512, 8192)
    assert c[4].kv_dtype == W.FP8_E4M3 and c[4].k_scale == 0.05 and c[4].num_blocks == 262144
    assert c[5].block_size == 32 and c[5].shared_prefix_blocks == 1024
    assert c[4].x == 16 and c[2].x == 8


def test_tables_deterministic_and_distinct():
    for idx in (1, 3):
        cfg = W.WORKLOADS[idx]
        a = W.draw_tables(cfg)
        b = W.draw_tables(cfg)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
        sl, bt = a
        assert sl.min() >= cfg.seq_len_lo and sl.max() <= cfg.seq_len_hi
        used = bt[bt >= 0]
        assert used.numel() == used.unique().numel()
        for s, t in enumerate(sl.tolist()):
            n = -(-t // cfg.block_size)
            assert (bt[s, :n] >= 0).all() and (bt[s, n:] == -1).all()


def test_full_pool_permutation_config4():
    cfg = W.WORKLOADS[4]
    sl, bt = W.draw_tables(cfg)
    assert bt.shape == (256, 1024)
    assert torch.equal(bt.flatten().sort().values, torch.arange(262144, dtype=torch.int32))


def test_shared_prefix_config5():
    cfg = W.WORKLOADS[5]
    sl, bt = W.draw_tables(cfg)
    assert (bt[:, :1024] == bt[0:1, :1024]).all()
    rest = bt[:, 1024:]
    assert rest.numel() == rest.unique().numel()
    assert not bool(torch.isin(rest, bt[0, :1024]).any())


def test_poison_and_data():
    cfg = W.reduced(1, num_seqs=3, seq_len_hi=40, seq_len_lo=17)
    wl = W.make_workload(cfg)
    kc, vc = wl.key_cache, wl.value_cache
    bt, sl = wl.block_tables, wl.seq_lens
    ref = set(bt[bt >= 0].tolist())
    for b in range(cfg.num_blocks):
        if b not in ref:
            assert torch.isnan(kc[b].float()).all() and torch.isnan(vc[b].float()).all()
    for s, t in enumerate(sl.tolist()):
        r = t % cfg.block_size
        last = int(bt[s, (t - 1) // cfg.block_size])
        if r:
            assert torch.isnan(kc[last, :, :, r:, :].float()).all()
            assert not torch.isnan(kc[last, :, :, :r, :].float()).any()
            assert torch.isnan(vc[last, :, :, r:].float()).all()


def test_fp8_codes():
    cfg = W.reduced(4, num_seqs=2, seq_len_hi=64, seq_len_lo=64)
    wl = W.make_workload(cfg)
    assert wl.key_cache.dtype == torch.uint8
    ref = wl.block_tables[wl.block_tables >= 0].long()
    codes = wl.key_cache[ref]
    assert not (codes == W.E4M3_NAN_CODE).any() and not (codes == 0xFF).any()
    vals = codes.view(torch.float8_e4m3fn).float() * 0.05
    assert 0.8 < vals.std().item() < 1.2
