"""Seeded synthetic inputs for paged decode attention.

This module only *draws inputs*: sequence lengths, block tables, the paged
K/V caches, the query and the FP8 scales.  It holds none of the attention
arithmetic, and both the CUDA path (through the tests and the bench) and the
CPU oracle read the tensors it makes.

Layouts follow the pages' description of the legacy kernel's arguments
("Why PagedAttention was retired", section 2, the k_cache/v_cache comments):

* key_cache   ``[num_blocks, num_kv_heads, head_size/x, block_size, x]``
* value_cache ``[num_blocks, num_kv_heads, head_size, block_size]``
* block_tables int32 ``[num_seqs, max_blocks_per_seq]`` (section 1 of the same
  page: sequence ``s`` reads its j-th logical block from physical block
  ``block_tables[s][j]``)
* seq_lens int32 ``[num_seqs]``

``x`` is not defined on the pages; it is taken as 16 bytes / element size
(8 for bf16, 16 for fp8), so that one x-group is one 16-byte vector.

Poison: every physical block that no sequence references, and every slot of a
sequence's last block at or beyond its length, holds NaN (bf16 0x7FC0,
e4m3 0x7F).  A kernel that reads outside the logical KV shows it as NaN.
Unused block-table entries hold -1.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

BF16 = "bf16"
FP8_E4M3 = "fp8_e4m3"

BF16_NAN_BITS = 0x7FC0
E4M3_NAN_CODE = 0x7F
E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class PagedConfig:
    """One synthetic decode batch.  Sizes only; no arithmetic."""

    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    num_blocks: int
    seq_len_lo: int
    seq_len_hi: int
    kv_dtype: str = BF16
    k_scale: float = 1.0
    v_scale: float = 1.0
    shared_prefix_blocks: int = 0
    seed: int = 1000

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_size)

    @property
    def max_seq_len(self) -> int:
        return self.seq_len_hi

    @property
    def max_blocks_per_seq(self) -> int:
        return -(-self.seq_len_hi // self.block_size)

    @property
    def elem_bytes(self) -> int:
        return 1 if self.kv_dtype == FP8_E4M3 else 2

    @property
    def x(self) -> int:
        return 16 // self.elem_bytes

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    def key_cache_shape(self):
        return (self.num_blocks, self.num_kv_heads, self.head_size // self.x,
                self.block_size, self.x)

    def value_cache_shape(self):
        return (self.num_blocks, self.num_kv_heads, self.head_size, self.block_size)

    def page_bytes(self) -> int:
        """Bytes of one (block, kv head) K page; the V page has the same size."""
        return self.head_size * self.block_size * self.elem_bytes

    def replace(self, **kw) -> "PagedConfig":
        return dataclasses.replace(self, **kw)


# The five workloads of the decode benchmark (sizes as stated for each).
WORKLOADS = {
    1: PagedConfig("tiny MHA decode: 4 seqs, 8/8 heads, D=64, B=16, T~U[1,256], bf16",
                   num_seqs=4, num_heads=8, num_kv_heads=8, head_size=64, block_size=16,
                   num_blocks=128, seq_len_lo=1, seq_len_hi=256, seed=1001),
    2: PagedConfig("Llama-style MHA decode: 64 seqs, 32/32 heads, D=128, B=16, T=4096, bf16",
                   num_seqs=64, num_heads=32, num_kv_heads=32, head_size=128, block_size=16,
                   num_blocks=131072, seq_len_lo=4096, seq_len_hi=4096, seed=1002),
    3: PagedConfig("GQA decode: 128 seqs, 64/8 heads, D=128, B=16, T~U[512,8192], bf16",
                   num_seqs=128, num_heads=64, num_kv_heads=8, head_size=128, block_size=16,
                   num_blocks=131072, seq_len_lo=512, seq_len_hi=8192, seed=1003),
    4: PagedConfig("FP8 KV decode: 256 seqs, 32/8 heads, D=128, B=16, T=16384, e4m3 K/V",
                   num_seqs=256, num_heads=32, num_kv_heads=8, head_size=128, block_size=16,
                   num_blocks=262144, seq_len_lo=16384, seq_len_hi=16384,
                   kv_dtype=FP8_E4M3, k_scale=0.05, v_scale=0.05, seed=1004),
    5: PagedConfig("long-context split-KV: 8 seqs, 32/8 heads, D=128, B=32, T=131072, "
                   "shared 1024-block prefix, bf16",
                   num_seqs=8, num_heads=32, num_kv_heads=8, head_size=128, block_size=32,
                   num_blocks=131072, seq_len_lo=131072, seq_len_hi=131072,
                   shared_prefix_blocks=1024, seed=1005),
}


def reduced(idx: int, num_seqs: Optional[int] = None, seq_len_hi: Optional[int] = None,
            seq_len_lo: Optional[int] = None, num_blocks: Optional[int] = None,
            shared_prefix_blocks: Optional[int] = None) -> PagedConfig:
    """A smaller batch with the same heads, head size, block size, dtype and
    length mix as WORKLOADS[idx], small enough for the oracle to finish in seconds."""
    c = WORKLOADS[idx]
    hi = seq_len_hi if seq_len_hi is not None else c.seq_len_hi
    lo = seq_len_lo if seq_len_lo is not None else min(c.seq_len_lo, hi)
    S = num_seqs if num_seqs is not None else c.num_seqs
    pref = shared_prefix_blocks if shared_prefix_blocks is not None else c.shared_prefix_blocks
    need = pref + S * (-(-hi // c.block_size) - pref)
    nb = num_blocks if num_blocks is not None else max(need + 16, 64)
    return c.replace(name=c.name + f" (reduced: S={S}, T<={hi})", num_seqs=S,
                     seq_len_lo=lo, seq_len_hi=hi, num_blocks=nb,
                     shared_prefix_blocks=pref)


def draw_tables(cfg: PagedConfig, seq_lens: Optional[torch.Tensor] = None):
    """seq_lens int32 [S] and block_tables int32 [S, max_blocks_per_seq] on the CPU.

    Physical ids come from one seeded random permutation of all blocks, handed
    out in (sequence, logical block) order; with a shared prefix, the first
    ``shared_prefix_blocks`` entries of every row are the same ids.  Entries past
    a sequence's last block are -1.
    """
    g = torch.Generator().manual_seed(cfg.seed)
    if seq_lens is None:
        seq_lens = torch.randint(cfg.seq_len_lo, cfg.seq_len_hi + 1, (cfg.num_seqs,),
                                 generator=g, dtype=torch.int64)
    else:
        seq_lens = torch.as_tensor(seq_lens, dtype=torch.int64)
        g.manual_seed(cfg.seed + 7)
    B = cfg.block_size
    maxb = max(cfg.max_blocks_per_seq, 1)
    perm = torch.randperm(cfg.num_blocks, generator=g)
    nblk = [(-(-int(t) // B)) for t in seq_lens.tolist()]
    pref = cfg.shared_prefix_blocks
    need = pref + sum(max(n - pref, 0) for n in nblk)
    if need > cfg.num_blocks:
        raise ValueError(f"{cfg.name}: needs {need} blocks, pool has {cfg.num_blocks}")
    bt = torch.full((cfg.num_seqs, maxb), -1, dtype=torch.int32)
    shared = perm[:pref]
    nxt = pref
    for s, n in enumerate(nblk):
        k = min(n, pref)
        bt[s, :k] = shared[:k].to(torch.int32)
        rest = n - k
        bt[s, k:n] = perm[nxt:nxt + rest].to(torch.int32)
        nxt += rest
    return seq_lens.to(torch.int32), bt


def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _encode(vals: torch.Tensor, cfg: PagedConfig, which: str) -> torch.Tensor:
    if cfg.kv_dtype == BF16:
        return vals.to(torch.bfloat16)
    s = cfg.k_scale if which == "k" else cfg.v_scale
    codes = (vals / torch.tensor(s, dtype=torch.float32, device=vals.device))
    codes = codes.clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes.view(torch.uint8)


def _empty_cache(shape, cfg: PagedConfig, device):
    if cfg.kv_dtype == BF16:
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        t.view(torch.int16).fill_(BF16_NAN_BITS)
    else:
        t = torch.empty(shape, dtype=torch.uint8, device=device)
        t.fill_(E4M3_NAN_CODE)
    return t


def fill_caches(cfg: PagedConfig, seq_lens: torch.Tensor, block_tables: torch.Tensor,
                device="cpu", chunk_blocks: int = 8192):
    """NaN-poisoned K/V caches with N(0,1) data in every referenced block.

    Returns (key_cache, value_cache): bf16 tensors, or uint8 tensors holding
    e4m3 codes of N(0,1)/scale (clamped to +-448, round-to-nearest-even).
    """
    dev = torch.device(device)
    kc = _empty_cache(cfg.key_cache_shape(), cfg, dev)
    vc = _empty_cache(cfg.value_cache_shape(), cfg, dev)
    ids = block_tables[block_tables >= 0].unique().to(torch.int64)
    gen = torch.Generator(device=dev).manual_seed(cfg.seed + 1)
    ids_d = ids.to(dev)
    for i in range(0, ids.numel(), chunk_blocks):
        sel = ids_d[i:i + chunk_blocks]
        kc[sel] = _encode(_randn((sel.numel(),) + cfg.key_cache_shape()[1:], gen, dev), cfg, "k")
        vc[sel] = _encode(_randn((sel.numel(),) + cfg.value_cache_shape()[1:], gen, dev), cfg, "v")
    # Poison the slots of each last block that lie at or past the sequence end,
    # unless another sequence also maps that block (a shared block stays whole).
    B = cfg.block_size
    counts = torch.bincount(block_tables[block_tables >= 0].to(torch.int64).cpu(),
                            minlength=cfg.num_blocks)
    for s, t in enumerate(seq_lens.tolist()):
        r = t % B
        if t <= 0 or r == 0:
            continue
        pb = int(block_tables[s, t // B])
        if int(counts[pb]) > 1:
            continue
        if cfg.kv_dtype == BF16:
            kc[pb, :, :, r:, :].view(torch.int16).fill_(BF16_NAN_BITS)
            vc[pb, :, :, r:].view(torch.int16).fill_(BF16_NAN_BITS)
        else:
            kc[pb, :, :, r:, :].fill_(E4M3_NAN_CODE)
            vc[pb, :, :, r:].fill_(E4M3_NAN_CODE)
    return kc, vc


def draw_query(cfg: PagedConfig, device="cpu") -> torch.Tensor:
    """bf16 N(0,1) query [num_seqs, num_heads, head_size]."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(cfg.seed + 2)
    return _randn((cfg.num_seqs, cfg.num_heads, cfg.head_size), gen, dev).to(torch.bfloat16)


@dataclasses.dataclass
class Workload:
    cfg: PagedConfig
    query: torch.Tensor
    key_cache: torch.Tensor
    value_cache: torch.Tensor
    block_tables: torch.Tensor
    seq_lens: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor

    @property
    def kv_bytes(self) -> int:
        """K+V bytes a single pass must read: 2 pages' worth per referenced
        (token, kv head), counted per token."""
        tok = int(self.seq_lens.to(torch.int64).clamp(min=0).sum())
        c = self.cfg
        return 2 * tok * c.num_kv_heads * c.head_size * c.elem_bytes

    @property
    def unique_kv_bytes(self) -> int:
        """K+V bytes of distinct (block, kv head) pages referenced, counting the
        used slots of each distinct block once."""
        c = self.cfg
        B = c.block_size
        used = {}
        bt = self.block_tables.cpu()
        for s, t in enumerate(self.seq_lens.cpu().tolist()):
            n = -(-t // B)
            for j in range(n):
                pb = int(bt[s, j])
                slots = min(B, t - j * B)
                used[pb] = max(used.get(pb, 0), slots)
        tok = sum(used.values())
        return 2 * tok * c.num_kv_heads * c.head_size * c.elem_bytes

    @property
    def q_out_bytes(self) -> int:
        c = self.cfg
        return 2 * (c.num_seqs * c.num_heads * c.head_size * 2)


def make_workload(cfg: PagedConfig, device="cpu", seq_lens=None) -> Workload:
    sl, bt = draw_tables(cfg, seq_lens)
    kc, vc = fill_caches(cfg, sl, bt, device)
    q = draw_query(cfg, device)
    dev = torch.device(device)
    ks = torch.tensor([cfg.k_scale], dtype=torch.float32, device=dev)
    vs = torch.tensor([cfg.v_scale], dtype=torch.float32, device=dev)
    return Workload(cfg, q, kc, vc, bt.to(dev), sl.to(dev), ks, vs)
