"""Checks that tie the fp64 oracle to facts outside itself.

Each ``pin_*`` function takes an oracle library handle (the real build, or a
copy with a planted mistake) and raises AssertionError when the oracle
disagrees with:

* dense attention on the same K/V laid out contiguously, computed by
  torch's scaled_dot_product_attention in fp64 (a library routine), with the
  paged layout produced here by reshapes/permutes, not by the oracle's index
  formula;
* itself under a random relabelling of physical blocks (bit-identical);
* the closed form for uniform logits (q = 0 gives the mean of V);
* seq_len = 1 (the output is V_0 exactly);
* brute force in scalar Python (math.exp / math.fsum) for T <= 4;
* a hand-worked golden case (tests/golden/tiny_paged_case.txt);
* torch's e4m3 / bf16 conversions for every code.
"""

from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# contiguous <-> paged helpers written with reshapes, independent of the
# oracle's scalar index arithmetic
# ---------------------------------------------------------------------------

def paged_from_dense(Kd, Vd, seq_lens, block_tables, num_blocks, B, x, fill):
    """Kd, Vd: lists over s of [Hk, T_s, D] code tensors.  Returns paged caches
    [num_blocks, Hk, D/x, B, x] and [num_blocks, Hk, D, B] filled with ``fill``
    everywhere no token lives."""
    Hk, _, D = Kd[0].shape
    dt = Kd[0].dtype
    kc = torch.full((num_blocks, Hk, D // x, B, x), 0, dtype=dt)
    vc = torch.full((num_blocks, Hk, D, B), 0, dtype=dt)
    kc.view(torch.uint8 if dt == torch.uint8 else torch.int16).fill_(fill)
    vc.view(torch.uint8 if dt == torch.uint8 else torch.int16).fill_(fill)
    for s, T in enumerate(seq_lens):
        nb = -(-T // B)
        if nb == 0:
            continue
        pad = nb * B - T
        k = Kd[s]
        v = Vd[s]
        if pad:
            kpad = torch.zeros((Hk, pad, D), dtype=dt)
            kpad.view(torch.uint8 if dt == torch.uint8 else torch.int16).fill_(fill)
            k = torch.cat([k, kpad], dim=1)
            v = torch.cat([v, kpad.clone()], dim=1)
        # [Hk, nb*B, D] -> [Hk, nb, B, D/x, x] -> [nb, Hk, D/x, B, x]
        kp = k.reshape(Hk, nb, B, D // x, x).permute(1, 0, 3, 2, 4)
        # [Hk, nb*B, D] -> [Hk, nb, B, D] -> [nb, Hk, D, B]
        vp = v.reshape(Hk, nb, B, D).permute(1, 0, 3, 2)
        ids = torch.as_tensor(block_tables[s][:nb], dtype=torch.int64)
        kc[ids] = kp.contiguous()
        vc[ids] = vp.contiguous()
    return kc, vc


def decode_codes(t, kv):
    """Codes -> float64 with torch's own converters."""
    if kv == oracle.KV_BF16:
        return t.view(torch.bfloat16).to(torch.float64)
    return t.view(torch.float8_e4m3fn).to(torch.float64)


class Case:
    """A random paged problem plus its dense description."""

    def __init__(self, seed, S, Hq, Hk, D, B, seq_lens, kv=oracle.KV_BF16, k_scale=1.0,
                 v_scale=1.0, spare_blocks=5):
        g = torch.Generator().manual_seed(seed)
        self.S, self.Hq, self.Hk, self.D, self.B = S, Hq, Hk, D, B
        self.kv, self.k_scale, self.v_scale = kv, k_scale, v_scale
        self.x = 8 if kv == oracle.KV_BF16 else 16
        self.seq_lens = list(seq_lens)
        self.scale = 1.0 / math.sqrt(D)
        nbs = [-(-T // B) for T in self.seq_lens]
        self.num_blocks = sum(nbs) + spare_blocks
        maxb = max(max(nbs), 1)
        perm = torch.randperm(self.num_blocks, generator=g).tolist()
        self.block_tables = np.full((S, maxb), -1, dtype=np.int32)
        k = 0
        for s, nb in enumerate(nbs):
            self.block_tables[s, :nb] = perm[k:k + nb]
            k += nb
        self.q = torch.randn((S, Hq, D), generator=g).to(torch.bfloat16)
        self.Kd, self.Vd = [], []
        for T in self.seq_lens:
            a = torch.randn((Hk, T, D), generator=g)
            b = torch.randn((Hk, T, D), generator=g)
            self.Kd.append(self._enc(a, k_scale))
            self.Vd.append(self._enc(b, v_scale))
        self.fill = 0x7FC0 if kv == oracle.KV_BF16 else 0x7F
        self.build()

    def _enc(self, a, s):
        if self.kv == oracle.KV_BF16:
            return a.to(torch.bfloat16).view(torch.int16)
        return (a / s).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)

    def build(self):
        self.kc, self.vc = paged_from_dense(self.Kd, self.Vd, self.seq_lens, self.block_tables,
                                            self.num_blocks, self.B, self.x, self.fill)

    def run(self, lib, **kw):
        return oracle.pa_decode(self.q, self.kc, self.vc, self.Hk, self.scale, self.block_tables,
                                np.asarray(self.seq_lens, np.int32), self.B, self.kv,
                                self.k_scale, self.v_scale, x=self.x, lib=lib, **kw)

    def dense(self, alibi_slopes=None):
        """fp64 SDPA on the contiguous K/V (library routine); an ALiBi bias
        enters as SDPA's additive float mask."""
        G = self.Hq // self.Hk
        out = torch.zeros((self.S, self.Hq, self.D), dtype=torch.float64)
        for s, T in enumerate(self.seq_lens):
            if T == 0:
                continue
            K = decode_codes(self.Kd[s], self.kv) * (self.k_scale if self.kv else 1.0)
            V = decode_codes(self.Vd[s], self.kv) * (self.v_scale if self.kv else 1.0)
            K = K.repeat_interleave(G, dim=0)  # [Hq, T, D]
            V = V.repeat_interleave(G, dim=0)
            q = self.q[s].to(torch.float64).unsqueeze(1)  # [Hq, 1, D]
            mask = None
            if alibi_slopes is not None:
                pos = torch.arange(T, dtype=torch.float64) - (T - 1)
                mask = (torch.as_tensor(alibi_slopes, dtype=torch.float32).to(torch.float64)
                        [:, None, None] * pos[None, None, :])
            o = F.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=self.scale)
            out[s] = o[:, 0, :]
        return out.numpy()


DENSE_CASES = [
    dict(seed=1, S=3, Hq=4, Hk=4, D=64, B=16, seq_lens=[1, 37, 80]),
    dict(seed=2, S=2, Hq=8, Hk=2, D=128, B=16, seq_lens=[33, 16]),
    dict(seed=3, S=2, Hq=4, Hk=1, D=128, B=32, seq_lens=[95, 64]),
    dict(seed=4, S=3, Hq=8, Hk=2, D=128, B=16, seq_lens=[17, 50, 3],
         kv=oracle.KV_E4M3, k_scale=0.05, v_scale=0.05),
    dict(seed=5, S=2, Hq=16, Hk=1, D=64, B=16, seq_lens=[40, 15],
         kv=oracle.KV_E4M3, k_scale=0.03, v_scale=0.07),
]


def pin_dense_equivalence(lib):
    for kw in DENSE_CASES:
        c = Case(**kw)
        got = c.run(lib)
        ref = c.dense()
        err = np.max(np.abs(got - ref))
        assert err < 1e-12, f"dense equivalence {kw}: max |diff| {err}"


def pin_permutation_invariance(lib):
    for kw in DENSE_CASES[:2] + DENSE_CASES[3:4]:
        c = Case(**kw)
        a = c.run(lib)
        g = torch.Generator().manual_seed(99)
        relabel = torch.randperm(c.num_blocks, generator=g).numpy().astype(np.int32)
        bt = c.block_tables.copy()
        mask = bt >= 0
        bt[mask] = relabel[bt[mask]]
        c.block_tables = bt
        c.build()
        b = c.run(lib)
        assert np.array_equal(a, b), f"permutation invariance {kw}"


def pin_uniform_logits(lib):
    for kw in (DENSE_CASES[0], DENSE_CASES[3]):
        c = Case(**kw)
        c.q = torch.zeros_like(c.q)
        got = c.run(lib)
        G = c.Hq // c.Hk
        for s, T in enumerate(c.seq_lens):
            V = decode_codes(c.Vd[s], c.kv).numpy() * (c.v_scale if c.kv else 1.0)
            mean = V.mean(axis=1)  # [Hk, D]
            for h in range(c.Hq):
                err = np.max(np.abs(got[s, h] - mean[h // G]))
                assert err < 1e-13, f"uniform logits s={s} h={h}: {err}"


def pin_seq_len_one(lib):
    for kv in (oracle.KV_BF16, oracle.KV_E4M3):
        c = Case(seed=7, S=3, Hq=4, Hk=2, D=64, B=16, seq_lens=[1, 1, 1], kv=kv,
                 k_scale=0.05, v_scale=0.05)
        got = c.run(lib)
        for s in range(c.S):
            V = decode_codes(c.Vd[s], c.kv).numpy() * (c.v_scale if c.kv else 1.0)
            for h in range(c.Hq):
                assert np.array_equal(got[s, h], V[h // 2, 0]), f"seq_len=1 s={s} h={h}"


def _brute(q, Kd, Vd, seq_lens, Hq, Hk, scale, kv, ks, vs):
    """Scalar Python: logits, max, exp, fsum, weighted sum."""
    G = Hq // Hk
    S = len(seq_lens)
    out = []
    for s in range(S):
        rows = []
        K = decode_codes(Kd[s], kv).tolist()
        V = decode_codes(Vd[s], kv).tolist()
        qs = q[s].to(torch.float64).tolist()
        for h in range(Hq):
            g = h // G
            T = seq_lens[s]
            D = len(qs[h])
            if T == 0:
                rows.append([0.0] * D)
                continue
            logits = [scale * math.fsum(qs[h][d] * (K[g][t][d] * ks) for d in range(D))
                      for t in range(T)]
            m = max(logits)
            w = [math.exp(l - m) for l in logits]
            den = math.fsum(w)
            rows.append([math.fsum(w[t] * V[g][t][d] * vs for t in range(T)) / den
                         for d in range(D)])
        out.append(rows)
    return np.array(out)


def pin_brute_force(lib):
    specs = [
        dict(seed=11, S=2, Hq=2, Hk=1, D=8, B=2, seq_lens=[3, 4]),
        dict(seed=12, S=3, Hq=4, Hk=2, D=64, B=16, seq_lens=[4, 1, 2]),
        dict(seed=13, S=2, Hq=2, Hk=2, D=32, B=2, seq_lens=[4, 3],
             kv=oracle.KV_E4M3, k_scale=0.05, v_scale=0.25),
    ]
    for kw in specs:
        c = Case(**kw)
        got = c.run(lib)
        ks = c.k_scale if c.kv else 1.0
        vs = c.v_scale if c.kv else 1.0
        ref = _brute(c.q, c.Kd, c.Vd, c.seq_lens, c.Hq, c.Hk, c.scale, c.kv, ks, vs)
        err = np.max(np.abs(got - ref))
        assert err < 1e-13, f"brute force {kw}: {err}"


def load_golden(name="tiny_paged_case.txt"):
    spec = {"key": [], "value": [], "nan_slot": [], "nan_block": [], "query": [], "expect": []}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            tag, *rest = line.split()
            if tag == "sizes":
                spec["sizes"] = {k: float(v) if k == "scale" else int(v)
                                 for k, v in (r.split("=") for r in rest)}
            elif tag == "block_table":
                spec["block_table"] = [int(v) for v in rest]
            else:
                spec[tag].append([float(v) for v in rest])
    return spec


def pin_golden(lib):
    g = load_golden()
    z = g["sizes"]
    S, Hq, Hk, D, B, x, NB = z["S"], z["Hq"], z["Hk"], z["D"], z["B"], z["x"], z["num_blocks"]
    kc = torch.zeros((NB, Hk, D // x, B, x), dtype=torch.bfloat16)
    vc = torch.zeros((NB, Hk, D, B), dtype=torch.bfloat16)
    for b, hk, j, o, l, val in g["key"]:
        kc[int(b), int(hk), int(j), int(o), int(l)] = val
    for b, hk, d, o, val in g["value"]:
        vc[int(b), int(hk), int(d), int(o)] = val
    for b, o in g["nan_slot"]:
        kc[int(b), :, :, int(o), :] = float("nan")
        vc[int(b), :, :, int(o)] = float("nan")
    for (b,) in g["nan_block"]:
        kc[int(b)] = float("nan")
        vc[int(b)] = float("nan")
    q = torch.zeros((S, Hq, D), dtype=torch.bfloat16)
    for h, d, val in g["query"]:
        q[0, int(h), int(d)] = val
    bt = np.array([g["block_table"]], dtype=np.int32)
    sl = np.array([z["seq_len"]], dtype=np.int32)
    got = oracle.pa_decode(q, kc, vc, Hk, z["scale"], bt, sl, B, oracle.KV_BF16, x=x, lib=lib)
    want = np.zeros((S, Hq, D))
    e = math.e
    for h, d, a, b, c, f in g["expect"]:
        want[0, int(h), int(d)] = (a + b * e) / (c + f * e)
    err = np.max(np.abs(got - want))
    assert err < 1e-15, f"golden case: {err}"


def pin_e4m3_table(lib):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = lib.oracle_e4m3_to_double(c)
        if math.isnan(ref[c]):
            assert math.isnan(v), f"e4m3 code {c:#x} should be NaN"
        else:
            assert v == ref[c] and math.copysign(1, v) == math.copysign(1, ref[c]), \
                f"e4m3 code {c:#x}: {v} vs {ref[c]}"
    # spot values of the format: max finite, smallest subnormal, smallest normal, one
    assert lib.oracle_e4m3_to_double(0x7E) == 448.0
    assert lib.oracle_e4m3_to_double(0x01) == 2.0 ** -9
    assert lib.oracle_e4m3_to_double(0x08) == 2.0 ** -6
    assert lib.oracle_e4m3_to_double(0x38) == 1.0
    assert lib.oracle_e4m3_to_double(0xB8) == -1.0


def pin_bf16_table(lib):
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    for b in range(0, 65536, 1):
        v = lib.oracle_bf16_to_double(b)
        r = ref[b]
        if math.isnan(r):
            assert math.isnan(v)
        else:
            assert v == r, f"bf16 {b:#x}"


def _slopes(Hq, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(Hq, generator=g) * 0.5).to(torch.float32)


def pin_alibi_dense(lib):
    for kw in (DENSE_CASES[0], DENSE_CASES[2], DENSE_CASES[3]):
        c = Case(**kw)
        sl = _slopes(c.Hq, 21)
        got = c.run(lib, alibi_slopes=sl)
        ref = c.dense(alibi_slopes=sl)
        err = np.max(np.abs(got - ref))
        assert err < 1e-12, f"alibi dense {kw}: {err}"


def pin_alibi_brute_force(lib):
    c = Case(seed=14, S=2, Hq=4, Hk=2, D=8, B=2, seq_lens=[4, 3])
    sl = _slopes(4, 22).tolist()
    got = c.run(lib, alibi_slopes=torch.tensor(sl, dtype=torch.float32))
    G = 2
    for s, T in enumerate(c.seq_lens):
        K = decode_codes(c.Kd[s], c.kv).tolist()
        V = decode_codes(c.Vd[s], c.kv).tolist()
        qs = c.q[s].to(torch.float64).tolist()
        for h in range(4):
            g = h // G
            lg = [c.scale * math.fsum(qs[h][d] * K[g][t][d] for d in range(8))
                  + float(torch.tensor(sl[h], dtype=torch.float32)) * (t - (T - 1))
                  for t in range(T)]
            m = max(lg)
            w = [math.exp(x - m) for x in lg]
            den = math.fsum(w)
            want = [math.fsum(w[t] * V[g][t][d] for t in range(T)) / den for d in range(8)]
            assert np.max(np.abs(got[s, h] - np.array(want))) < 1e-13, (s, h)


def pin_alibi_zero_slopes_is_plain(lib):
    c = Case(**DENSE_CASES[1])
    a = c.run(lib)
    b = c.run(lib, alibi_slopes=torch.zeros(c.Hq, dtype=torch.float32))
    assert np.array_equal(a, b), "zero ALiBi slopes must leave the output unchanged"


def _pair_list(c, seed, n):
    """n (sequence, q head) pairs in random order, with repeats, covering the
    first and last row; every pair's head runs over all of a kv head's group."""
    g = torch.Generator().manual_seed(seed)
    pairs = [(0, 0), (c.S - 1, c.Hq - 1)]
    for _ in range(n):
        pairs.append((int(torch.randint(0, c.S, (1,), generator=g)),
                      int(torch.randint(0, c.Hq, (1,), generator=g))))
    pairs.append(pairs[2])  # a repeated row
    perm = torch.randperm(len(pairs), generator=g).tolist()
    return [pairs[i] for i in perm]


def pin_sampled_rows(lib):
    """The oracle's sampled-row mode (an explicit list of (s, h) pairs, the
    mode the full-size GPU checks read their references through): each
    listed row must equal dense SDPA on the contiguous K/V of that
    (sequence, query head) to 1e-12, and must be bit-identical to the same
    row of the whole-batch result."""
    for i, kw in enumerate(DENSE_CASES[1:] + [DENSE_CASES[0]]):
        c = Case(**kw)
        pairs = _pair_list(c, 70 + i, 3 * c.S * c.Hq // 2)
        got = c.run(lib, pairs=pairs)
        assert got.shape == (len(pairs), c.D), got.shape
        dense = c.dense()
        full = c.run(lib)
        for r, (s, h) in enumerate(pairs):
            err = np.max(np.abs(got[r] - dense[s, h]))
            assert err < 1e-12, f"sampled row {r} = ({s}, {h}) of {kw}: {err}"
            assert np.array_equal(got[r], full[s, h]), f"sampled row ({s}, {h}) of {kw}"
    # ALiBi slopes follow the listed query head, not the row's position.
    c = Case(**DENSE_CASES[1])
    sl = _slopes(c.Hq, 23)
    pairs = _pair_list(c, 80, 12)
    got = c.run(lib, pairs=pairs, alibi_slopes=sl)
    dense = c.dense(alibi_slopes=sl)
    for r, (s, h) in enumerate(pairs):
        assert np.max(np.abs(got[r] - dense[s, h])) < 1e-12, f"sampled ALiBi row ({s}, {h})"


ALL_PINS = [pin_golden, pin_dense_equivalence, pin_permutation_invariance, pin_uniform_logits,
            pin_seq_len_one, pin_brute_force, pin_e4m3_table, pin_bf16_table, pin_alibi_dense,
            pin_alibi_brute_force, pin_alibi_zero_slopes_is_plain, pin_sampled_rows]
