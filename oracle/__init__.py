"""fp64 CPU oracle for paged decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``paged_kv_cache_471_b200``) never imports it, and the two share no code: the
oracle is plain C (``pa_oracle.c``) compiled with gcc, fp64, no fast-math,
OpenMP over output rows.

Every function here only marshals arguments; the arithmetic is in
``pa_oracle.c``, which cites the passages it follows.

Parity status of each oracle function (what pins it is in tests/test_oracle.py):
  * oracle_pa_decode   -- pinned: dense SDPA equivalence, block-permutation
    invariance, uniform-logit mean, seq_len = 1, brute force at T <= 4,
    a hand-derived golden case, planted-mistake sensitivity; with ALiBi
    slopes: SDPA with the additive bias as its mask, brute force, and zero
    slopes reproducing the unbiased result bit for bit.
  * e4m3 / bf16 decode -- pinned: all 256 / 65536 codes against torch's
    float8_e4m3fn / bfloat16 conversions, and spot values of the format.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "pa_oracle.c")
LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
          "-ffp-contract=off"]

KV_BF16 = 0
KV_E4M3 = 1

_lib = None


def compile_oracle(source: str = SOURCE, out: str = LIB) -> str:
    """Compile the C oracle with gcc into a shared library and return its path."""
    cmd = ["gcc", *CFLAGS, source, "-o", out, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SOURCE):
        compile_oracle()
    return LIB


def _bind(lib):
    lib.oracle_pa_decode.restype = ctypes.c_int
    lib.oracle_pa_decode.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_double,
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.oracle_bf16_to_double.restype = ctypes.c_double
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """The oracle library (built on first use).  ``path`` loads another build of
    the same source, e.g. a deliberately broken copy in a sensitivity test."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _np(t, dtype):
    """A C-contiguous numpy view of a CPU tensor or array, reinterpreted as dtype."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().cpu().contiguous()
            if t.dtype in (torch.bfloat16, torch.float16, torch.int16):
                t = t.view(torch.int16)
            elif t.dtype in (torch.float8_e4m3fn, torch.uint8, torch.int8):
                t = t.view(torch.uint8)
            t = t.numpy()
    except ImportError:
        pass
    return np.ascontiguousarray(t).view(dtype)


def pa_decode(query, key_cache, value_cache, num_kv_heads: int, scale: float, block_tables,
              seq_lens, block_size: int, kv_dtype: int = KV_BF16, k_scale: float = 1.0,
              v_scale: float = 1.0, x: int | None = None, pairs=None, threads: int = 0,
              lib=None, alibi_slopes=None) -> np.ndarray:
    """fp64 attention output.

    query bf16 [S, Hq, D]; caches in the paged layouts (bf16 or e4m3 codes);
    block_tables int32 [S, max_blocks]; seq_lens int32 [S].
    Returns float64 [S, Hq, D], or [len(pairs), D] when pairs = [(s, h), ...].
    """
    lib = lib or load()
    q = _np(query, np.uint16)
    S, Hq, D = q.shape
    elem = 2 if kv_dtype == KV_BF16 else 1
    kc = _np(key_cache, np.uint16 if elem == 2 else np.uint8)
    vc = _np(value_cache, np.uint16 if elem == 2 else np.uint8)
    if x is None:
        x = 16 // elem
    bt = _np(block_tables, np.int32)
    sl = _np(seq_lens, np.int32)
    if pairs is not None:
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        n_rows = pr.shape[0]
        pr_ptr = pr.ctypes.data
    else:
        pr = None
        n_rows = S * Hq
        pr_ptr = None
    out = np.zeros((n_rows, D), dtype=np.float64)
    slopes = None if alibi_slopes is None else np.ascontiguousarray(
        _np(alibi_slopes, np.float32), dtype=np.float32)
    if slopes is not None and slopes.shape != (Hq,):
        raise ValueError("alibi_slopes must have one entry per query head")
    rc = lib.oracle_pa_decode(out.ctypes.data, q.ctypes.data, kc.ctypes.data, vc.ctypes.data,
                              int(kv_dtype), S, Hq, int(num_kv_heads), D, int(block_size),
                              int(x), float(scale), bt.ctypes.data, bt.shape[1], sl.ctypes.data,
                              float(k_scale), float(v_scale), n_rows if pr is not None else 0,
                              pr_ptr, int(threads),
                              None if slopes is None else slopes.ctypes.data)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out if pairs is not None else out.reshape(S, Hq, D)


def e4m3_to_double(code: int) -> float:
    return load().oracle_e4m3_to_double(int(code) & 0xFF)


def bf16_to_double(bits: int) -> float:
    return load().oracle_bf16_to_double(int(bits) & 0xFFFF)


def max_threads() -> int:
    return load().oracle_max_threads()
