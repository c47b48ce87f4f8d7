"""The fp64 oracle against facts outside itself (CPU only)."""

import os
import shutil
import subprocess
import sys
import tempfile

import pytest

import oracle
import oracle_pins as pins


@pytest.fixture(scope="module")
def lib():
    oracle.build(force=True)
    return oracle.load()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(lib, pin):
    pin(lib)


def test_oracle_uses_threads(lib):
    assert oracle.max_threads() >= 1


# ---------------------------------------------------------------------------
# Planted mistakes: each plausible slip in the oracle must trip at least one
# pin.  The mutation is a textual edit of a private copy of pa_oracle.c built
# into a temporary library; the real oracle is untouched.  Every mutant keeps
# all reads inside the buffers it is given.
# ---------------------------------------------------------------------------

MUTANTS = {
    "gqa head map h % Hk": ("h / G, k_scale", "h % Hk, k_scale"),
    "scale dropped": ("logit[t] = scale * acc + slope", "logit[t] = acc + slope"),
    "x-lane reversed": (") * x) + d % x;", ") * x) + (x - 1 - d % x);"),
    "V slot reversed": ("+ d) * B + o;", "+ d) * B + (B - 1 - o);"),
    "identity block map": ("int64_t pb = (int64_t)bt_row[t / B];\n        int o = t % B;\n        double acc",
                           "int64_t pb = (int64_t)(t / B);\n        int o = t % B;\n        double acc"),
    "e4m3 exponent bias": ("e - 10);", "e - 9);"),
    "e4m3 subnormal scale": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "normalised by T": ("out_row[d] /= denom;", "out_row[d] /= (double)T;"),
    "k_scale on V": ("load_elem(value_cache, vi, kv_dtype, v_scale)",
                     "load_elem(value_cache, vi, kv_dtype, k_scale)"),
    "ALiBi bias sign": ("slope * (double)(t - (T - 1));", "slope * (double)((T - 1) - t);"),
    "ALiBi slope of the kv head": ("(double)alibi_slopes[h]", "(double)alibi_slopes[h / G]"),
    # the sampled-row mode (rows listed as (s, h) pairs)
    "pairs: s and h swapped": ("int s = pairs ? pairs[2 * i] : i / Hq;\n            int h = pairs ? pairs[2 * i + 1] : i % Hq;",
                               "int s = pairs ? pairs[2 * i + 1] % S : i / Hq;\n            int h = pairs ? pairs[2 * i] : i % Hq;"),
    "pairs: first pair for every row": ("int s = pairs ? pairs[2 * i] : i / Hq;\n            int h = pairs ? pairs[2 * i + 1] : i % Hq;",
                                        "int s = pairs ? pairs[0] : i / Hq;\n            int h = pairs ? pairs[1] : i % Hq;"),
    "pairs: last pair dropped": ("int n_rows = pairs ? n_pairs : S * Hq;",
                                 "int n_rows = pairs ? n_pairs - 1 : S * Hq;"),
    "pairs: row order reversed": ("one_row(out + (int64_t)i * D,",
                                  "one_row(out + (int64_t)(pairs ? n_rows - 1 - i : i) * D,"),
    "last token dropped": ("for (t = 0; t < T; ++t) {\n        int64_t pb = (int64_t)bt_row[t / B];\n        int o = t % B;\n        double p",
                           "for (t = 0; t < T - (T > 1); ++t) {\n        int64_t pb = (int64_t)bt_row[t / B];\n        int o = t % B;\n        double p"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation anchor for {name!r} not unique"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    so = str(tmp_path / "libmutant.so")
    oracle.compile_oracle(str(mpath), so)
    mlib = oracle.load(so)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(mlib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {name!r}"
