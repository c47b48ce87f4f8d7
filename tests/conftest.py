import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # Without any CUDA device, GPU tests are skipped rather than failed; on a
    # machine with a GPU they run and fail loudly if the library is missing.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this machine")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the parity statistics the GPU comparisons gathered: every
    full-size comparison in full, and the worst of each statistic over the
    rest."""
    mod = sys.modules.get("parity_helpers")
    log = getattr(mod, "PARITY_LOG", None) if mod is not None else None
    if not log:
        return
    tr = terminalreporter
    tr.section("parity against the fp64 oracle")
    fmt = "{:<58} rows {:>7}  max-abs {:.2e}  mean-abs {:.2e}  max-abs/rms {:.4f}  row max/rms {:.4f}"
    for what, st, full in log:
        if full:
            tr.write_line(fmt.format(what[:58], st["rows"], st["max_abs"], st["mean_abs"],
                                     st["max_abs_over_rms"], st["max_row_rel"]))
    rest = [st for _, st, full in log if not full]
    if rest:
        tr.write_line(f"other comparisons: {len(rest)}; worst max-abs "
                      f"{max(s['max_abs'] for s in rest):.2e}, mean-abs "
                      f"{max(s['mean_abs'] for s in rest):.2e}, max-abs/rms "
                      f"{max(s['max_abs_over_rms'] for s in rest):.4f}, row max/rms "
                      f"{max(s['max_row_rel'] for s in rest):.4f}")
