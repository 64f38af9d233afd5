import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_sessionstart(session):
    """With SLOPE_DEBUG_BOUNDS=1 the session must run on the bounds-checking build."""
    if os.environ.get("SLOPE_DEBUG_BOUNDS", "0") not in ("", "0"):
        from structured_sparse_pretraining_b200 import _lib
        assert _lib.load().slope_debug_bounds() == 1, "SLOPE_DEBUG_BOUNDS=1 but the release library loaded"


def gpu_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if gpu_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Report, per output name, the worst relative Frobenius error and the
    worst plain max|err|/rms(ref) of every parity check in this session, with
    how many checks meet the literal 2e-2 max-abs bound without the rounding
    term (the tests assert the rounding-aware bound; this is the plain one)."""
    try:
        from parity_util import MAX_ABS_OF_RMS, RECORD
    except Exception:
        return
    if not RECORD:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity figures (plain max-abs criterion reported, not asserted)")
    by = {}
    for what, rel, plain in RECORD:
        by.setdefault(what, []).append((rel, plain))
    tr.write_line(f"{'output':8s} {'checks':>6s} {'worst rel-Frob':>15s} {'worst max/rms':>14s} "
                  f"{'plain <= 2e-2':>14s}")
    for what in sorted(by):
        v = by[what]
        ok = sum(1 for _, p in v if p <= MAX_ABS_OF_RMS)
        tr.write_line(f"{what:8s} {len(v):6d} {max(r for r, _ in v):15.3e} {max(p for _, p in v):14.3e} "
                      f"{ok:>9d}/{len(v)}")
