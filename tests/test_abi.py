"""Host-only checks of the C ABI (no GPU needed, no kernel launched):
the library loads, exports every symbol include/slope.h declares, and its
argument validation rejects bad calls before touching the device."""
import ctypes
import os
import re

import pytest

from structured_sparse_pretraining_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "slope.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(slope_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path():
    syms = declared_symbols()
    for s in ["slope_prune24", "slope_double_prune", "slope_fwd", "slope_bwd_dx", "slope_bwd_dw_masked",
              "slope_adapter_fwd", "slope_adapter_bwd"]:
        assert s in syms


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for s in declared_symbols():
        assert hasattr(lib, s), f"{s} declared in slope.h but not exported"
    assert set(declared_symbols()) == set(_lib.SIGNATURES), "binding and header disagree"


def test_null_and_alignment_rejected_on_host():
    lib = _lib.load()
    buf = (ctypes.c_uint8 * 4096)()
    base = (ctypes.addressof(buf) + 15) & ~15
    # NULL input -> SLOPE_ERR_ARG, decided before any CUDA call
    assert lib.slope_prune24(None, 64, 64, base, base, None) == 1
    assert b"W is NULL" in lib.slope_last_error()
    # misaligned pointer -> SLOPE_ERR_ALIGN
    assert lib.slope_prune24(base + 2, 64, 64, base, base, None) == 3
    assert lib.slope_double_prune(base, base + 8, 64, 64, base, base, None) == 3


@pytest.mark.parametrize("K,code", [(96, 2), (0, 1), (-64, 1)])
def test_shape_rules_on_host(K, code):
    lib = _lib.load()
    buf = (ctypes.c_uint8 * 4096)()
    base = (ctypes.addressof(buf) + 15) & ~15
    assert lib.slope_prune24(base, 64, K, base, base, None) == code


@pytest.mark.parametrize("r,code", [(12, 2), (264, 2), (-8, 1)])
def test_rank_rules_on_host(r, code):
    lib = _lib.load()
    buf = (ctypes.c_uint8 * 4096)()
    b = (ctypes.addressof(buf) + 15) & ~15
    assert lib.slope_fwd(b, b, b, b, b, 16, 64, 64, r, b, None) == code
    assert lib.slope_bwd_dx(b, b, b, b, b, 16, 64, 64, r, b, None) == code


def test_missing_adapter_operands_rejected():
    lib = _lib.load()
    buf = (ctypes.c_uint8 * 4096)()
    b = (ctypes.addressof(buf) + 15) & ~15
    assert lib.slope_fwd(b, b, b, None, b, 16, 64, 64, 8, b, None) == 1
    assert lib.slope_adapter_fwd(b, b, 16, 64, 0, b, None) == 1


def test_launch_counter_resets():
    lib = _lib.load()
    lib.slope_launch_count(1)
    assert lib.slope_launch_count(0) == 0
