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


def test_debug_build_exports_the_same_symbols_and_reports_its_checks():
    """libslope_debug.so (-DSLOPE_DEBUG_BOUNDS) is the same ABI with bounds
    checks in the kernels; slope_debug_bounds() tells the builds apart."""
    dbg = ctypes.CDLL(os.path.join(_lib.HERE, "libslope_debug.so"))
    for s in declared_symbols():
        assert hasattr(dbg, s), f"{s} declared in slope.h but not exported by the debug build"
    assert dbg.slope_debug_bounds() == 1
    rel = ctypes.CDLL(os.path.join(_lib.HERE, "libslope.so"))
    assert rel.slope_debug_bounds() == 0
    assert _lib.load().slope_debug_bounds() == (1 if _lib.DEBUG_BOUNDS else 0)


def test_fused_launch_choice_on_host():
    """The planner fuses the rank product where its 512 x 224 tiles fill the
    SM pairs, and keeps two launches for a few tokens (host-only query)."""
    from structured_sparse_pretraining_b200 import ops
    assert ops.fused_launches(27648, 8192, 9216, 96) == 1   # OPT-66B fc1 forward, training batch
    assert ops.fused_launches(27648, 1, 9216, 96) == 2      # the same layer at one token
    assert ops.fused_launches(9216, 16, 36864, 96) == 2     # long reduction, few output tiles
    assert ops.fused_launches(3072, 8192, 768, 16) == 1     # GPT-2-small fc1
    assert ops.fused_launches(1024, 64, 1024, 192) == 2     # rank above 128
    assert ops.fused_launches(1024, 64, 1024, 0) == 1       # no adapter: one launch
    lib = _lib.load()
    assert lib.slope_fused_launches(64, 64, 64, 8, 148, None) == 1


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


def test_adamw_arguments_rejected_on_host():
    lib = _lib.load()
    buf = (ctypes.c_uint8 * 4096)()
    b = (ctypes.addressof(buf) + 15) & ~15
    ok = dict(lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, step=1)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.slope_adamw_double_prune(b, b, b, b, b, 64, 64, a["lr"], a["b1"], a["b2"], a["eps"], a["wd"],
                                            a["step"], b, b, None)
    assert call(step=0) == 1
    assert call(b1=1.0) == 1
    assert call(eps=0.0) == 1
    assert call(lr=-1.0) == 1
    assert lib.slope_adamw_double_prune(b, b, None, b, b, 64, 64, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, b, b, None) == 1
    assert lib.slope_adamw_double_prune(b, b, b, b, b, 64, 100, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1, b, b, None) == 2


def test_prune_nm_rules_on_host():
    lib = _lib.load()
    buf = (ctypes.c_uint8 * 4096)()
    b = (ctypes.addressof(buf) + 15) & ~15
    assert lib.slope_prune_nm(b, 4, 64, 2, 6, b, b, None) == 2     # M not 4, 8, 16
    assert lib.slope_prune_nm(b, 4, 64, 0, 4, b, b, None) == 2     # N < 1
    assert lib.slope_prune_nm(b, 4, 64, 4, 4, b, b, None) == 2     # N == M
    assert lib.slope_prune_nm(b, 4, 72, 2, 16, b, b, None) == 2    # K % M
    assert lib.slope_prune_nm(None, 4, 64, 2, 4, b, b, None) == 1  # NULL


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


# ------------------------------------------------------------------ launch plan of the sparse products
BNS = {240, 224, 192, 176, 128, 64, 32, 16}
# (out, in) of the four largest-workload layers (QKV, out-proj, FFN up, FFN down)
C5_LAYERS = [(27648, 9216), (9216, 9216), (36864, 9216), (9216, 36864)]


def plan(M, T, K, sms=148):
    from structured_sparse_pretraining_b200 import ops
    return ops.sparse_plan(M, T, K, sms)


@pytest.mark.parametrize("M,T,K", [(512, 256, 512), (3072, 8192, 768), (768, 8192, 3072), (27648, 1, 9216),
                                   (9216, 16, 36864), (64, 1, 64), (36864, 128, 9216), (1024, 300, 192),
                                   (9216, 2048, 9216), (256, 5, 65536)])
def test_sparse_plan_is_well_formed(M, T, K):
    bn, s = plan(M, T, K)
    assert bn in BNS
    kt = (K + 127) // 128
    kps = -(-kt // s)
    assert 1 <= s <= 8 and -(-kt // kps) == s, "every split holds at least one k-tile"
    if s > 1:
        assert bn < 176 and kps >= 4


@pytest.mark.parametrize("cfg", ["C2", "C3", "C4", "C5"])
def test_training_workloads_use_wide_unsplit_tiles(cfg):
    """At the training token counts every layer has several waves of wide
    tiles: no K split, BN >= 176 (the tiles the sparse-kernel timings cover)."""
    from structured_sparse_pretraining_b200 import inputs as I
    w = I.WORKLOADS[cfg]
    for lay in w.layers:
        for M, K in ((lay.out_features, lay.in_features), (lay.in_features, lay.out_features)):  # fwd, bwd_dx
            bn, s = plan(M, w.tokens, K)
            assert s == 1 and bn >= 176, (cfg, M, K, bn, s)


@pytest.mark.parametrize("T", [1, 16])
def test_weight_streaming_fills_the_sm_pairs(T):
    """At a handful of tokens one 16-wide token tile covers T, and the K split
    gives every layer enough work units to keep >= 90% of the 74 SM pairs busy
    over the waves it runs."""
    for out, inn in C5_LAYERS:
        bn, s = plan(out, T, inn)
        assert bn == 16
        units = -(-out // 256) * s
        waves = -(-units // 74)
        assert units / (waves * 74) >= 0.9, (out, inn, s)


@pytest.mark.parametrize("cfg", ["C2", "C3", "C4", "C5"])
def test_training_workloads_fuse_the_rank_products(cfg):
    """At the training token counts every fused call of the bench step runs
    as one launch (the wide tiles fill the SM pairs)."""
    from structured_sparse_pretraining_b200 import inputs as I
    from structured_sparse_pretraining_b200 import ops
    w = I.WORKLOADS[cfg]
    for lay in w.layers:
        for M, K in ((lay.out_features, lay.in_features), (lay.in_features, lay.out_features)):
            assert ops.fused_launches(M, w.tokens, K, w.rank_stored) == 1, \
                (cfg, M, K)


def test_fused_launch_choice_follows_the_planner():
    """Wherever the planner itself takes the 512-row tiles for the sparse
    product, the fused call takes one launch (its cost is then below the
    best pair tiling's, let alone that plus a launch)."""
    from structured_sparse_pretraining_b200 import ops
    for M in (768, 3072, 9216, 27648):
        for K in (1024, 4096, 9216):
            for T in (1, 16, 128, 512, 2048, 8192):
                if ops.sparse_tile_rows(M, T, K) == 512:
                    assert ops.fused_launches(M, T, K, 64) == 1, (M, T, K)


def test_sparse_plan_rejects_bad_arguments():
    lib = _lib.load()
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    assert lib.slope_sparse_plan(0, 1, 64, 148, ctypes.byref(a), ctypes.byref(b)) == 1
    assert lib.slope_sparse_plan(64, 1, 64, 0, ctypes.byref(a), ctypes.byref(b)) == 1
    assert lib.slope_sparse_plan(64, 1, 64, 148, None, ctypes.byref(b)) == 1


def test_every_declared_call_is_documented():
    """Each entry point in slope.h is preceded by its own comment block (what
    it computes, arguments, errors)."""
    text = open(HEADER).read()
    for name in declared_symbols():
        m = re.search(r"^[A-Za-z_][A-Za-z0-9_ ]*\**\s*" + name + r"\(", text, flags=re.M)
        assert m, f"no declaration line for {name}"
        lines = text[:m.start()].rstrip().split("\n")
        while lines and lines[-1].startswith("#define"):  # constants that belong to the call
            lines.pop()
        assert "\n".join(lines).rstrip().endswith("*/"), f"{name} has no comment block right above it"
