"""ctypes loader for libslope.so: the C ABI declared in include/slope.h.

There is no fallback: if the library is missing or cannot be loaded, every
call raises.  bf16 tensors cross the ABI as pointers to their bit patterns.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# SLOPE_DEBUG_BOUNDS=1 selects the debug build (global-memory bounds checks
# in every kernel, reported as SLOPE_ERR_BOUNDS); it is for tests only.
DEBUG_BOUNDS = os.environ.get("SLOPE_DEBUG_BOUNDS", "0") not in ("", "0")
LIB_PATH = os.path.join(HERE, "libslope_debug.so" if DEBUG_BOUNDS else "libslope.so")

# every symbol include/slope.h declares, with (restype, argtypes)
_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
SIGNATURES = {
    "slope_prune24": (_int, [_p, _i64, _i64, _p, _p, _p]),
    "slope_double_prune": (_int, [_p, _p, _i64, _i64, _p, _p, _p]),
    "slope_prune24_double": (_int, [_p, _i64, _i64, _p, _p, _p, _p, _p]),
    "slope_prune_nm": (_int, [_p, _i64, _i64, _int, _int, _p, _p, _p]),
    "slope_adamw_double_prune": (_int, [_p, _p, _p, _p, _p, _i64, _i64, ctypes.c_float, ctypes.c_float,
                                        ctypes.c_float, ctypes.c_float, ctypes.c_float, _i64, _p, _p, _p]),
    "slope_adapter_fwd": (_int, [_p, _p, _i64, _i64, _i64, _p, _p]),
    "slope_fwd": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p]),
    "slope_adapter_bwd": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _p, _p]),
    "slope_fwd_fused": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _p]),
    "slope_bwd_dx_fused": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _p]),
    "slope_bwd_dx": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p]),
    "slope_bwd_dw_masked": (_int, [_p, _p, _p, _i64, _i64, _i64, _p, _p]),
    "slope_bwd_dw_masked_noalloc": (_int, [_p, _p, _p, _i64, _i64, _i64, _p, _p]),
    "slope_bwd_dw_fused": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _p, _p]),
    "slope_selftest_wait_timeout": (_int, [_p]),
    "slope_sparse_plan": (_int, [_i64, _i64, _i64, _int, ctypes.POINTER(_int), ctypes.POINTER(_int)]),
    "slope_sparse_tile_rows": (_int, [_i64, _i64, _i64, _int, ctypes.POINTER(_int)]),
    "slope_fused_launches": (_int, [_i64, _i64, _i64, _i64, _int, ctypes.POINTER(_int)]),
    "slope_status_sync": (_int, [_p]),
    "slope_debug_bounds": (_int, []),
    "slope_device_check": (_int, []),
    "slope_last_error": (ctypes.c_char_p, []),
    "slope_launch_count": (ctypes.c_int64, [_int]),
}

STATUS = {0: "SLOPE_OK", 1: "SLOPE_ERR_ARG", 2: "SLOPE_ERR_SHAPE", 3: "SLOPE_ERR_ALIGN",
          4: "SLOPE_ERR_NONFINITE", 5: "SLOPE_ERR_TIMEOUT", 6: "SLOPE_ERR_CUDA", 7: "SLOPE_ERR_UNSUPPORTED",
          8: "SLOPE_ERR_BOUNDS"}


class SlopeError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


_lib = None


def load():
    """Load libslope.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; "
                               "run structured_sparse_pretraining_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def call(name, *args):
    """Call an entry point; raise SlopeError on a non-zero status."""
    lib = load()
    rc = getattr(lib, name)(*args)
    if rc != 0:
        raise SlopeError(rc, lib.slope_last_error().decode())
    return rc
