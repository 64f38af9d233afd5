"""Build libslope.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a,
and its debug build libslope_debug.so (-DSLOPE_DEBUG_BOUNDS: bounds checks on
every plain global-memory access of the kernels, for tests)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "slope_api.cu")
LIB = os.path.join(HERE, "libslope.so")
LIB_DEBUG = os.path.join(HERE, "libslope_debug.so")
DEPS = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))] + [
    os.path.join(ROOT, "include", "slope.h")]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v"]


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _build_one(lib: str, extra, force: bool, verbose: bool) -> str:
    if not force and os.path.exists(lib):
        newest = max(os.path.getmtime(d) for d in DEPS)
        if os.path.getmtime(lib) >= newest:
            return lib
    cmd = [nvcc()] + NVCC_FLAGS + list(extra) + ["-o", lib, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(res.stderr)
    return lib


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Build libslope.so (and, with debug=True, libslope_debug.so beside it,
    in parallel); returns the release library's path."""
    if not debug:
        return _build_one(LIB, [], force, verbose)
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(2) as ex:
        rel = ex.submit(_build_one, LIB, [], force, verbose)
        dbg = ex.submit(_build_one, LIB_DEBUG, ["-DSLOPE_DEBUG_BOUNDS"], force, False)
        dbg.result()
        return rel.result()


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
