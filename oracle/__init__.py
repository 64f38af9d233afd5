"""CPU oracle for the SLoPe 2:4 double-pruned sparse linear layer.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
``cpu_baseline`` / ``--impl reference`` legs of bench.py may import this
package.  The product path (structured_sparse_pretraining_b200) never imports
it, and this package never imports the product.

All arithmetic lives in slope_oracle.c (plain scalar C, fp64 sums); this module
only marshals numpy arrays.  bf16 tensors travel as uint16 bit patterns.

Functions whose results are pinned by tests/test_oracle_pins.py:
  prune24, decompress, double_prune, adapter_fwd, fwd, bwd_dx, adapter_g,
  adapter_dr, adapter_dl, bwd_dw_masked, prune_nm, adamw_compressed, mem_ratio.
Parity unpinned: none of the above; the unbiasedness claim of the pages'
Theorem 2.2 is not computed here (its text is not on the pages).
"""
import ctypes
import os

import numpy as np

from . import build as _build

OK, BAD_SHAPE, NONFINITE = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.oracle_threads.argtypes = [ctypes.c_int]
        L.oracle_threads.restype = ctypes.c_int
        L.oracle_prune24.argtypes = [p, i64, i64, p, p]
        L.oracle_prune24.restype = ctypes.c_int
        L.oracle_decompress.argtypes = [p, p, i64, i64, p]
        L.oracle_decompress.restype = ctypes.c_int
        L.oracle_double_prune.argtypes = [p, p, i64, i64, p, p]
        L.oracle_double_prune.restype = ctypes.c_int
        L.oracle_adapter_fwd.argtypes = [p, p, i64, i64, i64, p, i64, p]
        L.oracle_fwd.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, i64, p]
        L.oracle_bwd_dx.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, i64, p]
        L.oracle_adapter_g.argtypes = [p, p, i64, i64, i64, p, i64, p]
        L.oracle_adapter_dr.argtypes = [p, p, i64, i64, i64, p, i64, p]
        L.oracle_adapter_dl.argtypes = [p, p, i64, i64, i64, p, i64, p]
        L.oracle_bwd_dw_masked.argtypes = [p, p, p, i64, i64, i64, p, i64, p]
        L.oracle_mem_ratio.argtypes = [ctypes.c_int] * 8 + [p]
        L.oracle_prune_nm.argtypes = [p, i64, i64, ctypes.c_int, ctypes.c_int, p, p]
        L.oracle_prune_nm.restype = ctypes.c_int
        f32 = ctypes.c_float
        L.oracle_adamw_compressed.argtypes = [p, p, p, p, i64, f32, f32, f32, f32, f32, i64]
        _lib = L
    return _lib


def threads(n: int = 0) -> int:
    """Set (n > 0) and return the number of OpenMP threads the oracle uses."""
    return lib().oracle_threads(int(n))


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a


def _rows(rows, n):
    if rows is None:
        return None, n
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, len(r)


def _ptr(a):
    return None if a is None else a.ctypes.data


def prune24(W):
    """W: uint16 [rows, K] -> (vals uint16 [rows, K/2], meta uint16 [rows, K/16], status)."""
    W = _u16(W)
    rows, K = W.shape
    vals = np.zeros((rows, K // 2), np.uint16)
    meta = np.zeros((rows, max(K // 16, 0)), np.uint16)
    st = lib().oracle_prune24(_ptr(W), rows, K, _ptr(vals), _ptr(meta))
    return vals, meta, st


def decompress(vals, meta, K):
    vals, meta = _u16(vals), _u16(meta)
    rows = vals.shape[0]
    dense = np.zeros((rows, K), np.uint16)
    st = lib().oracle_decompress(_ptr(vals), _ptr(meta), rows, K, _ptr(dense))
    assert st == OK
    return dense


def double_prune(vals, meta, out, in_):
    vals, meta = _u16(vals), _u16(meta)
    vals_t = np.zeros((in_, out // 2), np.uint16)
    meta_t = np.zeros((in_, out // 16), np.uint16)
    st = lib().oracle_double_prune(_ptr(vals), _ptr(meta), out, in_, _ptr(vals_t), _ptr(meta_t))
    assert st == OK, st
    return vals_t, meta_t


def adapter_fwd(X, L, rows=None):
    X, L = _u16(X), _u16(L)
    T, in_ = X.shape
    r = L.shape[1]
    rr, n = _rows(rows, T)
    XL = np.zeros((n, r), np.float64)
    lib().oracle_adapter_fwd(_ptr(X), _ptr(L), T, in_, r, _ptr(rr), n, _ptr(XL))
    return XL


def fwd(X, vals, meta, XL, R, out, rows=None):
    """XL: float64 [n_rows, r] for the selected rows (or [T, r] when rows is None)."""
    X, vals, meta = _u16(X), _u16(vals), _u16(meta)
    T, in_ = X.shape
    r = 0 if R is None else R.shape[0]
    rr, n = _rows(rows, T)
    XLp = _f64(XL) if r else None
    Rp = _u16(R) if r else None
    Y = np.zeros((n, out), np.float64)
    lib().oracle_fwd(_ptr(X), _ptr(vals), _ptr(meta), _ptr(XLp), _ptr(Rp), T, in_, out, r, _ptr(rr), n, _ptr(Y))
    return Y


def bwd_dx(dY, vals_t, meta_t, G, L, in_, rows=None):
    """G: float64 [n_rows, r] for the selected rows (or [T, r])."""
    dY, vals_t, meta_t = _u16(dY), _u16(vals_t), _u16(meta_t)
    T, out = dY.shape
    r = 0 if L is None else L.shape[1]
    rr, n = _rows(rows, T)
    Gp = _f64(G) if r else None
    Lp = _u16(L) if r else None
    dX = np.zeros((n, in_), np.float64)
    lib().oracle_bwd_dx(_ptr(dY), _ptr(vals_t), _ptr(meta_t), _ptr(Gp), _ptr(Lp), T, in_, out, r, _ptr(rr), n, _ptr(dX))
    return dX


def adapter_g(dY, R, rows=None):
    dY, R = _u16(dY), _u16(R)
    T, out = dY.shape
    r = R.shape[0]
    rr, n = _rows(rows, T)
    G = np.zeros((n, r), np.float64)
    lib().oracle_adapter_g(_ptr(dY), _ptr(R), T, out, r, _ptr(rr), n, _ptr(G))
    return G


def adapter_dr(XL, dY, cols=None):
    """Returns dR restricted to the selected columns, transposed: [n_cols, r]."""
    XL, dY = _f64(XL), _u16(dY)
    T, out = dY.shape
    r = XL.shape[1]
    cc, n = _rows(cols, out)
    dRt = np.zeros((n, r), np.float64)
    lib().oracle_adapter_dr(_ptr(XL), _ptr(dY), T, out, r, _ptr(cc), n, _ptr(dRt))
    return dRt


def adapter_dl(X, G, rows=None):
    X, G = _u16(X), _f64(G)
    T, in_ = X.shape
    r = G.shape[1]
    rr, n = _rows(rows, in_)
    dL = np.zeros((n, r), np.float64)
    lib().oracle_adapter_dl(_ptr(X), _ptr(G), T, in_, r, _ptr(rr), n, _ptr(dL))
    return dL


def bwd_dw_masked(dY, X, meta, rows=None):
    dY, X, meta = _u16(dY), _u16(X), _u16(meta)
    T, out = dY.shape
    in_ = X.shape[1]
    rr, n = _rows(rows, out)
    dW = np.zeros((n, in_ // 2), np.float64)
    lib().oracle_bwd_dw_masked(_ptr(dY), _ptr(X), _ptr(meta), T, in_, out, _ptr(rr), n, _ptr(dW))
    return dW


def prune_nm(W, N, M):
    """Row-wise N:M magnitude pruning: W [rows, K] uint16 bf16 patterns ->
    (vals [rows, K*N/M] uint16, pos [rows, K*N/M] uint8, status)."""
    W = _u16(W)
    rows, K = W.shape
    vals = np.zeros((rows, K // M * N), np.uint16)
    pos = np.zeros((rows, K // M * N), np.uint8)
    st = lib().oracle_prune_nm(_ptr(W), rows, K, int(N), int(M), _ptr(vals), _ptr(pos))
    if st == BAD_SHAPE:
        raise ValueError("prune_nm: bad shape or pattern")
    return vals, pos, st


def adamw_compressed(vals, grad, m, v, lr, b1, b2, eps, wd, step):
    """One AdamW step on the kept values: returns new (vals, m, v); the inputs
    are not modified.  vals/grad: uint16 bf16 patterns, m/v: float32, any
    matching shapes (element by element)."""
    vals = np.array(vals, dtype=np.uint16, order="C", copy=True)
    grad = np.ascontiguousarray(grad, dtype=np.uint16)
    m = np.array(m, dtype=np.float32, order="C", copy=True)
    v = np.array(v, dtype=np.float32, order="C", copy=True)
    assert vals.shape == grad.shape == m.shape == v.shape
    lib().oracle_adamw_compressed(_ptr(vals), _ptr(grad), _ptr(m), _ptr(v), vals.size, float(lr), float(b1),
                                  float(b2), float(eps), float(wd), int(step))
    return vals, m, v


def mem_ratio(n_keep=2, m_group=4, b_val=16, b_idx=3, b_mask=8, b_grad=16, b_state=32, n_states=2):
    """(inference ratio, training ratio) per four weights."""
    out = np.zeros(2, np.float64)
    lib().oracle_mem_ratio(n_keep, m_group, b_val, b_idx, b_mask, b_grad, b_state, n_states, _ptr(out))
    return float(out[0]), float(out[1])


def bf16_values(bits):
    """Exact float64 values of bf16 bit patterns (a decode, not method arithmetic)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def layer_step(X, W, L, R, dY):
    """The whole layer on the CPU, fp64 throughout (XL and G are not rounded):
    prune24 -> double_prune -> adapter_fwd -> fwd -> adapter_bwd -> bwd_dx ->
    bwd_dw_masked.  Returns a dict of every intermediate and output."""
    T, in_ = X.shape
    out = W.shape[0]
    vals, meta, st = prune24(W)
    vals_t, meta_t = double_prune(vals, meta, out, in_)
    r = 0 if L is None else L.shape[1]
    XL = adapter_fwd(X, L) if r else None
    Y = fwd(X, vals, meta, XL, R, out)
    G = adapter_g(dY, R) if r else None
    dR = adapter_dr(XL, dY).T.copy() if r else None
    dL = adapter_dl(X, G) if r else None
    dX = bwd_dx(dY, vals_t, meta_t, G, L, in_)
    dW = bwd_dw_masked(dY, X, meta)
    return dict(status=st, vals=vals, meta=meta, vals_t=vals_t, meta_t=meta_t, XL=XL, Y=Y,
                G=G, dR=dR, dL=dL, dX=dX, dW=dW)
