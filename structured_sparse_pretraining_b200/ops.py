"""Torch-facing wrappers of the C ABI: argument marshalling only.

Every op checks dtype, device and contiguity, allocates its outputs with torch
when none are given, and passes raw pointers plus the current CUDA stream to
libslope.so.  No arithmetic of the layer happens here.

bf16 tensors are torch.bfloat16; the 16-bit position-code words ("meta") are
torch.int16 tensors holding the uint16 patterns.
"""
import ctypes

import torch

from . import _lib


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, dtype, name, shape=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _empty(shape, dtype, like):
    return torch.empty(shape, dtype=dtype, device=like.device)


def prune24(W, vals=None, meta=None):
    """Row-wise 2:4 magnitude pruning: W [rows, K] -> (vals [rows, K/2], meta [rows, K/16])."""
    _need(W, torch.bfloat16, "W")
    rows, K = W.shape
    vals = _empty((rows, K // 2), torch.bfloat16, W) if vals is None else _need(vals, torch.bfloat16, "vals", (rows, K // 2))
    meta = _empty((rows, K // 16), torch.int16, W) if meta is None else _need(meta, torch.int16, "meta", (rows, K // 16))
    _lib.call("slope_prune24", _ptr(W), rows, K, _ptr(vals), _ptr(meta), _stream())
    return vals, meta


def prune_nm(W, N, M, vals=None, pos=None):
    """Row-wise N:M magnitude pruning: W [rows, K] -> (vals [rows, K*N/M] bf16,
    pos [rows, K*N/M] uint8 positions within each group)."""
    _need(W, torch.bfloat16, "W")
    rows, K = W.shape
    shape = (rows, K // M * N) if M > 0 and K % M == 0 else (rows, 0)
    vals = _empty(shape, torch.bfloat16, W) if vals is None else _need(vals, torch.bfloat16, "vals", shape)
    pos = _empty(shape, torch.uint8, W) if pos is None else _need(pos, torch.uint8, "pos", shape)
    _lib.call("slope_prune_nm", _ptr(W), rows, K, int(N), int(M), _ptr(vals), _ptr(pos), _stream())
    return vals, pos


def double_prune(vals, meta, out_features, in_features, vals_t=None, meta_t=None):
    """W^R (compressed [out, in]) -> (W^{R,C})^T compressed: (vals_t [in, out/2], meta_t [in, out/16])."""
    _need(vals, torch.bfloat16, "vals", (out_features, in_features // 2))
    _need(meta, torch.int16, "meta", (out_features, in_features // 16))
    if vals_t is None:
        vals_t = _empty((in_features, out_features // 2), torch.bfloat16, vals)
    if meta_t is None:
        meta_t = _empty((in_features, out_features // 16), torch.int16, vals)
    _need(vals_t, torch.bfloat16, "vals_t", (in_features, out_features // 2))
    _need(meta_t, torch.int16, "meta_t", (in_features, out_features // 16))
    _lib.call("slope_double_prune", _ptr(vals), _ptr(meta), out_features, in_features, _ptr(vals_t), _ptr(meta_t),
              _stream())
    return vals_t, meta_t


def prune24_double(W, vals=None, meta=None, vals_t=None, meta_t=None):
    """Both prunings in one launch: W [out, in] bf16 -> (vals, meta, vals_t, meta_t),
    equal to prune24 followed by double_prune."""
    _need(W, torch.bfloat16, "W")
    out, in_ = W.shape
    vals = _empty((out, in_ // 2), torch.bfloat16, W) if vals is None else _need(vals, torch.bfloat16, "vals", (out, in_ // 2))
    meta = _empty((out, in_ // 16), torch.int16, W) if meta is None else _need(meta, torch.int16, "meta", (out, in_ // 16))
    vals_t = (_empty((in_, out // 2), torch.bfloat16, W) if vals_t is None
              else _need(vals_t, torch.bfloat16, "vals_t", (in_, out // 2)))
    meta_t = (_empty((in_, out // 16), torch.int16, W) if meta_t is None
              else _need(meta_t, torch.int16, "meta_t", (in_, out // 16)))
    _lib.call("slope_prune24_double", _ptr(W), out, in_, _ptr(vals), _ptr(meta), _ptr(vals_t), _ptr(meta_t),
              _stream())
    return vals, meta, vals_t, meta_t


def adamw_double_prune(vals, meta, dW_vals, m, v, out_features, in_features, lr, beta1, beta2, eps,
                       weight_decay, step, vals_t=None, meta_t=None):
    """One AdamW step on the kept values (vals, m, v updated in place) fused
    with the second pruning of the updated W^R: returns (vals_t, meta_t)."""
    _need(vals, torch.bfloat16, "vals", (out_features, in_features // 2))
    _need(meta, torch.int16, "meta", (out_features, in_features // 16))
    _need(dW_vals, torch.bfloat16, "dW_vals", (out_features, in_features // 2))
    _need(m, torch.float32, "m", (out_features, in_features // 2))
    _need(v, torch.float32, "v", (out_features, in_features // 2))
    if vals_t is None:
        vals_t = _empty((in_features, out_features // 2), torch.bfloat16, vals)
    if meta_t is None:
        meta_t = _empty((in_features, out_features // 16), torch.int16, vals)
    _need(vals_t, torch.bfloat16, "vals_t", (in_features, out_features // 2))
    _need(meta_t, torch.int16, "meta_t", (in_features, out_features // 16))
    _lib.call("slope_adamw_double_prune", _ptr(vals), _ptr(meta), _ptr(dW_vals), _ptr(m), _ptr(v), out_features,
              in_features, float(lr), float(beta1), float(beta2), float(eps), float(weight_decay), int(step),
              _ptr(vals_t), _ptr(meta_t), _stream())
    return vals_t, meta_t


def adapter_fwd(X, L, XL=None):
    """XL = X . L  (X [T, in], L [in, r])."""
    _need(X, torch.bfloat16, "X")
    T, in_ = X.shape
    _need(L, torch.bfloat16, "L")
    r = L.shape[1]
    XL = _empty((T, r), torch.bfloat16, X) if XL is None else _need(XL, torch.bfloat16, "XL", (T, r))
    _lib.call("slope_adapter_fwd", _ptr(X), _ptr(L), T, in_, r, _ptr(XL), _stream())
    return XL


def fwd(X, vals, meta, XL, R, out_features, Y=None):
    """Y = X . (W^R)^T + XL . R  (XL, R may be None: no adapter)."""
    _need(X, torch.bfloat16, "X")
    T, in_ = X.shape
    _need(vals, torch.bfloat16, "vals", (out_features, in_ // 2))
    _need(meta, torch.int16, "meta", (out_features, in_ // 16))
    r = 0
    if R is not None:
        r = R.shape[0]
        _need(R, torch.bfloat16, "R", (r, out_features))
        _need(XL, torch.bfloat16, "XL", (T, r))
    Y = _empty((T, out_features), torch.bfloat16, X) if Y is None else _need(Y, torch.bfloat16, "Y", (T, out_features))
    _lib.call("slope_fwd", _ptr(X), _ptr(vals), _ptr(meta), _ptr(XL), _ptr(R), T, in_, out_features, r, _ptr(Y),
              _stream())
    return Y


def fwd_fused(X, vals, meta, L, R, out_features, XL=None, Y=None):
    """(XL, Y): XL = X . L and Y = X . (W^R)^T + XL . R in one launch where
    the shapes allow (L, R None: no adapter, XL is None)."""
    _need(X, torch.bfloat16, "X")
    T, in_ = X.shape
    _need(vals, torch.bfloat16, "vals", (out_features, in_ // 2))
    _need(meta, torch.int16, "meta", (out_features, in_ // 16))
    r = 0
    if R is not None:
        r = R.shape[0]
        _need(R, torch.bfloat16, "R", (r, out_features))
        _need(L, torch.bfloat16, "L", (in_, r))
        XL = _empty((T, r), torch.bfloat16, X) if XL is None else _need(XL, torch.bfloat16, "XL", (T, r))
    Y = _empty((T, out_features), torch.bfloat16, X) if Y is None else _need(Y, torch.bfloat16, "Y", (T, out_features))
    _lib.call("slope_fwd_fused", _ptr(X), _ptr(vals), _ptr(meta), _ptr(L), _ptr(R), T, in_, out_features, r,
              _ptr(XL) if r else None, _ptr(Y), _stream())
    return (XL if r else None), Y


def bwd_dx_fused(dY, vals_t, meta_t, R, L, in_features, G=None, dX=None):
    """(G, dX): G = dY . R^T and dX = dY . W^{R,C} + G . L^T in one launch
    where the shapes allow (R, L None: no adapter, G is None)."""
    _need(dY, torch.bfloat16, "dY")
    T, out = dY.shape
    _need(vals_t, torch.bfloat16, "vals_t", (in_features, out // 2))
    _need(meta_t, torch.int16, "meta_t", (in_features, out // 16))
    r = 0
    if L is not None:
        r = L.shape[1]
        _need(L, torch.bfloat16, "L", (in_features, r))
        _need(R, torch.bfloat16, "R", (r, out))
        G = _empty((T, r), torch.bfloat16, dY) if G is None else _need(G, torch.bfloat16, "G", (T, r))
    dX = _empty((T, in_features), torch.bfloat16, dY) if dX is None else _need(dX, torch.bfloat16, "dX", (T, in_features))
    _lib.call("slope_bwd_dx_fused", _ptr(dY), _ptr(vals_t), _ptr(meta_t), _ptr(R), _ptr(L), T, in_features, out, r,
              _ptr(G) if r else None, _ptr(dX), _stream())
    return (G if r else None), dX


def adapter_bwd(X, dY, XL, R, dL=None, dR=None, G=None):
    """(dL [in, r] fp32, dR [r, out] fp32, G [T, r] bf16) for Y += (X L) R."""
    _need(X, torch.bfloat16, "X")
    _need(dY, torch.bfloat16, "dY")
    T, in_ = X.shape
    out = dY.shape[1]
    r = R.shape[0]
    _need(XL, torch.bfloat16, "XL", (T, r))
    _need(R, torch.bfloat16, "R", (r, out))
    dL = _empty((in_, r), torch.float32, X) if dL is None else _need(dL, torch.float32, "dL", (in_, r))
    dR = _empty((r, out), torch.float32, X) if dR is None else _need(dR, torch.float32, "dR", (r, out))
    G = _empty((T, r), torch.bfloat16, X) if G is None else _need(G, torch.bfloat16, "G", (T, r))
    _lib.call("slope_adapter_bwd", _ptr(X), _ptr(dY), _ptr(XL), _ptr(R), T, in_, out, r, _ptr(dL), _ptr(dR),
              _ptr(G), _stream())
    return dL, dR, G


def bwd_dx(dY, vals_t, meta_t, G, L, in_features, dX=None):
    """dX = dY . W^{R,C} + G . L^T."""
    _need(dY, torch.bfloat16, "dY")
    T, out = dY.shape
    _need(vals_t, torch.bfloat16, "vals_t", (in_features, out // 2))
    _need(meta_t, torch.int16, "meta_t", (in_features, out // 16))
    r = 0
    if L is not None:
        r = L.shape[1]
        _need(L, torch.bfloat16, "L", (in_features, r))
        _need(G, torch.bfloat16, "G", (T, r))
    dX = _empty((T, in_features), torch.bfloat16, dY) if dX is None else _need(dX, torch.bfloat16, "dX", (T, in_features))
    _lib.call("slope_bwd_dx", _ptr(dY), _ptr(vals_t), _ptr(meta_t), _ptr(G), _ptr(L), T, in_features, out, r,
              _ptr(dX), _stream())
    return dX


def bwd_dw_masked(dY, X, meta, dW_vals=None):
    """dW restricted to the static mask, compressed like vals: [out, in/2]."""
    _need(dY, torch.bfloat16, "dY")
    _need(X, torch.bfloat16, "X")
    T, out = dY.shape
    in_ = X.shape[1]
    _need(meta, torch.int16, "meta", (out, in_ // 16))
    if dW_vals is None:
        dW_vals = _empty((out, in_ // 2), torch.bfloat16, X)
    _need(dW_vals, torch.bfloat16, "dW_vals", (out, in_ // 2))
    _lib.call("slope_bwd_dw_masked", _ptr(dY), _ptr(X), _ptr(meta), T, in_, out, _ptr(dW_vals), _stream())
    return dW_vals


def bwd_dw_fused(dY, X, meta, XL, G, dW_vals=None, dL=None, dR=None):
    """(dW_vals, dL, dR): the masked weight gradient and the adapter gradients
    dR = XL^T . dY, dL = X^T . G in one launch (XL, G None: no adapter)."""
    _need(dY, torch.bfloat16, "dY")
    _need(X, torch.bfloat16, "X")
    T, out = dY.shape
    in_ = X.shape[1]
    _need(meta, torch.int16, "meta", (out, in_ // 16))
    dW_vals = _empty((out, in_ // 2), torch.bfloat16, X) if dW_vals is None else _need(dW_vals, torch.bfloat16, "dW_vals",
                                                                                         (out, in_ // 2))
    r = 0
    if XL is not None:
        r = XL.shape[1]
        _need(XL, torch.bfloat16, "XL", (T, r))
        _need(G, torch.bfloat16, "G", (T, r))
        dL = _empty((in_, r), torch.float32, X) if dL is None else _need(dL, torch.float32, "dL", (in_, r))
        dR = _empty((r, out), torch.float32, X) if dR is None else _need(dR, torch.float32, "dR", (r, out))
    _lib.call("slope_bwd_dw_fused", _ptr(dY), _ptr(X), _ptr(meta), _ptr(XL), _ptr(G), T, in_, out, r, _ptr(dW_vals),
              _ptr(dL) if r else None, _ptr(dR) if r else None, _stream())
    return dW_vals, (dL if r else None), (dR if r else None)


def bwd_dw_masked_noalloc(dY, X, meta, dW_vals):
    """bwd_dw_masked into a caller-provided dW_vals; the library allocates
    nothing (token-split scratch from a fixed device array; see slope.h)."""
    _need(dY, torch.bfloat16, "dY")
    _need(X, torch.bfloat16, "X")
    T, out = dY.shape
    in_ = X.shape[1]
    _need(meta, torch.int16, "meta", (out, in_ // 16))
    _need(dW_vals, torch.bfloat16, "dW_vals", (out, in_ // 2))
    _lib.call("slope_bwd_dw_masked_noalloc", _ptr(dY), _ptr(X), _ptr(meta), T, in_, out, _ptr(dW_vals), _stream())
    return dW_vals


def sparse_plan(M, T, K, sms=148):
    """(BN, splits) the sparse products use for an M x K operand and T tokens
    on a device with `sms` SMs (host-only query, no GPU needed)."""
    bn, splits = ctypes.c_int(0), ctypes.c_int(0)
    _lib.call("slope_sparse_plan", M, T, K, sms, ctypes.byref(bn), ctypes.byref(splits))
    return bn.value, splits.value


def sparse_tile_rows(M, T, K, sms=148):
    """Output-tile height (256 or 512 rows) the sparse products use for an
    M x K operand and T tokens (host-only query, no GPU needed)."""
    rows = ctypes.c_int(0)
    _lib.call("slope_sparse_tile_rows", M, T, K, sms, ctypes.byref(rows))
    return rows.value


def fused_launches(M, T, K, r, sms=148):
    """Launches (1 or 2) of fwd_fused (M = out, K = in) or bwd_dx_fused
    (M = in, K = out) for these sizes (host-only query, no GPU needed)."""
    n = ctypes.c_int(0)
    _lib.call("slope_fused_launches", M, T, K, r, sms, ctypes.byref(n))
    return n.value


def status_sync():
    """Wait for the current stream and raise if a kernel flagged an error."""
    _lib.call("slope_status_sync", _stream())


def selftest_wait_timeout():
    """Launch the failure-path self-test: a bounded wait that runs out; the next
    status_sync raises SlopeError with SLOPE_ERR_TIMEOUT (5)."""
    _lib.call("slope_selftest_wait_timeout", _stream())


def device_check():
    _lib.call("slope_device_check")


def launch_count(reset=False):
    return int(_lib.load().slope_launch_count(1 if reset else 0))
