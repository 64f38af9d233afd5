"""Shared helpers of the parity tests: tolerance checks and input plumbing.

Tolerance for floating-point outputs (bf16 or fp32 from the GPU against the
oracle's fp64): relative Frobenius error <= 5e-3 and, element by element,
|error| <= 2e-2 of the reference's RMS plus the rounding of that element to
the output's own format (2^-8 |ref| for a bf16 output, whose 8-bit
significand puts half an ulp at most 2^-8 of the value; 0 for fp32 outputs).
The max-abs bound is meant for the arithmetic; without the rounding term it
cannot hold for any bf16 output whose values are heavy-tailed (dW at one
token is an outer product: its largest values reach ~13 RMS, and rounding
them alone moves them by up to 0.05 RMS).  Rounding a result to bf16 alone
costs about 1.1e-3 in relative Frobenius error (half an ulp of an 8-bit
significand, uniformly spread), so the bounds leave room for fp32
accumulation order and for the GPU's bf16 intermediates (XL, G), and still
fail on any dropped term, wrong index or transposed operand.
"""
import numpy as np
import torch

from structured_sparse_pretraining_b200 import inputs as I

REL_FROB = 5e-3
MAX_ABS_OF_RMS = 2e-2

# Every check's figures, for the end-of-session report (conftest): the
# relative Frobenius error and the plain max |err| / rms(ref) ratio, which is
# also judged against the literal 2e-2 bound without the rounding term.
RECORD = []


def to_f64(t):
    """GPU/CPU tensor (bf16 / fp32) -> numpy fp64."""
    return t.detach().float().cpu().numpy().astype(np.float64)


FP32_OUTPUTS = ("dL", "dR")  # the adapter gradients stay fp32; every other float output is bf16


def check_close(got, ref, what, out_rounding=None):
    """`out_rounding`: the relative rounding of the output format (2^-8 for
    bf16 outputs, 0 for fp32 ones; by default chosen from `what`)."""
    if out_rounding is None:
        out_rounding = 0.0 if what in FP32_OUTPUTS else 2.0 ** -8
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = got - ref
    nref = np.linalg.norm(ref)
    rms = nref / np.sqrt(max(ref.size, 1))
    rel = np.linalg.norm(err) / max(nref, 1e-300)
    mx = np.abs(err).max() if err.size else 0.0
    RECORD.append((what, float(rel), float(mx / max(rms, 1e-300))))
    assert rel <= REL_FROB, f"{what}: relative Frobenius error {rel:.3e} > {REL_FROB}"
    excess = np.abs(err) - (MAX_ABS_OF_RMS * rms + out_rounding * np.abs(ref))
    if excess.size and excess.max() > 0:
        i = np.unravel_index(np.argmax(excess), err.shape)
        raise AssertionError(f"{what}: |err| {abs(err[i]):.3e} at {i} (ref {ref[i]:.3e}) > {MAX_ABS_OF_RMS} * rms "
                             f"{rms:.3e} + {out_rounding:.3g} * |ref|")
    return rel, mx / max(rms, 1e-300)


def bits_i16(t):
    """int16 / bf16 CUDA tensor -> numpy uint16 patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def cuda_bf16(a_bits):
    return I.from_bits(a_bits, "cuda")


def cuda_i16(a_bits):
    return torch.from_numpy(np.ascontiguousarray(a_bits).view(np.int16)).to("cuda")


# ------------------------------------------------------------------ canary guard bands
# Out-of-bounds-write evidence without compute-sanitizer: an output tensor is
# a view into a larger buffer whose GUARD elements before and after it hold a
# NaN bit pattern; after the kernels ran, the bands must be unchanged bit for
# bit.  A store past the end of a row block, a tile or the whole output (or
# before its start) lands in a band.
GUARD = 8192
_CANARY = {torch.bfloat16: 0x7FA5, torch.int16: 0x7FA5, torch.float32: 0x7FA5A5A5, torch.uint8: 0xA5}
_GUARDED = []


def guarded_empty(shape, dtype, device="cuda"):
    """An uninitialised-looking output of `shape` (filled with the canary too)
    with canary bands before and after it; check_guards() verifies every band
    handed out since the last check."""
    n = 1
    for d in shape:
        n *= d
    bits = {torch.bfloat16: torch.int16, torch.int16: torch.int16, torch.float32: torch.int32,
            torch.uint8: torch.uint8}[dtype]
    pat = _CANARY[dtype]
    if bits == torch.int16 and pat >= 0x8000:
        pat -= 0x10000
    if bits == torch.int32 and pat >= 0x80000000:
        pat -= 0x100000000
    # 16-byte alignment of the view: the band is a multiple of 16 bytes long
    buf = torch.full((n + 2 * GUARD,), pat, dtype=bits, device=device)
    view = buf[GUARD:GUARD + n].view(dtype).view(*shape)
    _GUARDED.append((buf, n, pat))
    return view


def check_guards():
    """Assert that no band handed out since the last call was written."""
    try:
        for buf, n, pat in _GUARDED:
            head = buf[:GUARD]
            tail = buf[GUARD + n:]
            bad_h = int((head != pat).sum().item())
            bad_t = int((tail != pat).sum().item())
            assert bad_h == 0 and bad_t == 0, (f"write outside an output of {n} elements: {bad_h} changed before it, "
                                               f"{bad_t} after it")
    finally:
        _GUARDED.clear()
