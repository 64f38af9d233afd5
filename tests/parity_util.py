"""Shared helpers of the parity tests: tolerance checks and input plumbing.

Tolerance for floating-point outputs (bf16 or fp32 from the GPU against the
oracle's fp64): relative Frobenius error <= 5e-3 and max |error| <= 2e-2 of
the reference's RMS.  Rounding a result to bf16 alone costs about 1.1e-3 in
relative Frobenius error (half an ulp of an 8-bit significand, uniformly
spread), so the bound leaves room for fp32 accumulation order and for the
GPU's bf16 intermediates (XL, G), and still fails on any dropped term, wrong
index or transposed operand.
"""
import numpy as np
import torch

from structured_sparse_pretraining_b200 import inputs as I

REL_FROB = 5e-3
MAX_ABS_OF_RMS = 2e-2


def to_f64(t):
    """GPU/CPU tensor (bf16 / fp32) -> numpy fp64."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = got - ref
    nref = np.linalg.norm(ref)
    rms = nref / np.sqrt(max(ref.size, 1))
    rel = np.linalg.norm(err) / max(nref, 1e-300)
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_FROB, f"{what}: relative Frobenius error {rel:.3e} > {REL_FROB}"
    assert mx <= MAX_ABS_OF_RMS * rms, f"{what}: max |err| {mx:.3e} > {MAX_ABS_OF_RMS} * rms {rms:.3e}"
    return rel, mx / max(rms, 1e-300)


def bits_i16(t):
    """int16 / bf16 CUDA tensor -> numpy uint16 patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def cuda_bf16(a_bits):
    return I.from_bits(a_bits, "cuda")


def cuda_i16(a_bits):
    return torch.from_numpy(np.ascontiguousarray(a_bits).view(np.int16)).to("cuda")
