"""The no-allocation masked weight gradient (slope_bwd_dw_masked_noalloc).

It is meant for callers that may not allocate device memory (a fixed memory
budget, or a context where the allocator must not be entered), so its
token-split scratch is a fixed array inside the library.  The call clears the
counters it uses before every launch, so a call never depends on what an
earlier one left behind.

It must give bit-identical results to slope_bwd_dw_masked (same kernel, same
plan; only the split scratch differs), on two calls in a row; match the CPU
oracle within the parity tolerance; and reject layers whose split scratch
exceeds its fixed array.  Collected last so that it also runs after every
other test in the same process.
"""
import os

import pytest
import torch

import oracle
from parity_util import bits_i16, check_close, to_f64
from structured_sparse_pretraining_b200 import _lib, ops
from structured_sparse_pretraining_b200 import inputs as I


def _layer(T, inn, out, seed):
    X = I.normal_bf16((T, inn), 1.0, seed, 0, "X").cuda()
    dY = I.normal_bf16((T, out), 1e-2, seed, 0, "dY").cuda()
    W = I.normal_bf16((out, inn), 0.02, seed, 0, "W").cuda()
    _, meta = ops.prune24(W)
    return X, dY, meta


@pytest.mark.gpu
@pytest.mark.parametrize("T,inn,out", [
    (4096, 512, 512),    # split 8 ways over tokens: uses the fixed scratch
    (9000, 128, 256),    # 128-wide tile, split 8 ways
    (8192, 768, 3072),   # split 2 ways (the GPT-2-small MLP's fc1)
    (2048, 2560, 2560),  # 100 tiles: not split, no scratch at all
])
def test_noalloc_matches_allocating_entry(T, inn, out):
    X, dY, meta = _layer(T, inn, out, 11)
    ref = ops.bwd_dw_masked(dY, X, meta)
    for _ in range(2):  # two calls in a row on the shared scratch
        got = torch.full_like(ref, float("nan"))
        ops.bwd_dw_masked_noalloc(dY, X, meta, got)
        ops.status_sync()
        assert torch.equal(got, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("T,inn,out", [(4096, 512, 512), (9000, 128, 256)])
def test_noalloc_matches_oracle(T, inn, out):
    """Against the CPU oracle's masked gradient (the whole layer), on its own."""
    oracle.threads(len(os.sched_getaffinity(0)))
    X, dY, meta = _layer(T, inn, out, 13)
    got = torch.empty(out, inn // 2, dtype=torch.bfloat16, device="cuda")
    ops.bwd_dw_masked_noalloc(dY, X, meta, got)
    ops.status_sync()
    ref = oracle.bwd_dw_masked(I.bits(dY.cpu()), I.bits(X.cpu()), bits_i16(meta))
    check_close(to_f64(got), ref, "dW")


@pytest.mark.gpu
def test_noalloc_rejects_oversize_split():
    # 1024 -> 3072 over 16384 tokens splits 3 ways: 3 x 3072 x 512 floats > 2^22
    X, dY, meta = _layer(16384, 1024, 3072, 12)
    out = torch.empty(3072, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.SlopeError) as e:
        ops.bwd_dw_masked_noalloc(dY, X, meta, out)
    assert e.value.code == 2
    ops.status_sync()
