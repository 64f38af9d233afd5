"""The no-allocation masked weight gradient (slope_bwd_dw_masked_noalloc).

It must give bit-identical results to slope_bwd_dw_masked (same kernel, same
plan; only the split scratch differs), on two calls in a row (its counters
must be left at zero by the first), and reject layers whose split scratch
exceeds its fixed array.  Collected last so that it also runs after every
other test in the same process.
"""
import pytest
import torch

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
    for _ in range(2):  # the second call starts from the counters the first left
        got = torch.full_like(ref, float("nan"))
        ops.bwd_dw_masked_noalloc(dY, X, meta, got)
        ops.status_sync()
        assert torch.equal(got, ref)


@pytest.mark.gpu
def test_noalloc_rejects_oversize_split():
    # 1024 -> 3072 over 16384 tokens splits 3 ways: 3 x 3072 x 512 floats > 2^22
    X, dY, meta = _layer(16384, 1024, 3072, 12)
    out = torch.empty(3072, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.SlopeError) as e:
        ops.bwd_dw_masked_noalloc(dY, X, meta, out)
    assert e.value.code == 2
    ops.status_sync()
