"""The data-parallel path on two and three CPU ranks (gloo): each rank takes
its share of the tokens, computes the replicated parameters' gradients (the
oracle stands in for the GPU kernels here) in the formats the kernels write
them (masked dW bf16, dL and dR fp32), and the library's all-reduce sums them
in one fp32 bucket, exactly as bench.py does with NCCL.  The sums must match
the gradients of the whole token set, because the masked dW, dL and dR are
sums over tokens; the only differences are the per-rank bf16 rounding of dW,
the fp32 sum and the final rounding of dW, which the test bounds.  Weights and
the static mask are the same on every rank.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from structured_sparse_pretraining_b200 import dp
from structured_sparse_pretraining_b200 import inputs as I

T, IN, OUT, R = 96, 128, 64, 8


def _grads(X, dY, W, L, Rm, meta):
    """Oracle masked dW [out, in/2], dL [in, r], dR [r, out] of one token set (fp64)."""
    XL = oracle.adapter_fwd(I.bits(X), I.bits(L))
    G = oracle.adapter_g(I.bits(dY), I.bits(Rm))
    Gb = oracle.bf16_values(I.bits(torch.from_numpy(G).float().bfloat16()))  # G as the library stores it
    XLb = oracle.bf16_values(I.bits(torch.from_numpy(XL).float().bfloat16()))
    dW = oracle.bwd_dw_masked(I.bits(dY), I.bits(X), meta)
    dL = oracle.adapter_dl(I.bits(X), Gb)
    dR = oracle.adapter_dr(XLb, I.bits(dY)).T
    return dW, dL, dR


def _as_stored(dW, dL, dR):
    """The gradients in the formats the GPU kernels write: dW bf16, dL and dR fp32."""
    dWb = torch.from_numpy(np.ascontiguousarray(dW)).float().bfloat16()
    return dp.replicated_gradients(dWb, torch.from_numpy(np.ascontiguousarray(dL)).float(),
                                   torch.from_numpy(np.ascontiguousarray(dR)).float())


def _inputs():
    X = I.normal_bf16((T, IN), 1.0, dp.token_seed(0), 0, "X")
    dY = I.normal_bf16((T, OUT), 1e-2, dp.token_seed(0), 0, "dY")
    W = I.normal_bf16((OUT, IN), 0.02, dp.WEIGHT_SEED, 0, "W")
    L = I.normal_bf16((IN, R), 0.02, dp.WEIGHT_SEED, 0, "L")
    Rm = I.normal_bf16((R, OUT), 0.02, dp.WEIGHT_SEED, 0, "R")
    return X, dY, W, L, Rm


def _rank(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, dY, W, L, Rm = _inputs()
        _, meta, _ = oracle.prune24(I.bits(W))  # every rank prunes the same weights
        a, b = dp.shard(T, world, rank)
        ts = _as_stored(*_grads(X[a:b], dY[a:b], W, L, Rm, meta))
        if rank == 0:
            torch.save([t.clone() for t in ts], out_path + ".shard0")
        dp.allreduce_gradients(ts)
        if rank == 0:
            torch.save([t.clone() for t in ts], out_path)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_allreduced_shard_gradients_equal_full_batch(tmp_path, world):
    out_path = str(tmp_path / "grads.pt")
    mp.start_processes(_rank, args=(world, _free_port(), out_path), nprocs=world, start_method="spawn", join=True)
    got = torch.load(out_path)
    assert got[0].dtype == torch.bfloat16 and got[1].dtype == got[2].dtype == torch.float32
    X, dY, W, L, Rm = _inputs()
    _, meta, _ = oracle.prune24(I.bits(W))
    want = _grads(X, dY, W, L, Rm, meta)
    # every rank's shard, as stored, summed in fp64 here: the fp32 sum differs
    # from it by fp32 rounding only
    shards = []
    for r in range(world):
        a, b = dp.shard(T, world, r)
        shards.append([t.double().numpy() for t in _as_stored(*_grads(X[a:b], dY[a:b], W, L, Rm, meta))])
    for i, name in enumerate(("dW", "dL", "dR")):
        g = got[i].double().numpy()
        exact = sum(sh[i] for sh in shards)
        # fp32 sum: |err| <= (world - 1) * 2^-24 * sum|terms|; dW then rounds once to bf16 (half an ulp: at most 2^-8 of the value)
        tol = (world - 1) * 2.0 ** -24 * sum(np.abs(sh[i]) for sh in shards)
        if name == "dW":
            tol = tol + 2.0 ** -8 * np.abs(exact) * (1 + 1e-6)
        assert np.all(np.abs(g - exact) <= tol + 1e-30), name
        # and against the whole token set's gradient (fp64 oracle): only the
        # per-rank bf16 rounding of dW adds to the above
        if name == "dW":
            bound = 2.0 ** -8 * sum(np.abs(sh[i]) for sh in shards) + tol
        else:
            bound = 1e-6 * np.abs(want[i]).max() + tol
        assert np.all(np.abs(g - want[i]) <= bound + 1e-30), name
    if world == 2:   # two terms: the fp32 sum is exact in any order, then one bf16 rounding
        s0 = torch.load(out_path + ".shard0")
        exact0 = [(s0[i].float() + torch.from_numpy(shards[1][i]).float()) for i in range(3)]
        assert torch.equal(got[0], exact0[0].bfloat16())
        assert torch.equal(got[1], exact0[1]) and torch.equal(got[2], exact0[2])


def test_shard_covers_every_item_once():
    for n in (0, 1, 7, 96, 1000):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = dp.shard(n, world, r)
                assert 0 <= a <= b <= n
                seen.extend(range(a, b))
            assert seen == list(range(n))


def _rank_step(rank, world, port, out_prefix):
    """A full data-parallel step: shard gradients, all-reduce, then every rank
    takes the same AdamW step on its replica of the kept values and prunes
    the updated W^R again (the oracle stands in for the fused GPU kernel)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, dY, W, L, Rm = _inputs()
        vals, meta, _ = oracle.prune24(I.bits(W))
        a, b = dp.shard(T, world, rank)
        ts = _as_stored(*_grads(X[a:b], dY[a:b], W, L, Rm, meta))
        dp.allreduce_gradients(ts)
        g = I.bits(ts[0])  # the summed compressed gradient, bf16 as the optimizer step takes it
        m = np.zeros(vals.shape, np.float32)
        v = np.zeros(vals.shape, np.float32)
        vals, m, v = oracle.adamw_compressed(vals, g, m, v, 1e-3, 0.9, 0.999, 1e-8, 0.01, 1)
        vt, mt = oracle.double_prune(vals, meta, OUT, IN)
        np.savez(f"{out_prefix}{rank}.npz", vals=vals, m=m, v=v, vt=vt, mt=mt)
    finally:
        dist.destroy_process_group()


def test_replicas_stay_identical_after_the_optimizer_step(tmp_path):
    world = 2
    prefix = str(tmp_path / "rank")
    mp.start_processes(_rank_step, args=(world, _free_port(), prefix), nprocs=world, start_method="spawn", join=True)
    res = [np.load(f"{prefix}{r}.npz") for r in range(world)]
    for k in ("vals", "m", "v", "vt", "mt"):
        np.testing.assert_array_equal(res[0][k], res[1][k], err_msg=k)
    W = _inputs()[2]
    vals0, _, _ = oracle.prune24(I.bits(W))
    assert np.mean(res[0]["vals"] != vals0) > 0.3  # the step moved most kept values
