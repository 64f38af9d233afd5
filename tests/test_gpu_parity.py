"""GPU parity: every entry point of libslope.so, called through the C ABI,
against the CPU oracle on the same seeded inputs.

Integer work (vals, meta, vals_t, meta_t) must match bit for bit; floating
point outputs must meet the tolerance of parity_util.check_close.  Small
cases span several 128 x 128 tiles and a ragged tail (T not a multiple of
128, in not a multiple of 128, out not a multiple of 128); full-size cases
use the workloads' own shapes and the bench's launch configuration and
compare sampled rows that the oracle computes one by one.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from parity_util import bits_i16, check_close, check_guards, cuda_bf16, cuda_i16, guarded_empty, to_f64
from structured_sparse_pretraining_b200 import _lib, ops
from structured_sparse_pretraining_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    oracle.threads(len(os.sched_getaffinity(0)))
    ops.device_check()
    yield
    ops.status_sync()


def small_inputs(T, inn, out, r, seed=0, std_r=0.02):
    w = I.Workload("case", (I.Layer(inn, out),), T, r, r, std_r=std_r)
    return I.layer_inputs(w, 0, seed=seed)


# (T, in, out, r): several tiles in every direction and ragged tails
SMALL = [
    (256, 512, 512, 8),     # the single-layer workload's shape
    (300, 192, 320, 8),     # ragged T, K with a half k-tile, ragged M tile
    (129, 256, 128, 0),     # no adapter
    (1, 64, 64, 8),         # one token, one group-tile
    (16, 128, 192, 16),
    (200, 384, 256, 96),    # rank above 64: two adapter k-tiles, 128-wide adapter tiles
    (130, 320, 448, 64),
    (1800, 1024, 2560, 16), # more tiles than SM pairs: pairs loop over several tiles, adapter stages interleave
    (9000, 128, 256, 8),    # one weight-row pair, many token tiles: unshared token tiles
    (520, 256, 384, 32),    # rank 32: adapter tile in its own buffer, 64-byte swizzle
    (333, 448, 320, 24),    # rank 24 padded to 32 (zero fill past r)
    (2100, 640, 1536, 32),  # rank 32 over several tiles per pair: the adapter buffer is reused
    (4096, 512, 512, 8),    # masked dW split over tokens 8 ways (256-wide tiles): last-arriver reduction
    (8500, 128, 512, 8),    # fwd on 240-wide token tiles (one wave where 224 needs two): 8-slot code ring
    (700, 256, 4096, 8),    # fwd on 176-wide token tiles
    (1300, 2048, 512, 8),   # bwd_dx on 224-wide token tiles
    # few tokens: narrow token tiles, the sum over K split across SM pairs
    (1, 4096, 512, 8),      # fwd split 4 ways on 16-wide tiles, adapter (own buffer) in split 0
    (40, 2112, 832, 96),    # fwd split 5 ways: ragged M tile, half k-tile, adapter k-tiles in split 0; bwd_dx split 2, codes not by TMA
    (200, 512, 4096, 8),    # fwd on 64-wide tiles; bwd_dx 32-wide split 4 ways
    (128, 2048, 1536, 64),  # 64-wide tiles split 4 (fwd) and 3 (bwd_dx) ways, rank-64 adapter k-tile
    (96, 1536, 2048, 24),   # 32-wide tiles split 3 and 4 ways, rank 24 padded to 32
    (700, 2048, 2048, 16),  # 128-wide tiles split 3 ways
    # rank products on CUDA cores (<= 32 tokens) at the rank limits, and just past them
    (32, 512, 256, 256),    # 2 blocks of 16 tokens, rank 256 (2 k-groups per column pair)
    (5, 1024, 640, 200),    # a ragged token block, rank 200
    (12, 36864, 512, 96),   # 64 splits of K: both levels of the final sum (8 groups of 8)
    (33, 1024, 640, 8),     # 33 tokens: the tensor-core path with rank 8
]


# ------------------------------------------------------------------ prune kernels
@pytest.mark.parametrize("rows,K", [(64, 64), (320, 192), (512, 512), (3072, 768), (1000, 1024),
                                    (20000, 2048)])  # several grid-stride passes of four chunks per thread
def test_prune24_bitexact(rows, K):
    W = I.normal_bf16((rows, K), 0.02, 3, 0, "W")
    vals_o, meta_o, st = oracle.prune24(I.bits(W))
    assert st == oracle.OK
    vals, meta = ops.prune24(W.cuda())
    np.testing.assert_array_equal(bits_i16(vals), vals_o)
    np.testing.assert_array_equal(bits_i16(meta), meta_o)


def test_prune24_ties_and_signed_zeros():
    alphabet = np.array([0.0, -0.0, 1.0, -1.0, 2.0, 0.5, -2.0, 3.0], np.float32)
    g = torch.Generator().manual_seed(9)
    idx = torch.randint(0, len(alphabet), (256, 128), generator=g).numpy()
    Wb = (alphabet[idx].view(np.uint32) >> 16).astype(np.uint16)
    vals_o, meta_o, _ = oracle.prune24(Wb)
    vals, meta = ops.prune24(cuda_bf16(Wb))
    np.testing.assert_array_equal(bits_i16(vals), vals_o)
    np.testing.assert_array_equal(bits_i16(meta), meta_o)


@pytest.mark.parametrize("out,inn", [(64, 64), (320, 192), (512, 512), (768, 3072), (1024, 4096),
                                     (4096, 4096),   # 128-row tiles, several per CTA: the prefetched next tile
                                     (8128, 1024)])  # 64-row tiles (out % 128 == 64), several per CTA
def test_double_prune_bitexact(out, inn):
    W = I.normal_bf16((out, inn), 0.02, 4, 0, "W")
    vals_o, meta_o, _ = oracle.prune24(I.bits(W))
    vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
    vt, mt = ops.double_prune(cuda_bf16(vals_o), cuda_i16(meta_o), out, inn)
    np.testing.assert_array_equal(bits_i16(vt), vt_o)
    np.testing.assert_array_equal(bits_i16(mt), mt_o)


def _edge_alphabet_weights(out, inn, seed):
    """W over an alphabet with +0, -0, repeated magnitudes of both signs and a
    subnormal; some 4-row blocks are all zero and some hold one non-zero per
    column, so that W^R has column groups with 0, 1 and 2+ kept entries, kept
    -0 values next to the +0 of pruned slots, and equal magnitudes inside a
    column group (the second pruning must then keep the lower rows)."""
    alphabet = np.array([0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 0.5, 3.0, -3.0, 1e-40], np.float32)
    g = torch.Generator().manual_seed(seed)
    idx = torch.randint(0, len(alphabet), (out, inn), generator=g).numpy()
    Wb = (alphabet[idx].view(np.uint32) >> 16).astype(np.uint16)
    Wb[0:4, :] = 0                    # an all-zero block of four rows: every column group empty
    Wb[4:8, :] = 0x8000               # -0 everywhere in the next block
    Wb[8:12, :] = 0
    Wb[9, :] = 0x3F80                 # one non-zero (+1) per column group
    Wb[12:16, :] = 0xBF80             # -1 in every row: all magnitudes equal
    return Wb


@pytest.mark.parametrize("out,inn", [(64, 64), (320, 192), (512, 1024), (8128, 1024)])
def test_double_prune_ties_and_signed_zeros(out, inn):
    """The second pruning on a W^R with kept -0 values beside the +0 padding,
    equal magnitudes inside column groups and groups with fewer than two
    non-zeros: bit-exact against the oracle (ties to the lower out index,
    +0 == -0)."""
    Wb = _edge_alphabet_weights(out, inn, 21)
    vals_o, meta_o, _ = oracle.prune24(Wb)
    vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
    vt, mt = ops.double_prune(cuda_bf16(vals_o), cuda_i16(meta_o), out, inn)
    ops.status_sync()
    np.testing.assert_array_equal(bits_i16(vt), vt_o)
    np.testing.assert_array_equal(bits_i16(mt), mt_o)
    # the case covers what it claims: kept -0 and empty column groups exist
    assert np.any(vals_o == 0x8000)
    Wr = oracle.decompress(vals_o, meta_o, inn)
    nnz = ((Wr & 0x7FFF) != 0).reshape(out // 4, 4, inn).sum(axis=1)
    assert np.any(nnz == 0) and np.any(nnz == 1)


@pytest.mark.parametrize("out,inn", [(64, 64), (320, 192), (768, 3072), (4096, 4096),  # 128-row tiles, several per CTA
                                     (8128, 1024),                                     # 64-row tiles
                                     (20480, 2048)])                                   # many grid-stride passes
def test_prune24_double_bitexact(out, inn):
    """Both prunings in one launch: the four outputs bit for bit equal to the
    oracle's prune24 then double_prune."""
    W = I.normal_bf16((out, inn), 0.02, 5, 0, "W")
    vals_o, meta_o, st = oracle.prune24(I.bits(W))
    assert st == oracle.OK
    vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
    vals, meta, vt, mt = ops.prune24_double(W.cuda())
    ops.status_sync()
    np.testing.assert_array_equal(bits_i16(vals), vals_o)
    np.testing.assert_array_equal(bits_i16(meta), meta_o)
    np.testing.assert_array_equal(bits_i16(vt), vt_o)
    np.testing.assert_array_equal(bits_i16(mt), mt_o)


@pytest.mark.parametrize("out,inn", [(64, 64), (320, 192), (512, 1024), (8128, 1024)])
def test_prune24_double_ties_and_signed_zeros(out, inn):
    """The one-launch pruning on the edge alphabet (±0, equal magnitudes,
    empty and single-entry column groups, a subnormal)."""
    Wb = _edge_alphabet_weights(out, inn, 23)
    vals_o, meta_o, _ = oracle.prune24(Wb)
    vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
    vals, meta, vt, mt = ops.prune24_double(cuda_bf16(Wb))
    ops.status_sync()
    for got, ref in ((vals, vals_o), (meta, meta_o), (vt, vt_o), (mt, mt_o)):
        np.testing.assert_array_equal(bits_i16(got), ref)


def test_prune24_double_reports_nonfinite():
    """A NaN in W is reported by the one-launch pruning as by prune24."""
    W = I.normal_bf16((256, 256), 0.02, 6, 0, "W")
    W[17, 33] = float("nan")
    ops.prune24_double(W.cuda())
    with pytest.raises(_lib.SlopeError) as e:
        ops.status_sync()
    assert e.value.code == 4
    ops.status_sync()  # cleared


@pytest.mark.parametrize("out,inn", [(320, 192), (512, 1024), (8128, 1024)])
@pytest.mark.parametrize("lr,wd", [(1e-3, 0.1), (0.0, 0.0)])
def test_adamw_double_prune_ties_and_signed_zeros(out, inn, lr, wd):
    """The fused AdamW step + second pruning on the same edge-case W^R, with a
    gradient drawn from a small alphabet (zeros included) so that equal
    weights with equal gradients stay tied after the step, and with lr = 0
    (the weights do not move: the pruning sees the edge cases unchanged)."""
    Wb = _edge_alphabet_weights(out, inn, 22)
    vals_o, meta_o, _ = oracle.prune24(Wb)
    galpha = np.array([0.0, -0.0, 0.25, -0.25, 1.0], np.float32)
    gi = torch.randint(0, len(galpha), (out, inn // 2), generator=torch.Generator().manual_seed(23)).numpy()
    gb = (galpha[gi].view(np.uint32) >> 16).astype(np.uint16)
    vals = cuda_bf16(vals_o)
    m = torch.zeros(out, inn // 2, dtype=torch.float32, device="cuda")
    v = torch.zeros_like(m)
    m_o = np.zeros((out, inn // 2), np.float32)
    v_o = np.zeros_like(m_o)
    hp = dict(lr=lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wd)
    for step in (1, 2):
        vt, mt = ops.adamw_double_prune(vals, cuda_i16(meta_o), cuda_bf16(gb), m, v, out, inn, step=step, **hp)
        ops.status_sync()
        vals_o, m_o, v_o = oracle.adamw_compressed(vals_o, gb, m_o, v_o, hp["lr"], hp["beta1"], hp["beta2"],
                                                   hp["eps"], hp["weight_decay"], step)
        vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
        np.testing.assert_array_equal(bits_i16(vals), vals_o, err_msg=f"vals, step {step}")
        np.testing.assert_array_equal(m.cpu().numpy().view(np.uint32), m_o.view(np.uint32), err_msg=f"m, step {step}")
        np.testing.assert_array_equal(v.cpu().numpy().view(np.uint32), v_o.view(np.uint32), err_msg=f"v, step {step}")
        np.testing.assert_array_equal(bits_i16(vt), vt_o, err_msg=f"vals_t, step {step}")
        np.testing.assert_array_equal(bits_i16(mt), mt_o, err_msg=f"meta_t, step {step}")
    assert np.any(vals_o == 0x8000)   # kept -0 values survive into the pruned step


@pytest.mark.parametrize("out,inn", [(64, 64), (320, 192), (768, 3072), (4096, 1024),
                                     (8128, 1024)])  # 64-row tiles (out % 128 == 64)
def test_adamw_double_prune_bitexact(out, inn):
    """Two fused AdamW + second-pruning steps against the oracle's AdamW and
    double_prune: updated values, states, vals_t and meta_t bit for bit."""
    W = I.normal_bf16((out, inn), 0.02, 6, 0, "W")
    vals_o, meta_o, _ = oracle.prune24(I.bits(W))
    vals = cuda_bf16(vals_o)
    meta = cuda_i16(meta_o)
    m = torch.zeros(out, inn // 2, dtype=torch.float32, device="cuda")
    v = torch.zeros_like(m)
    m_o = np.zeros((out, inn // 2), np.float32)
    v_o = np.zeros_like(m_o)
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1)
    for step in (1, 2):
        g = I.normal_bf16((out, inn // 2), 1e-2, 7, step, "dW")
        vt, mt = ops.adamw_double_prune(vals, meta, g.cuda(), m, v, out, inn, step=step, **hp)
        ops.status_sync()
        vals_o, m_o, v_o = oracle.adamw_compressed(vals_o, I.bits(g), m_o, v_o, hp["lr"], hp["beta1"], hp["beta2"],
                                                   hp["eps"], hp["weight_decay"], step)
        vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
        np.testing.assert_array_equal(bits_i16(vals), vals_o, err_msg=f"vals, step {step}")
        np.testing.assert_array_equal(m.cpu().numpy(), m_o, err_msg=f"m, step {step}")
        np.testing.assert_array_equal(v.cpu().numpy(), v_o, err_msg=f"v, step {step}")
        np.testing.assert_array_equal(bits_i16(vt), vt_o, err_msg=f"vals_t, step {step}")
        np.testing.assert_array_equal(bits_i16(mt), mt_o, err_msg=f"meta_t, step {step}")
    assert np.mean(vals_o != oracle.prune24(I.bits(W))[0]) > 0.3  # the two steps moved most weights


@pytest.mark.parametrize("N,M", [(1, 4), (2, 4), (3, 4), (1, 8), (2, 8), (4, 8), (7, 8), (2, 16), (8, 16), (15, 16)])
@pytest.mark.parametrize("rows,K", [(64, 64), (300, 192), (1000, 4096)])
def test_prune_nm_bitexact(N, M, rows, K):
    W = I.normal_bf16((rows, K), 0.02, 8, M, "W")
    Wb = I.bits(W).copy()
    Wb[0, :M] = 0          # an all-zero group (ties among +0)
    Wb[1, :M] = 0x8000     # -0 everywhere
    Wb[2, 0:M:2] = Wb[2, 1]  # repeated magnitudes
    vals_o, pos_o, _ = oracle.prune_nm(Wb, N, M)
    vals, pos = ops.prune_nm(cuda_bf16(Wb), N, M)
    ops.status_sync()
    np.testing.assert_array_equal(bits_i16(vals), vals_o)
    np.testing.assert_array_equal(pos.cpu().numpy(), pos_o)


def test_prune_nm_two_of_four_is_prune24():
    W = I.normal_bf16((512, 1024), 0.02, 9, 0, "W").cuda()
    v, p = ops.prune_nm(W, 2, 4)
    v24, m24 = ops.prune24(W)
    ops.status_sync()
    assert torch.equal(v.view(torch.int16), v24.view(torch.int16))
    codes = m24.cpu().numpy().view(np.uint16)
    codes = np.stack([(codes >> (4 * q)) & 0xF for q in range(4)], axis=2).reshape(512, -1)
    pn = p.cpu().numpy()
    np.testing.assert_array_equal(pn[:, 0::2], codes & 3)
    np.testing.assert_array_equal(pn[:, 1::2], codes >> 2)


def test_nonfinite_input_is_reported():
    W = I.normal_bf16((128, 256), 0.02, 5, 0, "W")
    W[7, 33] = float("nan")
    ops.prune24(W.cuda())
    with pytest.raises(_lib.SlopeError) as e:
        ops.status_sync()
    assert e.value.code == 4
    ops.status_sync()  # the error word was cleared


def test_bounded_wait_timeout_is_reported_and_the_device_stays_usable():
    # a wait on a barrier no one signals runs out after ~10 ms: no fault, no hang
    ops.selftest_wait_timeout()
    with pytest.raises(_lib.SlopeError) as e:
        ops.status_sync()
    assert e.value.code == 5
    ops.status_sync()  # the error word was cleared
    W = I.normal_bf16((256, 512), 0.02, 6, 0, "W")
    vals_o, meta_o, _ = oracle.prune24(I.bits(W))
    vals, meta = ops.prune24(W.cuda())
    ops.status_sync()
    np.testing.assert_array_equal(bits_i16(vals), vals_o)
    np.testing.assert_array_equal(bits_i16(meta), meta_o)


# ------------------------------------------------------------------ products, one call each
@pytest.mark.parametrize("T,inn,out,r", SMALL)
def test_fwd_parity(T, inn, out, r):
    d = small_inputs(T, inn, out, r)
    vals_o, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    XL = I.normal_bf16((T, r), 1.0, 0, 0, "L") if r else None   # a shared seeded XL input
    Y = ops.fwd(d["X"].cuda(), cuda_bf16(vals_o), cuda_i16(meta_o), XL.cuda() if r else None,
                d["R"].cuda() if r else None, out)
    ref = oracle.fwd(I.bits(d["X"]), vals_o, meta_o, oracle.bf16_values(I.bits(XL)) if r else None,
                     I.bits(d["R"]) if r else None, out)
    check_close(to_f64(Y), ref, "Y")


@pytest.mark.parametrize("T,inn,out,r", SMALL)
def test_bwd_dx_parity(T, inn, out, r):
    d = small_inputs(T, inn, out, r)
    vals_o, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
    G = I.normal_bf16((T, r), 0.05, 0, 0, "R") if r else None
    dX = ops.bwd_dx(d["dY"].cuda(), cuda_bf16(vt_o), cuda_i16(mt_o), G.cuda() if r else None,
                    d["L"].cuda() if r else None, inn)
    ref = oracle.bwd_dx(I.bits(d["dY"]), vt_o, mt_o, oracle.bf16_values(I.bits(G)) if r else None,
                        I.bits(d["L"]) if r else None, inn)
    check_close(to_f64(dX), ref, "dX")


@pytest.mark.parametrize("T,inn,out,r", SMALL)
def test_bwd_dw_masked_parity(T, inn, out, r):
    d = small_inputs(T, inn, out, r)
    vals_o, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    dW = ops.bwd_dw_masked(d["dY"].cuda(), d["X"].cuda(), cuda_i16(meta_o))
    ref = oracle.bwd_dw_masked(I.bits(d["dY"]), I.bits(d["X"]), meta_o)
    check_close(to_f64(dW), ref, "dW")


@pytest.mark.parametrize("T,inn,out,r", [c for c in SMALL if c[3] > 0])
def test_adapter_parity(T, inn, out, r):
    d = small_inputs(T, inn, out, r)
    XL = ops.adapter_fwd(d["X"].cuda(), d["L"].cuda())
    check_close(to_f64(XL), oracle.adapter_fwd(I.bits(d["X"]), I.bits(d["L"])), "XL")
    XLs = I.normal_bf16((T, r), 1.0, 1, 0, "L")                 # shared seeded XL input
    dL, dR, G = ops.adapter_bwd(d["X"].cuda(), d["dY"].cuda(), XLs.cuda(), d["R"].cuda())
    G_ref = oracle.adapter_g(I.bits(d["dY"]), I.bits(d["R"]))
    check_close(to_f64(G), G_ref, "G")
    check_close(to_f64(dR), oracle.adapter_dr(oracle.bf16_values(I.bits(XLs)), I.bits(d["dY"])).T, "dR")
    check_close(to_f64(dL), oracle.adapter_dl(I.bits(d["X"]), G_ref), "dL")


# ------------------------------------------------------------------ the whole layer step
def gpu_step(d, out, r, fused=True):
    """The hot path on the GPU for one layer: with `fused`, as bench.py runs it
    (both prunings in one launch, the rank products inside the sparse
    products and the masked gradient), else with the separate calls."""
    X, W, dY = d["X"].cuda(), d["W"].cuda(), d["dY"].cuda()
    L = d["L"].cuda() if r else None
    R = d["R"].cuda() if r else None
    inn = X.shape[1]
    if fused:
        vals, meta, vt, mt = ops.prune24_double(W)
        XL, Y = ops.fwd_fused(X, vals, meta, L, R, out)
        G, dX = ops.bwd_dx_fused(dY, vt, mt, R, L, inn)
        dW, dL, dR = ops.bwd_dw_fused(dY, X, meta, XL, G)
    else:
        vals, meta = ops.prune24(W)
        vt, mt = ops.double_prune(vals, meta, out, inn)
        XL = ops.adapter_fwd(X, L) if r else None
        Y = ops.fwd(X, vals, meta, XL, R, out)
        if r:
            dL, dR, G = ops.adapter_bwd(X, dY, XL, R)
        else:
            dL = dR = G = None
        dX = ops.bwd_dx(dY, vt, mt, G, L, inn)
        dW = ops.bwd_dw_masked(dY, X, meta)
    ops.status_sync()
    return dict(vals=vals, meta=meta, vals_t=vt, meta_t=mt, XL=XL, Y=Y, G=G, dL=dL, dR=dR, dX=dX, dW=dW)


@pytest.mark.parametrize("T,inn,out,r", SMALL)
@pytest.mark.parametrize("std_r", [1e-3, 0.02])
@pytest.mark.parametrize("fused", [False, True])
def test_layer_step_parity(T, inn, out, r, std_r, fused):
    d = small_inputs(T, inn, out, r, std_r=std_r)
    g = gpu_step(d, out, r, fused)
    o = oracle.layer_step(I.bits(d["X"]), I.bits(d["W"]), I.bits(d["L"]) if r else None,
                          I.bits(d["R"]) if r else None, I.bits(d["dY"]))
    for k in ("vals", "meta", "vals_t", "meta_t"):
        np.testing.assert_array_equal(bits_i16(g[k]), o[k], err_msg=k)
    for k in ("Y", "dX", "dW") + (("XL", "G", "dL", "dR") if r else ()):
        check_close(to_f64(g[k]), o[k], k)


def test_split_sum_is_deterministic():
    """A K-split product sums its partials in split order, whichever split
    arrives last: two calls give the same bits."""
    T, inn, out, r = 40, 2112, 832, 96
    assert ops.sparse_plan(out, T, inn)[1] > 1
    d = small_inputs(T, inn, out, r)
    vals, meta = ops.prune24(d["W"].cuda())
    X = d["X"].cuda()
    XL = ops.adapter_fwd(X, d["L"].cuda())
    Y1 = ops.fwd(X, vals, meta, XL, d["R"].cuda(), out)
    Y2 = ops.fwd(X, vals, meta, XL, d["R"].cuda(), out)
    ops.status_sync()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


# ------------------------------------------------------------------ rank products fused into the sparse products
# (T, in, out, r): the forward (XL = X . L in the same launch) and the input
# gradient (G = dY . R^T in the same launch); ragged token counts (partial
# 256-token units), ranks from 8 to 128 (L read MN-major with 16, 32 or 64
# columns per CTA; R read K-major), and shapes that take two launches (the
# planner's choice, ops.fused_launches, is asserted for each case).
FUSED = [
    (2100, 512, 2048, 16),    # 9 units, the last one of 52 tokens; in = 512: the shortest fusable reduction
    (4500, 1024, 1024, 8),    # rank 8: one L column block of 16, half zero
    (2048, 768, 3072, 96),    # the GPT-2-small fc1 shape at rank 96: 64 columns per CTA
    (1800, 1536, 2304, 24),   # rank 24 (32 padded); out = 2304 ragged against 512-row tiles
    (2500, 640, 1664, 64),    # in = 640 (5 k-tiles of 128); out ragged; a partial last unit
    (2305, 2048, 2048, 128),  # rank 128; 1 token in the last unit
    (300, 1024, 512, 8),      # rank 8 on 2 small tiles: still one launch
    (16, 4096, 4096, 16),     # 16 tokens: two launches (narrow tiles with the K split)
    (200, 576, 512, 16),      # in = 576 is not a multiple of 128: two launches
    (64, 1024, 1024, 192),    # rank above 128: two launches
]


FUSED_LAUNCHES = {(16, 4096, 4096, 16): 2, (200, 576, 512, 16): 2, (64, 1024, 1024, 192): 2}


@pytest.mark.parametrize("T,inn,out,r", FUSED)
def test_fwd_fused_parity(T, inn, out, r):
    assert ops.fused_launches(out, T, inn, r) == FUSED_LAUNCHES.get((T, inn, out, r), 1)
    d = small_inputs(T, inn, out, r)
    vals_o, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    X = d["X"].cuda()
    XL_ref = oracle.adapter_fwd(I.bits(d["X"]), I.bits(d["L"]))
    Y_ref = oracle.fwd(I.bits(d["X"]), vals_o, meta_o, XL_ref, I.bits(d["R"]), out)
    for _ in range(2):  # the second call starts from the flags the first left
        XL, Y = ops.fwd_fused(X, cuda_bf16(vals_o), cuda_i16(meta_o), d["L"].cuda(), d["R"].cuda(), out)
        ops.status_sync()
        check_close(to_f64(XL), XL_ref, "XL")
        check_close(to_f64(Y), Y_ref, "Y")


@pytest.mark.parametrize("T,inn,out,r", FUSED)
def test_bwd_dx_fused_parity(T, inn, out, r):
    # the input gradient's reduction runs over out: swap so that out takes the in sizes above
    assert ops.fused_launches(out, T, inn, r) == FUSED_LAUNCHES.get((T, inn, out, r), 1)
    inn, out = out, inn
    d = small_inputs(T, inn, out, r)
    vals_o, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
    dY = d["dY"].cuda()
    G_ref = oracle.adapter_g(I.bits(d["dY"]), I.bits(d["R"]))
    dX_ref = oracle.bwd_dx(I.bits(d["dY"]), vt_o, mt_o, G_ref, I.bits(d["L"]), inn)
    for _ in range(2):
        G, dX = ops.bwd_dx_fused(dY, cuda_bf16(vt_o), cuda_i16(mt_o), d["R"].cuda(), d["L"].cuda(), inn)
        ops.status_sync()
        check_close(to_f64(G), G_ref, "G")
        check_close(to_f64(dX), dX_ref, "dX")


# (T, in, out, r): the masked gradient with dR and dL in the same launch; split
# over tokens (few tiles) or not, ranks 8..128, ragged in (a partial 256-row
# block of dL) and a rank above 128 (separate reductions)
DWF = [
    (4096, 512, 512, 16),     # 4 tiles: split 8 ways; dR, dL partials summed in split order
    (8192, 768, 3072, 96),    # the GPT-2-small fc1 shape at rank 96
    (2048, 2560, 2560, 8),    # 100 tiles, not split; rank 8 (16 columns per CTA, half zero)
    (3000, 320, 448, 24),     # ragged T (a partial k-tile), in = 320: a partial dL block; 128-wide dW tiles
    (1024, 1024, 1536, 128),  # rank 128: 64 columns per CTA
    (512, 512, 768, 192),     # rank above 128: the separate reductions
]


@pytest.mark.parametrize("T,inn,out,r", DWF)
def test_bwd_dw_fused_parity(T, inn, out, r):
    d = small_inputs(T, inn, out, r)
    _, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    XL = I.normal_bf16((T, r), 1.0, 2, 0, "L")
    G = I.normal_bf16((T, r), 0.05, 2, 0, "R")
    dY, X = d["dY"].cuda(), d["X"].cuda()
    first = None
    for _ in range(2):  # two calls in a row: counters left at zero, same bits
        dW, dL, dR = ops.bwd_dw_fused(dY, X, cuda_i16(meta_o), XL.cuda(), G.cuda())
        ops.status_sync()
        if first is None:
            first = (dW.clone(), dL.clone(), dR.clone())
        elif r <= 128:
            assert torch.equal(dW, first[0]) and torch.equal(dL, first[1]) and torch.equal(dR, first[2])
    check_close(to_f64(dW), oracle.bwd_dw_masked(I.bits(d["dY"]), I.bits(d["X"]), meta_o), "dW")
    check_close(to_f64(dR), oracle.adapter_dr(oracle.bf16_values(I.bits(XL)), I.bits(d["dY"])).T, "dR")
    check_close(to_f64(dL), oracle.adapter_dl(I.bits(d["X"]), oracle.bf16_values(I.bits(G))), "dL")


def test_fused_rank_product_is_deterministic():
    """The fused XL sums each token row's products in one fixed order: two
    calls give the same bits."""
    T, inn, out, r = 2100, 1024, 2048, 96  # 40 tiles: one launch
    d = small_inputs(T, inn, out, r)
    vals, meta = ops.prune24(d["W"].cuda())
    a = ops.fwd_fused(d["X"].cuda(), vals, meta, d["L"].cuda(), d["R"].cuda(), out)
    b = ops.fwd_fused(d["X"].cuda(), vals, meta, d["L"].cuda(), d["R"].cuda(), out)
    ops.status_sync()
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))


# ------------------------------------------------------------------ no writes outside the outputs
# Every output of the step (fused and separate calls) handed to the library
# inside canary guard bands, on shapes with ragged tails in every direction,
# split launches (few tokens, few tiles), the two-block tiles and the fused
# rank products.
GUARDED = [
    (300, 192, 320, 8),      # ragged T, half k-tile, ragged M tile (pair tiles)
    (1, 4096, 512, 8),       # one token: K split, CUDA-core rank products
    (40, 2112, 832, 96),     # K split with adapter k-tiles, codes not by TMA
    (4096, 512, 512, 8),     # masked dW split over tokens
    (3000, 320, 448, 24),    # 128-wide dW tiles, partial dL block
    (2100, 512, 2048, 16),   # fused in one launch: partial token unit
    (16000, 2048, 1088, 96), # two-block tiles with a ragged last tile, fused rank products
]


@pytest.mark.parametrize("T,inn,out,r", GUARDED)
@pytest.mark.parametrize("fused", [False, True])
def test_no_writes_outside_outputs(T, inn, out, r, fused):
    d = small_inputs(T, inn, out, r)
    X, W, dY = d["X"].cuda(), d["W"].cuda(), d["dY"].cuda()
    L, R = d["L"].cuda(), d["R"].cuda()
    g = lambda *s, dt=torch.bfloat16: guarded_empty(s, dt)  # noqa: E731
    vals, meta = g(out, inn // 2), g(out, inn // 16, dt=torch.int16)
    vt, mt = g(inn, out // 2), g(inn, out // 16, dt=torch.int16)
    XL, G, Y, dX, dW = g(T, r), g(T, r), g(T, out), g(T, inn), g(out, inn // 2)
    dL, dR = g(inn, r, dt=torch.float32), g(r, out, dt=torch.float32)
    if fused:
        ops.prune24_double(W, vals, meta, vt, mt)
        ops.fwd_fused(X, vals, meta, L, R, out, XL, Y)
        ops.bwd_dx_fused(dY, vt, mt, R, L, inn, G, dX)
        ops.bwd_dw_fused(dY, X, meta, XL, G, dW, dL, dR)
    else:
        ops.prune24(W, vals, meta)
        ops.double_prune(vals, meta, out, inn, vt, mt)
        ops.adapter_fwd(X, L, XL)
        ops.fwd(X, vals, meta, XL, R, out, Y)
        ops.adapter_bwd(X, dY, XL, R, dL, dR, G)
        ops.bwd_dx(dY, vt, mt, G, L, inn, dX)
        ops.bwd_dw_masked(dY, X, meta, dW)
    ops.status_sync()
    check_guards()
    # and the outputs were all written (no canary left inside)
    for t in (vals, vt, XL, G, Y, dX, dW):
        assert not torch.isnan(t.float()).any()
    for t in (dL, dR):
        assert not torch.isnan(t).any()


def test_skinny_rank_product_is_deterministic():
    """At a few tokens the rank products run on CUDA cores and sum their 64
    K-split partials in a fixed two-level order: two calls give the same bits."""
    T, inn, r = 12, 36864, 96
    d = small_inputs(T, inn, 512, r)
    X, L = d["X"].cuda(), d["L"].cuda()
    a = ops.adapter_fwd(X, L)
    b = ops.adapter_fwd(X, L)
    ops.status_sync()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    check_close(to_f64(a), oracle.adapter_fwd(I.bits(d["X"]), I.bits(d["L"])), "XL")


def test_separate_adapter_spread_is_bounded():
    """The separate adapter calls add split partials with fp32 atomics (the
    fused calls sum them in a fixed order and repeat bit for bit), so two
    runs of the same call may differ in the last bits.  Bound the spread:
    XL and G (K split over 16 and 8 CTAs at 160 tokens) within one bf16 ulp
    of the larger magnitude plus an fp32-ordering term; dL = X^T G and
    dR = XL^T dY (split over tokens) within what the bf16 flips of G and XL
    carry into them, |X|^T |dG| and |dXL|^T |dY|, plus an fp32-ordering
    term of 1e-5 of their rms."""
    T, inn, out, r = 160, 9216, 4096, 96
    d = small_inputs(T, inn, out, r)
    X, dY, L, R = d["X"].cuda(), d["dY"].cuda(), d["L"].cuda(), d["R"].cuda()
    runs = []
    for _ in range(3):
        XL = ops.adapter_fwd(X, L)
        dL, dR, G = ops.adapter_bwd(X, dY, XL, R)
        ops.status_sync()
        runs.append([t.double().cpu() for t in (XL, G, dL, dR)])
    Xa, dYa = X.double().cpu().abs(), dY.double().cpu().abs()
    XL0, G0, dL0, dR0 = runs[0]
    for XLk, Gk, dLk, dRk in runs[1:]:
        for name, x, y in (("XL", XL0, XLk), ("G", G0, Gk)):
            rms = float(x.pow(2).mean().sqrt())
            bound = torch.maximum(x.abs(), y.abs()) * 2.0 ** -7 + 1e-5 * rms
            assert bool(((x - y).abs() <= bound).all()), f"{name}: beyond one bf16 ulp"
        for name, x, y, carried in (("dL", dL0, dLk, Xa.T @ (G0 - Gk).abs()),
                                    ("dR", dR0, dRk, (XL0 - XLk).abs().T @ dYa)):
            rms = float(x.pow(2).mean().sqrt())
            excess = (x - y).abs() - carried
            assert float(excess.max()) <= 1e-5 * rms, f"{name}: {float(excess.max())} vs rms {rms}"


# ------------------------------------------------------------------ 512-row pair tiles (two blocks per CTA)
# (T, in, out, r, op): shapes whose planner picks the two-block tile; sampled
# tokens, full rows (every m tile and both blocks of each).
WIDE = [
    (16000, 2048, 1088, 96, "fwd"),   # ragged M (2 tiles + 64 rows), ragged T, adapter R^T in 2 ring k-tiles
    (16384, 1024, 2048, 0, "fwd"),    # no adapter, 8 k-tiles
    (16384, 2048, 1024, 16, "fwd"),   # rank 16: one partial adapter k-tile
    (16000, 1088, 2048, 16, "dx"),    # input gradient: M = in = 1088 (ragged), adapter L K-major
    (9000, 2560, 1024, 64, "dx"),     # M = 2560: 5 tiles, one adapter k-tile
]


@pytest.mark.parametrize("T,inn,out,r,op", WIDE)
def test_wide_tile_parity(T, inn, out, r, op):
    M, K = (out, inn) if op == "fwd" else (inn, out)
    assert ops.sparse_tile_rows(M, T, K) == 512
    d = small_inputs(T, inn, out, r)
    vals_o, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    tok = I.sample_rows(T, 48)
    if op == "fwd":
        XL = I.normal_bf16((T, r), 1.0, 0, 0, "L") if r else None
        Y = ops.fwd(d["X"].cuda(), cuda_bf16(vals_o), cuda_i16(meta_o), XL.cuda() if r else None,
                    d["R"].cuda() if r else None, out)
        ops.status_sync()
        ref = oracle.fwd(I.bits(d["X"]), vals_o, meta_o, oracle.bf16_values(I.bits(XL))[tok] if r else None,
                         I.bits(d["R"]) if r else None, out, tok)
        check_close(to_f64(Y[tok]), ref, "Y")
    else:
        vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
        G = I.normal_bf16((T, r), 0.05, 0, 0, "R") if r else None
        dX = ops.bwd_dx(d["dY"].cuda(), cuda_bf16(vt_o), cuda_i16(mt_o), G.cuda() if r else None,
                        d["L"].cuda() if r else None, inn)
        ops.status_sync()
        ref = oracle.bwd_dx(I.bits(d["dY"]), vt_o, mt_o, oracle.bf16_values(I.bits(G))[tok] if r else None,
                            I.bits(d["L"]) if r else None, inn, tok)
        check_close(to_f64(dX[tok]), ref, "dX")


# ------------------------------------------------------------------ full-size workloads, sampled
FULL = [("C1", 0), ("C2", 0), ("C2", 1), ("C3", 0), ("C3", 3), ("C4", 0), ("C4", 1), ("C4", 2), ("C4", 3),
        ("C5", 0), ("C5", 1), ("C5", 2), ("C5", 3)]


@pytest.mark.parametrize("cfg,layer", FULL)
def test_full_size_sampled(cfg, layer):
    w = I.WORKLOADS[cfg]
    lay = w.layers[layer]
    inn, out, T = lay.in_features, lay.out_features, w.tokens
    d = I.layer_inputs(w, layer, seed=0)
    L, R = I.pad_rank(d["L"], d["R"], w.rank_stored)
    d_gpu = dict(d, L=L, R=R)
    g = gpu_step(d_gpu, out, w.rank_stored)
    Xb, Wb, dYb = I.bits(d["X"]), I.bits(d["W"]), I.bits(d["dY"])
    Lb, Rb = I.bits(d["L"]), I.bits(d["R"])
    # masks and compressed copies: in full
    vals_o, meta_o, _ = oracle.prune24(Wb)
    np.testing.assert_array_equal(bits_i16(g["vals"]), vals_o)
    np.testing.assert_array_equal(bits_i16(g["meta"]), meta_o)
    vt_o, mt_o = oracle.double_prune(vals_o, meta_o, out, inn)
    np.testing.assert_array_equal(bits_i16(g["vals_t"]), vt_o)
    np.testing.assert_array_equal(bits_i16(g["meta_t"]), mt_o)
    # products: sampled rows
    tok = I.sample_rows(T, 24)
    XL_rows = oracle.adapter_fwd(Xb, Lb, tok)
    r = w.rank
    check_close(to_f64(g["XL"][tok][:, :r]), XL_rows, "XL")
    check_close(to_f64(g["Y"][tok]), oracle.fwd(Xb, vals_o, meta_o, XL_rows, Rb, out, tok), "Y")
    G_full = oracle.adapter_g(dYb, Rb)
    check_close(to_f64(g["G"][tok][:, :r]), G_full[tok], "G")
    check_close(to_f64(g["dX"][tok]), oracle.bwd_dx(dYb, vt_o, mt_o, G_full[tok], Lb, inn, tok), "dX")
    orow = I.sample_rows(out, 8)
    check_close(to_f64(g["dW"][orow]), oracle.bwd_dw_masked(dYb, Xb, meta_o, orow), "dW")
    irow = I.sample_rows(inn, 8)
    check_close(to_f64(g["dL"][irow][:, :r]), oracle.adapter_dl(Xb, G_full, irow), "dL")
    XL_full = oracle.adapter_fwd(Xb, Lb)
    check_close(to_f64(g["dR"][:r, orow]).T, oracle.adapter_dr(XL_full, dYb, orow), "dR")
    if w.rank_stored > r:   # zero padding stays exactly zero
        assert torch.count_nonzero(g["dL"][:, r:]).item() == 0
        assert torch.count_nonzero(g["dR"][r:, :]).item() == 0


@pytest.mark.parametrize("T", [1, 16, 128, 2048])
def test_fwd_token_sweep_sampled(T):
    """The inference sweep of the largest workload (fwd only, rank 92 stored as 96)."""
    w = I.WORKLOADS["C5"]
    lay = w.layers[0]
    d = I.layer_inputs(w, 0, seed=0, tokens=T)
    L, R = I.pad_rank(d["L"], d["R"], w.rank_stored)
    vals, meta = ops.prune24(d["W"].cuda())
    X = d["X"].cuda()
    XL = ops.adapter_fwd(X, L.cuda())
    Y = ops.fwd(X, vals, meta, XL, R.cuda(), lay.out_features)
    ops.status_sync()
    vals_o, meta_o, _ = oracle.prune24(I.bits(d["W"]))
    tok = I.sample_rows(T, 8)
    XL_rows = oracle.adapter_fwd(I.bits(d["X"]), I.bits(d["L"]), tok)
    check_close(to_f64(Y[tok]), oracle.fwd(I.bits(d["X"]), vals_o, meta_o, XL_rows, I.bits(d["R"]),
                                          lay.out_features, tok), "Y")


# ------------------------------------------------------------------ argument errors (host-side)
def test_argument_errors():
    X = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    vals = torch.zeros(64, 32, dtype=torch.bfloat16, device="cuda")
    meta = torch.zeros(64, 4, dtype=torch.int16, device="cuda")
    Y = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    lib = _lib.load()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.slope_fwd(None, vals.data_ptr(), meta.data_ptr(), None, None, 8, 64, 64, 0, Y.data_ptr(), s) == 1
    assert lib.slope_fwd(X.data_ptr() + 2, vals.data_ptr(), meta.data_ptr(), None, None, 8, 64, 64, 0,
                         Y.data_ptr(), s) == 3
    assert lib.slope_fwd(X.data_ptr(), vals.data_ptr(), meta.data_ptr(), None, None, 8, 96, 64, 0,
                         Y.data_ptr(), s) == 2
    assert lib.slope_fwd(X.data_ptr(), vals.data_ptr(), meta.data_ptr(), X.data_ptr(), X.data_ptr(), 8, 64, 64,
                         12, Y.data_ptr(), s) == 2
    assert lib.slope_fwd(X.data_ptr(), vals.data_ptr(), meta.data_ptr(), None, None, 0, 64, 64, 0,
                         Y.data_ptr(), s) == 1
    assert b"multiple of 64" in lib.slope_last_error() or len(lib.slope_last_error()) > 0
    ops.status_sync()
