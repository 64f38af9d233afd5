"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks the oracle against one of: brute force on tiny inputs
(Python, written from the definition of top-2-of-4 magnitude pruning),
exhaustive enumeration, a closed form, an fp64 numpy matmul of dense
matrices, fp64 torch autograd, or a value printed on the pages.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from structured_sparse_pretraining_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LEGAL_CODES = {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}


# ---------------------------------------------------------------- helpers
def f32_to_bf16_bits(x):
    """Exact bf16 patterns for values that are exactly representable."""
    a = np.asarray(x, dtype=np.float32)
    b = a.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (b >> 16).astype(np.uint16)


def top2_bruteforce(group):
    """Kept positions of one group: the first two of a stable sort by
    decreasing |value| (Python floats; |-0.0| == 0.0)."""
    order = sorted(range(4), key=lambda k: (-abs(float(group[k])), k))
    return tuple(sorted(order[:2]))


def mask_numpy(Wf):
    """Row-wise 2:4 magnitude mask of a float matrix, written independently of
    the oracle: stable argsort of -|w| inside each group of four."""
    rows, K = Wf.shape
    g = np.abs(Wf).reshape(rows, K // 4, 4)
    order = np.argsort(-g, axis=2, kind="stable")
    keep = np.zeros_like(g, dtype=bool)
    np.put_along_axis(keep, order[:, :, :2], True, axis=2)
    return keep.reshape(rows, K)


def codes_of(meta, K):
    rows = meta.shape[0]
    out = np.zeros((rows, K // 4), np.int64)
    for g in range(K // 4):
        out[:, g] = (meta[:, g // 4].astype(np.int64) >> (4 * (g % 4))) & 0xF
    return out


def rand_bf16(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    return I.bits((torch.randn(*shape, generator=g) * std).to(torch.bfloat16))


# ---------------------------------------------------------------- P1 top-2 of 4
def test_p1_top2_exhaustive_alphabet():
    """Every 4-tuple over an alphabet with +-0, ties and a subnormal."""
    alphabet = np.array([0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 0.5, -0.5, 3.0, 2.0 ** -130], np.float32)
    groups = np.array(list(itertools.product(range(len(alphabet)), repeat=4)))
    vals_f = alphabet[groups]                                   # [10000, 4]
    W = f32_to_bf16_bits(vals_f).reshape(-1, 16)                # 2500 rows x 16
    vals, meta, st = oracle.prune24(W)
    assert st == oracle.OK
    codes = codes_of(meta, 16).reshape(-1)
    vflat = vals.reshape(-1, 2)
    for n, grp in enumerate(vals_f):
        i0, i1 = top2_bruteforce(grp)
        assert codes[n] == (i0 | (i1 << 2)), (grp, codes[n])
        bits = f32_to_bf16_bits(grp)
        assert vflat[n, 0] == bits[i0] and vflat[n, 1] == bits[i1]  # copied bit for bit (sign of 0 kept)


def test_p1_all_strict_orderings_with_signs():
    rng = np.random.default_rng(0)
    rows = []
    for perm in itertools.permutations([1.0, 2.0, 3.0, 4.0]):
        for signs in itertools.product([1.0, -1.0], repeat=4):
            rows.append(np.array(perm) * np.array(signs))
    rows = np.array(rows, np.float32)
    rng.shuffle(rows)
    W = f32_to_bf16_bits(rows).reshape(-1, 16)
    vals, meta, st = oracle.prune24(W)
    codes = codes_of(meta, 16).reshape(-1)
    for n, grp in enumerate(rows):
        big = set(np.argsort(-np.abs(grp))[:2].tolist())
        i0, i1 = sorted(big)
        assert codes[n] == (i0 | (i1 << 2))


def test_p1_nonfinite_is_flagged():
    W = rand_bf16((16, 64), 0.02, 3)
    W[5, 17] = 0x7FC0  # NaN
    assert oracle.prune24(W)[2] == oracle.NONFINITE
    W[5, 17] = 0xFF80  # -Inf
    assert oracle.prune24(W)[2] == oracle.NONFINITE


# ---------------------------------------------------------------- P2 W^R structure
@pytest.mark.parametrize("shape", [(64, 512), (48, 96)])
def test_p2_row_mask_structure(shape):
    W = rand_bf16(shape, 0.02, 7)
    vals, meta, st = oracle.prune24(W)
    assert st == oracle.OK
    codes = codes_of(meta, shape[1])
    assert set(np.unique(codes).tolist()) <= LEGAL_CODES
    Wf = oracle.bf16_values(W)
    keep = mask_numpy(Wf)
    dense = oracle.bf16_values(oracle.decompress(vals, meta, shape[1]))
    np.testing.assert_array_equal(dense, np.where(keep, Wf, 0.0))
    # |kept| >= |dropped| inside every group
    g = np.abs(Wf).reshape(shape[0], -1, 4)
    k = keep.reshape(shape[0], -1, 4)
    assert np.all(np.where(k, g, np.inf).min(axis=2) >= np.where(~k, g, -np.inf).max(axis=2))
    assert np.all(k.sum(axis=2) == 2)


# ---------------------------------------------------------------- P3 double prune
def _double_prune_expected(WRf):
    """Dense W^{R,C} from dense W^R by the rule applied down the columns."""
    keep = mask_numpy(WRf.T.copy()).T
    return np.where(keep, WRf, 0.0)


def _dp_dense(W):
    out, in_ = W.shape
    vals, meta, _ = oracle.prune24(W)
    vt, mt = oracle.double_prune(vals, meta, out, in_)
    WR = oracle.bf16_values(oracle.decompress(vals, meta, in_))
    WDP = oracle.bf16_values(oracle.decompress(vt, mt, out)).T
    return WR, WDP, mt


def test_p3_double_prune_random_invariants():
    W = rand_bf16((128, 256), 0.02, 11)
    WR, WDP, mt = _dp_dense(W)
    nz_r, nz_dp = WR != 0, WDP != 0
    assert np.all(nz_r | ~nz_dp)                                   # supp(W_dp) within supp(W^R)
    np.testing.assert_array_equal(WDP[nz_dp], WR[nz_dp])           # equal values there
    assert np.all(nz_dp.reshape(128, -1, 4).sum(2) <= 2)           # <=2 per 4 along in
    assert np.all(nz_dp.T.reshape(256, -1, 4).sum(2) <= 2)         # <=2 per 4 along out
    colcount = nz_r.T.reshape(256, -1, 4).sum(2)                   # per (column, out-group)
    small = np.repeat(colcount <= 2, 4, axis=1).T                  # groups untouched by the 2nd prune
    np.testing.assert_array_equal(WDP[small], WR[small])
    np.testing.assert_array_equal(WDP, _double_prune_expected(WR))
    assert set(np.unique(codes_of(mt, 128)).tolist()) <= LEGAL_CODES


PAIRS = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]


def test_p3_double_prune_exhaustive_4x4_blocks():
    """All 6^4 = 1296 combinations of row patterns of a 4x4 block, with
    distinct non-zero values: 4 block-rows x 324 block-columns of a 16 x 1296
    weight.  Also checks the exact expected density 26/64 of W^{R,C}."""
    rng = np.random.default_rng(5)
    combos = list(itertools.product(range(6), repeat=4))
    Wf = np.zeros((16, 1296), np.float32)
    for n, combo in enumerate(combos):
        br, bc = divmod(n, 324)
        mags = rng.permutation(np.arange(1, 9)).astype(np.float32)  # distinct magnitudes
        signs = rng.choice([-1.0, 1.0], 8).astype(np.float32)
        v = 0
        for j, p in enumerate(combo):
            for c in PAIRS[p]:
                Wf[4 * br + j, 4 * bc + c] = mags[v] * signs[v]
                v += 1
    W = f32_to_bf16_bits(Wf)
    WR, WDP, _ = _dp_dense(W)
    np.testing.assert_array_equal(WR, Wf)  # prune24 keeps exactly the planted pattern
    total_nnz = 0
    for n in range(1296):
        br, bc = divmod(n, 324)
        blk_r = WR[4 * br:4 * br + 4, 4 * bc:4 * bc + 4]
        blk_dp = WDP[4 * br:4 * br + 4, 4 * bc:4 * bc + 4]
        for c in range(4):
            col = blk_r[:, c]
            nz = np.flatnonzero(col)
            if len(nz) <= 2:
                exp = col
            else:
                keep = top2_bruteforce(col)
                exp = np.array([col[j] if j in keep else 0.0 for j in range(4)])
            np.testing.assert_array_equal(blk_dp[:, c], exp)
        total_nnz += int((blk_dp != 0).sum())
    assert Fraction(total_nnz, 1296 * 16) == Fraction(26, 64)


def test_p4_density_closed_form():
    """i.i.d. continuous W: each column out-group of W^R holds Binomial(4, 1/2)
    non-zeros, so W^{R,C} keeps E[min(B,2)]/4 = 26/64 of all positions."""
    W = rand_bf16((512, 512), 0.02, 21)
    _, WDP, _ = _dp_dense(W)
    dens = (WDP != 0).mean()
    # per 4x4 block the density has a spread we bound from the exhaustive
    # enumeration: nnz per block lies in [4, 8] -> sd(block density) <= 1/8
    n_blocks = (512 // 4) * (512 // 4)
    assert abs(dens - 26 / 64) < 5 * (1 / 8) / np.sqrt(n_blocks)


# ---------------------------------------------------------------- P5/P6 GEMMs
def _dense_layer(W):
    Wf = oracle.bf16_values(W)
    WR = np.where(mask_numpy(Wf), Wf, 0.0)
    WDP = _double_prune_expected(WR)
    return WR, WDP


@pytest.mark.parametrize("r", [0, 8, 16, 92])
def test_p5_fwd_bwd_against_numpy_matmul(r):
    T, inn, out = 48, 64, 96
    X = rand_bf16((T, inn), 1.0, 1)
    W = rand_bf16((out, inn), 0.02, 2)
    dY = rand_bf16((T, out), 1e-2, 3)
    L = rand_bf16((inn, r), 0.02, 4) if r else None
    R = rand_bf16((r, out), 0.02, 5) if r else None
    Xf, dYf = oracle.bf16_values(X), oracle.bf16_values(dY)
    WR, WDP = _dense_layer(W)
    vals, meta, _ = oracle.prune24(W)
    vt, mt = oracle.double_prune(vals, meta, out, inn)
    if r:
        Lf, Rf = oracle.bf16_values(L), oracle.bf16_values(R)
        XL_ref = Xf @ Lf
        G_ref = dYf @ Rf.T
    XL = oracle.adapter_fwd(X, L) if r else None
    G = oracle.adapter_g(dY, R) if r else None
    Y = oracle.fwd(X, vals, meta, XL, R, out)
    dX = oracle.bwd_dx(dY, vt, mt, G, L, inn)
    dW = oracle.bwd_dw_masked(dY, X, meta)
    Y_ref = Xf @ WR.T + (XL_ref @ Rf if r else 0.0)
    dX_ref = dYf @ WDP + (G_ref @ Lf.T if r else 0.0)
    keep = mask_numpy(oracle.bf16_values(W))
    dW_ref = (dYf.T @ Xf)[keep].reshape(out, inn // 2)   # row-major order of kept slots
    for got, ref in [(Y, Y_ref), (dX, dX_ref), (dW, dW_ref)]:
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
    if r:
        np.testing.assert_allclose(XL, XL_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(G, G_ref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(oracle.adapter_dr(XL, dY).T, XL_ref.T @ dYf, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(oracle.adapter_dl(X, G), Xf.T @ G_ref, rtol=1e-10, atol=1e-12)


def test_p5_zero_padded_rank_changes_nothing():
    """Rank 92 stored as 96 (extra zero columns of L, zero rows of R): every
    output is exactly the same, and the padded gradient columns are zero."""
    T, inn, out, r, rp = 40, 128, 64, 92, 96
    X = rand_bf16((T, inn), 1.0, 21)
    dY = rand_bf16((T, out), 1e-2, 22)
    W = rand_bf16((out, inn), 0.02, 23)
    L = rand_bf16((inn, r), 0.02, 24)
    R = rand_bf16((r, out), 0.02, 25)
    Lp = np.zeros((inn, rp), np.uint16)
    Lp[:, :r] = L
    Rp = np.zeros((rp, out), np.uint16)
    Rp[:r] = R
    vals, meta, _ = oracle.prune24(W)
    vt, mt = oracle.double_prune(vals, meta, out, inn)
    XL, XLp = oracle.adapter_fwd(X, L), oracle.adapter_fwd(X, Lp)
    G, Gp = oracle.adapter_g(dY, R), oracle.adapter_g(dY, Rp)
    np.testing.assert_array_equal(XLp[:, :r], XL)
    assert not XLp[:, r:].any() and not Gp[:, r:].any()
    np.testing.assert_array_equal(oracle.fwd(X, vals, meta, XLp, Rp, out), oracle.fwd(X, vals, meta, XL, R, out))
    np.testing.assert_array_equal(oracle.bwd_dx(dY, vt, mt, Gp, Lp, inn), oracle.bwd_dx(dY, vt, mt, G, L, inn))
    np.testing.assert_array_equal(oracle.adapter_dl(X, Gp)[:, :r], oracle.adapter_dl(X, G))
    assert not oracle.adapter_dl(X, Gp)[:, r:].any()
    assert not oracle.adapter_dr(XLp, dY)[:, r:].any()


def test_p5_zero_weight_reduces_to_lora_product():
    T, inn, out, r = 32, 64, 64, 16
    X = rand_bf16((T, inn), 1.0, 8)
    W = np.zeros((out, inn), np.uint16)
    L = rand_bf16((inn, r), 0.02, 9)
    R = rand_bf16((r, out), 0.02, 10)
    vals, meta, _ = oracle.prune24(W)
    assert set(np.unique(codes_of(meta, inn)).tolist()) == {0x4}   # all-equal groups keep 0 and 1
    Y = oracle.fwd(X, vals, meta, oracle.adapter_fwd(X, L), R, out)
    ref = (oracle.bf16_values(X) @ oracle.bf16_values(L)) @ oracle.bf16_values(R)
    np.testing.assert_allclose(Y, ref, rtol=1e-10, atol=1e-14)


def test_p6_autograd_when_double_prune_is_identity():
    """With a staggered mask (rows 4q, 4q+1 keep positions 0,1; rows 4q+2, 4q+3
    keep 2,3) every column group of W^R has two non-zeros, the second pruning
    keeps everything, and dX, dW, dL, dR, G must equal fp64 autograd of
    sum(dY * (X W^R^T + X L R))."""
    T, inn, out, r = 40, 64, 64, 8
    Wf = oracle.bf16_values(rand_bf16((out, inn), 0.02, 12)).reshape(out, inn // 4, 4)
    for o in range(out):
        drop = [2, 3] if (o % 4) < 2 else [0, 1]
        Wf[o, :, drop] = 0.0
    Wf = Wf.reshape(out, inn)
    W = f32_to_bf16_bits(Wf.astype(np.float32))
    X = rand_bf16((T, inn), 1.0, 13)
    dY = rand_bf16((T, out), 1e-2, 14)
    L = rand_bf16((inn, r), 0.02, 15)
    R = rand_bf16((r, out), 0.02, 16)
    res = oracle.layer_step(X, W, L, R, dY)
    np.testing.assert_array_equal(oracle.bf16_values(oracle.decompress(res["vals_t"], res["meta_t"], out)).T,
                                  oracle.bf16_values(oracle.decompress(res["vals"], res["meta"], inn)))
    tX = torch.tensor(oracle.bf16_values(X), requires_grad=True)
    tW = torch.tensor(Wf.astype(np.float64), requires_grad=True)
    tL = torch.tensor(oracle.bf16_values(L), requires_grad=True)
    tR = torch.tensor(oracle.bf16_values(R), requires_grad=True)
    tdY = torch.tensor(oracle.bf16_values(dY))
    Y = tX @ tW.T + (tX @ tL) @ tR
    (Y * tdY).sum().backward()
    np.testing.assert_allclose(res["Y"], Y.detach().numpy(), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(res["dX"], tX.grad.numpy(), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(res["dL"], tL.grad.numpy(), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(res["dR"], tR.grad.numpy(), rtol=1e-10, atol=1e-13)
    keep = Wf != 0
    np.testing.assert_allclose(res["dW"], tW.grad.numpy()[keep].reshape(out, inn // 2), rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(res["G"], (tdY @ tR.detach().T).numpy(), rtol=1e-10, atol=1e-13)


def test_p5_row_selection_matches_full():
    T, inn, out, r = 37, 64, 32, 8
    X = rand_bf16((T, inn), 1.0, 31)
    W = rand_bf16((out, inn), 0.02, 32)
    dY = rand_bf16((T, out), 1e-2, 33)
    L = rand_bf16((inn, r), 0.02, 34)
    R = rand_bf16((r, out), 0.02, 35)
    full = oracle.layer_step(X, W, L, R, dY)
    rows = [0, 5, 36]
    XL = oracle.adapter_fwd(X, L, rows)
    np.testing.assert_array_equal(XL, full["XL"][rows])
    np.testing.assert_array_equal(oracle.fwd(X, full["vals"], full["meta"], XL, R, out, rows), full["Y"][rows])
    G = oracle.adapter_g(dY, R, rows)
    np.testing.assert_array_equal(oracle.bwd_dx(dY, full["vals_t"], full["meta_t"], G, L, inn, rows), full["dX"][rows])
    np.testing.assert_array_equal(oracle.bwd_dw_masked(dY, X, full["meta"], [3, 31]), full["dW"][[3, 31]])
    np.testing.assert_array_equal(oracle.adapter_dl(X, full["G"], [2, 60]), full["dL"][[2, 60]])
    np.testing.assert_array_equal(oracle.adapter_dr(full["XL"], dY, [1, 30]), full["dR"][:, [1, 30]].T)


# ---------------------------------------------------------------- P9 memory ratios
def test_p9_memory_ratios_match_printed_values():
    with open(os.path.join(GOLDEN, "memory_ratios.json")) as f:
        gold = json.load(f)
    inf, train = oracle.mem_ratio(**gold["bit_widths"])
    assert inf == gold["inference"]["numerator_bits"] / gold["inference"]["denominator_bits"]
    assert train == gold["training"]["numerator_bits"] / gold["training"]["denominator_bits"]
    assert int(np.floor(100 * inf)) == gold["inference"]["printed_percent"]
    assert int(np.floor(100 * train)) == gold["training"]["printed_percent"]
    # this library's own layout: 4 index bits per group, no byte mask
    inf4, _ = oracle.mem_ratio(b_idx=4)
    assert inf4 == 36 / 64


# ------------------------------------------------------------------ P10: compressed AdamW step
def _bf16_bits_of(x64):
    """float64 array -> bf16 patterns, round to nearest even (via torch)."""
    return torch.from_numpy(np.asarray(x64, np.float64)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32_of_bf16(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def test_p10_adamw_against_torch_optim():
    """One step from arbitrary states against torch.optim.AdamW in fp64: the
    states agree to binary32 rounding, the weight to one bf16 ulp."""
    rng = np.random.default_rng(10)
    n = 4096
    w0 = _bf16_bits_of(rng.normal(0, 0.02, n))
    g = _bf16_bits_of(rng.normal(0, 1e-2, n))
    m0 = rng.normal(0, 1e-3, n).astype(np.float32)
    v0 = (rng.normal(0, 1e-3, n) ** 2).astype(np.float32)
    lr, b1, b2, eps, wd, step = 1e-3, 0.9, 0.999, 1e-8, 0.1, 7
    w1, m1, v1 = oracle.adamw_compressed(w0, g, m0, v0, lr, b1, b2, eps, wd, step)
    p = torch.nn.Parameter(torch.from_numpy(_f32_of_bf16(w0).astype(np.float64)))
    opt = torch.optim.AdamW([p], lr=np.float32(lr).item(), betas=(np.float32(b1).item(), np.float32(b2).item()),
                            eps=np.float32(eps).item(), weight_decay=np.float32(wd).item())
    p.grad = torch.from_numpy(_f32_of_bf16(g).astype(np.float64))
    st = opt.state[p]
    st["step"] = torch.tensor(float(step - 1), dtype=torch.float64)
    st["exp_avg"] = torch.from_numpy(m0.astype(np.float64))
    st["exp_avg_sq"] = torch.from_numpy(v0.astype(np.float64))
    opt.step()
    m_ref, v_ref, w_ref = st["exp_avg"].numpy(), st["exp_avg_sq"].numpy(), p.detach().numpy()
    # binary32 rounding of each term: a few ulps of the larger term (the two
    # terms of m can nearly cancel)
    m_scale = np.abs(0.9 * m0.astype(np.float64)) + np.abs(0.1 * _f32_of_bf16(g))
    v_scale = np.abs(0.999 * v0.astype(np.float64)) + 0.001 * _f32_of_bf16(g).astype(np.float64) ** 2
    assert np.all(np.abs(m1 - m_ref) <= 4 * 2.0 ** -24 * m_scale + 1e-30)
    assert np.all(np.abs(v1 - v_ref) <= 4 * 2.0 ** -24 * v_scale + 1e-30)
    ulp = np.abs(w_ref) * 2.0 ** -7  # a bf16 ulp is at most 2^-7 of the value
    assert np.all(np.abs(_f32_of_bf16(w1).astype(np.float64) - w_ref) <= ulp + 1e-30)
    assert np.mean(w1 != w0) > 0.5  # the step moves most weights by at least one bf16 ulp


def test_p10_adamw_first_step_closed_form():
    """Step 1 from zero states without decay: m = (1-b1) g, v = (1-b2) g^2,
    and the weight moves by lr * g / (|g| + eps), i.e. by about lr * sign(g)."""
    rng = np.random.default_rng(11)
    n = 2048
    w0 = _bf16_bits_of(rng.normal(0, 1.0, n))
    g = _bf16_bits_of(rng.normal(0, 1.0, n))
    z = np.zeros(n, np.float32)
    lr, b1, b2, eps = 1e-2, 0.9, 0.999, 1e-8
    w1, m1, v1 = oracle.adamw_compressed(w0, g, z, z, lr, b1, b2, eps, 0.0, 1)
    gf = _f32_of_bf16(g).astype(np.float64)
    np.testing.assert_allclose(m1, (1 - np.float32(b1)) * gf, rtol=1e-6)
    np.testing.assert_allclose(v1, (1 - np.float32(b2)) * gf * gf, rtol=1e-6)
    expect = _f32_of_bf16(w0).astype(np.float64) - lr * gf / (np.abs(gf) + eps)
    assert np.all(np.abs(_f32_of_bf16(w1) - expect) <= np.abs(expect) * 2.0 ** -8 * 1.01 + 1e-30)


def test_p10_adamw_invariants():
    """No gradient, no decay: the weight stays bit for bit and the states
    decay by exactly b1 and b2; with decay only, w becomes w (1 - lr wd)."""
    rng = np.random.default_rng(12)
    n = 1024
    w0 = _bf16_bits_of(rng.normal(0, 0.02, n))
    zero_g = np.zeros(n, np.uint16)
    m0 = rng.normal(0, 1e-3, n).astype(np.float32)
    v0 = np.abs(rng.normal(0, 1e-3, n)).astype(np.float32)
    w1, m1, v1 = oracle.adamw_compressed(w0, zero_g, m0 * 0, v0 * 0, 1e-3, 0.9, 0.999, 1e-8, 0.0, 3)
    np.testing.assert_array_equal(w1, w0)
    w1, m1, v1 = oracle.adamw_compressed(w0, zero_g, m0, v0, 0.0, 0.9, 0.999, 1e-8, 0.0, 3)
    np.testing.assert_array_equal(w1, w0)
    np.testing.assert_array_equal(m1, np.float32(0.9) * m0)
    np.testing.assert_array_equal(v1, np.float32(0.999) * v0)
    lr, wd = 1e-2, 0.5
    w1, _, _ = oracle.adamw_compressed(w0, zero_g, m0 * 0, v0 * 0, lr, 0.9, 0.999, 1e-8, wd, 1)
    decay = np.float32(1) - np.float32(lr) * np.float32(wd)
    np.testing.assert_array_equal(w1, _bf16_bits_of((_f32_of_bf16(w0) * decay).astype(np.float64)))


# ------------------------------------------------------------------ P11: general N:M pruning
def _nm_by_sort(W, N, M):
    """Independent selection: per group, a stable sort by descending magnitude
    (ties keep index order) picks the first N, reported in index order."""
    rows, K = W.shape
    mag = (W & 0x7FFF).astype(np.int64).reshape(rows, K // M, M)
    order = np.argsort(-mag, axis=2, kind="stable")[:, :, :N]
    pos = np.sort(order, axis=2)
    vals = np.take_along_axis(W.reshape(rows, K // M, M), pos, axis=2)
    return vals.reshape(rows, -1), pos.reshape(rows, -1).astype(np.uint8)


@pytest.mark.parametrize("N,M", [(1, 4), (2, 4), (3, 4), (1, 8), (2, 8), (4, 8), (7, 8), (2, 16), (8, 16)])
def test_p11_nm_matches_stable_sort(N, M):
    rng = np.random.default_rng(N * 100 + M)
    W = I.bits(torch.from_numpy(rng.normal(0, 0.02, (33, 4 * 16)).astype(np.float32)).to(torch.bfloat16))
    W = np.ascontiguousarray(W)
    # plant ties and signed zeros in some groups
    W[0, :M] = 0
    W[1, :M] = 0x8000
    W[2, 0:M:2] = W[2, 1]
    vals, pos, st = oracle.prune_nm(W, N, M)
    assert st == oracle.OK
    v_ref, p_ref = _nm_by_sort(W, N, M)
    np.testing.assert_array_equal(vals, v_ref)
    np.testing.assert_array_equal(pos, p_ref)


def test_p11_nm_structure_and_magnitudes():
    """Exactly N kept per group, strictly increasing positions, and every kept
    magnitude >= every dropped one."""
    rng = np.random.default_rng(3)
    for N, M in [(1, 4), (3, 8), (5, 16)]:
        W = I.bits(torch.from_numpy(rng.normal(0, 1, (16, 128)).astype(np.float32)).to(torch.bfloat16))
        vals, pos, _ = oracle.prune_nm(np.ascontiguousarray(W), N, M)
        G = 128 // M
        p = pos.reshape(16, G, N).astype(np.int64)
        assert np.all(np.diff(p, axis=2) > 0) and p.min() >= 0 and p.max() < M
        mag = (W & 0x7FFF).astype(np.int64).reshape(16, G, M)
        kept = np.zeros_like(mag, dtype=bool)
        np.put_along_axis(kept, p, True, axis=2)
        kmin = np.where(kept, mag, 1 << 20).min(axis=2)
        dmax = np.where(~kept, mag, -1).max(axis=2)
        assert np.all(kmin >= dmax)


def test_p11_two_of_four_equals_prune24():
    """N = 2, M = 4 is the row mask of prune24: same values, and the positions
    are the two fields of each group's code."""
    W = I.bits(I.normal_bf16((48, 256), 0.02, 9, 0, "W"))
    vals, pos, _ = oracle.prune_nm(W, 2, 4)
    v24, m24, _ = oracle.prune24(W)
    np.testing.assert_array_equal(vals, v24)
    codes = np.stack([(m24 >> (4 * q)) & 0xF for q in range(4)], axis=2).reshape(48, -1)  # group g = 4 w + q
    np.testing.assert_array_equal(pos[:, 0::2], codes & 3)
    np.testing.assert_array_equal(pos[:, 1::2], codes >> 2)
