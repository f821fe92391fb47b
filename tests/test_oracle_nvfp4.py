"""Pins for the oracle's NVFP4 functions (pairwise sparse FP4): the OCP E2M1
code table, round-to-nearest-even by exhaustive comparison with the table,
the two-level block scaling's closed-form properties, the pair prune against
the already pinned pairwise 4:8 function, the pair slide's completeness
(every kept pair lands in exactly one window), and the product against a
float64 library matmul of the decoded operands."""
import math

import numpy as np
import pytest

import oracle
from conftest import read_golden

PAIR_PATTERNS = ["2:4", "4:6", "6:8", "8:10"]


def test_e2m1_code_table_matches_ocp():
    for code, val in read_golden("e2m1_ocp.txt"):
        c = int(code, 16)
        assert oracle.e2m1_to_float(c) == float(val)
        assert math.copysign(1.0, oracle.e2m1_to_float(c)) == math.copysign(1.0, float(val))


def test_e2m1_rounds_to_nearest_even_and_saturates():
    table = [(c, oracle.e2m1_to_float(c)) for c in range(16)]
    for x in np.concatenate([np.linspace(-7.5, 7.5, 3001), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0,
                                                           -0.25, -5.0, 100.0, -100.0]]):
        x = float(np.float32(x))
        c = oracle.e2m1_from_float(x)
        v = oracle.e2m1_to_float(c)
        if abs(x) >= 6.0:
            assert v == math.copysign(6.0, x)
            continue
        dist = min(abs(x - t) for _, t in table)
        assert abs(x - v) == dist                       # nearest
        ties = [cc for cc, t in table if abs(x - t) == dist and math.copysign(1, t) == math.copysign(1, x)]
        if len(ties) > 1:                               # tie: the even code (mantissa bit 0)
            assert c % 2 == 0
        assert (c & 8 != 0) == (math.copysign(1.0, x) < 0)   # sign kept, -0 included


def test_nvfp4_block_scaling_closed_forms():
    """Per block: the element of largest magnitude codes to +-6 (the scale is
    within 2^-4 of amax / 6g), every element is within half an E2M1 step of
    its value times the block divisor, and a zero block codes to zeros."""
    rng = np.random.default_rng(11)
    X = (rng.standard_normal((40, 64)) * rng.uniform(0.01, 10, (40, 1))).astype(np.float32)
    X[3] = 0.0
    Xv, Xs, g = oracle.quant_nvfp4(X, "dense", 16)
    K_lp = Xv.shape[1] * 2
    D = oracle.decode_dense_nvfp4(Xv, Xs, K_lp, 16)
    # one global scale for the tensor (the NVFP4 row of the LLM-Compressor
    # compression-schemes page), from the amax of all its elements
    assert g.shape == (1,) and g[0] == np.float32(np.abs(X).max()) / np.float32(2688.0)
    for r in range(40):
        for b in range(4):
            blk = X[r, 16 * b:16 * b + 16].astype(np.float64)
            dq = D[r, 16 * b:16 * b + 16]
            if not blk.any():
                assert not dq.any()
                continue
            i = int(np.argmax(np.abs(blk)))
            s = dq[i] / 6.0 if dq[i] != 0 else 0.0
            assert abs(abs(dq[i]) - 6.0 * abs(s)) < 1e-12 and s != 0
            d = abs(s)                                   # block divisor without g
            for x, y in zip(blk / g[0], dq):
                step = 0.5 if abs(y) <= 2.0 else (1.0 if abs(y) <= 4.0 else 2.0)
                assert abs(x - y / d * d) <= 0.5 * step * d * (1 + 2 ** -3) + 1e-9 or abs(x / d) > 6
    assert not Xv[3].any() and not Xs[3].any()


def test_pair_prune_equals_pinned_pairwise_4of8():
    rng = np.random.default_rng(12)
    W = rng.standard_normal((30, 96)).astype(np.float32)
    ref = oracle.prune_pairwise_4of8(W)                      # element mask, pinned by the 20.8% energy
    pm = oracle.prune_pairs(W, 2, 4)
    np.testing.assert_array_equal(np.repeat(pm, 2, axis=1)[:, :96], ref)


@pytest.mark.parametrize("pat", PAIR_PATTERNS)
def test_pair_slide_is_complete_and_exact(pat):
    """Decoding the compressed weight and folding each window of 4 pairs back
    onto its pairs (window j of pair group g covers pairs g*2Nh + 2j ..
    + 3) gives every kept element exactly once, at a quantised value within
    the FP4 error of the weight, and nothing outside the kept pairs."""
    rng = np.random.default_rng(13)
    K = 150
    keep, group = oracle.pattern(pat)
    Nh = group // 2
    W = rng.standard_normal((9, K)).astype(np.float32)
    Wv, Wm, Ws, g = oracle.compress_weight_nvfp4(W, pat)
    K_lift, K_lp = oracle.fp4_shape(pat, K)
    A = oracle.decode_sparse_nvfp4(Wv, Wm, Ws, K_lp) * g
    assert np.all((A.reshape(9, -1, 8) != 0).reshape(9, -1, 4, 2).any(-1).sum(-1) <= 2)
    back = np.zeros((9, K + 4 * group))
    hits = np.zeros((9, K + 4 * group), dtype=int)
    for w in range(K_lift // 8):
        gi, j = divmod(w, Nh - 1)
        for t in range(8):
            k = 2 * (gi * group + 2 * j) + t
            back[:, k] += A[:, 8 * w + t]
            hits[:, k] += (A[:, 8 * w + t] != 0)
    kept = np.repeat(oracle.prune_pairs(W, keep, group), 2, axis=1)[:, :K].astype(bool)
    assert np.all(hits[:, :K][~kept] == 0) and np.all(hits <= 1)
    assert not back[:, K:].any() and not A[:, K_lift:].any()
    err = np.abs(back[:, :K] - np.where(kept, W, 0))
    # half an E2M1 step: <= 1/4 of the value, or 1/4 of the block divisor
    # (<= amax / 6 (1 + 2^-4)) for values that round to 0 or 0.5
    amax = np.abs(np.where(kept, W, 0)).max(axis=1, keepdims=True)
    assert np.all(err <= np.abs(W) * 0.26 + 0.05 * amax + 1e-9)


@pytest.mark.parametrize("pat", ["dense"] + PAIR_PATTERNS)
def test_lifted_activation_follows_the_pair_window_map(pat):
    rng = np.random.default_rng(14)
    K = 200
    X = rng.standard_normal((6, K)).astype(np.float32)
    keep, group = oracle.pattern(pat)
    block = 16 if pat == "dense" else 32
    Xv, Xs, g = oracle.quant_nvfp4(X, pat, block)
    K_lift, K_lp = oracle.fp4_shape(pat, K)
    D = oracle.decode_dense_nvfp4(Xv, Xs, K_lp, block) * g[0]
    for k in range(K_lp):
        if pat == "dense":
            src = k if k < K else -1
        elif k < K_lift:
            Nh = group // 2
            wi, t = divmod(k, 8)
            gi, j = divmod(wi, Nh - 1)
            src = 2 * (gi * group + 2 * j) + t
            src = src if src < K else -1
        else:
            src = -1
        if src < 0:
            assert not D[:, k].any()
        else:
            amax = np.abs(X).max()
            assert np.all(np.abs(D[:, k] - X[:, src]) <= np.abs(X[:, src]) * 0.26 + 0.05 * amax + 1e-9)


def test_nvfp4_matmul_matches_numpy_float64():
    rng = np.random.default_rng(15)
    Xd = rng.integers(-12, 13, (11, 64)) * 0.5 * rng.choice([0.25, 1.0, 2.0], (11, 64))
    Wd = rng.integers(-12, 13, (7, 64)) * 0.5 * rng.choice([0.125, 1.0, 4.0], (7, 64))
    gx = rng.uniform(0.1, 2, 11).astype(np.float32)
    gw = rng.uniform(0.1, 2, 7).astype(np.float32)
    Y = oracle.matmul_nvfp4(Xd, gx, Wd, gw, oracle.OUT_F32)
    acc = (Xd @ Wd.T).astype(np.float32)
    np.testing.assert_array_equal(Y, (acc * gx[:, None]).astype(np.float32) * gw[None, :])


@pytest.mark.parametrize("pat", PAIR_PATTERNS)
def test_sparse_nvfp4_product_approximates_pruned_matmul(pat):
    rng = np.random.default_rng(16)
    M, N, K = 12, 20, 256
    keep, group = oracle.pattern(pat)
    W = rng.standard_normal((N, K)).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    kept = np.repeat(oracle.prune_pairs(W, keep, group), 2, axis=1)[:, :K].astype(bool)
    ref = X.astype(np.float64) @ np.where(kept, W, 0).T
    Wv, Wm, Ws, g_w = oracle.compress_weight_nvfp4(W, pat)
    Xv, Xs, g_x = oracle.quant_nvfp4(X, pat, 32)
    _, K_lp = oracle.fp4_shape(pat, K)
    Y = oracle.sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp, oracle.OUT_F32)
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    # E2M1 with 16/32-element scales leaves ~10% normwise error per Gaussian
    # operand (measured 0.09-0.10 here); the product carries both
    assert rel < 0.2
    # and the dense comparator on unpruned W approximates X W^T
    Wd_v, Wd_s, gwd = oracle.quant_nvfp4(W, "dense", 16)
    Xd_v, Xd_s, gxd = oracle.quant_nvfp4(X, "dense", 16)
    Yd = oracle.dense_gemm_nvfp4(Xd_v, Xd_s, gxd, Wd_v, Wd_s, gwd[0], oracle.OUT_F32)
    full = X.astype(np.float64) @ W.T.astype(np.float64)
    assert np.linalg.norm(Yd - full) / np.linalg.norm(full) < 0.2


def _src(pat, k, K, K_lift):
    """Source of lifted position k: window i of 4 pairs reads 8 elements from
    2 * (2Nh * (i // (Nh - 1)) + 2 * (i % (Nh - 1))) (the SlideSparse
    write-up's window map, 3.2, on pairs); -1 for padding."""
    if pat == "dense":
        return k if k < K else -1
    if k >= K_lift:
        return -1
    _, group = oracle.pattern(pat)
    wi, t = divmod(k, 8)
    gi, j = divmod(wi, group // 2 - 1)
    src = 2 * (gi * group + 2 * j) + t
    return src if src < K else -1


@pytest.mark.parametrize("pat", ["dense"] + PAIR_PATTERNS)
def test_page_activation_is_the_dense_group16_quantiser_then_the_lift(pat):
    """The NVFP4 definition's activation (16-element groups along the original
    K, one global scale) is the dense 16-block quantiser -- pinned above by
    its closed forms -- followed by the window map: every lifted position
    holds exactly the decoded value of its source element."""
    rng = np.random.default_rng(17)
    K = 512
    X = (rng.standard_normal((5, K)) * rng.uniform(0.1, 4, (5, 1))).astype(np.float32)
    Xl, g = oracle.nvfp4_act_page(X, pat)
    Dv, Ds, gd = oracle.quant_nvfp4(X, "dense", 16)
    D = oracle.decode_dense_nvfp4(Dv, Ds, K, 16)
    assert g[0] == gd[0] == np.float32(np.abs(X).max()) / np.float32(2688.0)
    K_lift, K_lp = oracle.fp4_shape(pat, K)
    assert Xl.shape == (5, K_lp)
    for k in range(K_lp):
        src = _src(pat, k, K, K_lift)
        if src < 0:
            assert not Xl[:, k].any()
        else:
            np.testing.assert_array_equal(Xl[:, k], D[:, src])


def _block_cost(X, W, pat):
    """Normwise errors of the two activation forms against the exact product
    of X with the (common) quantised sparse weight."""
    M, K = X.shape
    N = W.shape[0]
    Wv, Wm, Ws, g_w = oracle.compress_weight_nvfp4(W, pat)
    K_lift, K_lp = oracle.fp4_shape(pat, K)
    Wd = oracle.decode_sparse_nvfp4(Wv, Wm, Ws, K_lp) * np.float64(g_w)
    Xlift = np.zeros((M, K_lp))
    for k in range(K_lp):
        src = _src(pat, k, K, K_lift)
        if src >= 0:
            Xlift[:, k] = X[:, src]
    exact = Xlift @ Wd.T                                   # = X . dequant(prune(W))^T
    Xv, Xs, g_x = oracle.quant_nvfp4(X, pat, 32)
    Y32 = oracle.sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp, oracle.OUT_F32)
    Y16 = oracle.sparse_gemm_nvfp4_page(Wv, Wm, Ws, g_w, X, pat, oracle.OUT_F32)
    nrm = np.linalg.norm(exact)
    return (np.linalg.norm(Y16 - exact) / nrm, np.linalg.norm(Y32 - exact) / nrm,
            np.linalg.norm(Y32 - Y16) / nrm)


@pytest.mark.parametrize("kind", ["gauss", "outlier"])
@pytest.mark.parametrize("pat", ["2:4", "6:8"])
def test_block32_activation_cost_against_the_group16_definition(pat, kind):
    """The sparse FP4 instruction scales the dense operand per 32 lifted K, the
    NVFP4 definition per 16 elements.  Against the exact product with the
    (common) quantised weight, the 32-block activation error stays within 1.4x
    of the definition's on Gaussian activations and with 1% of channels x20.
    Measured here (normwise): 16-block 0.091-0.096, 32-block 0.100 (Gaussian)
    and 0.117-0.121 (outliers: a x20 channel coarsens the scale of 31 other
    elements instead of 15), distance between the two 0.089-0.095.  A
    Gaussian block of 32 has a larger expected maximum than one of 16
    (about 2.4 against 2.1 standard deviations), so its E2M1 steps are ~1.1x
    coarser; that is the Gaussian ratio."""
    rng = np.random.default_rng(18)
    M, N, K = 48, 40, 1024
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    if kind == "outlier":
        X[:, rng.choice(K, K // 100, replace=False)] *= 20.0
    e16, e32, dist = _block_cost(X, W, pat)
    assert 0.0 < e16 < 0.11
    assert e16 <= e32 <= 1.4 * e16
    assert dist < 0.11
