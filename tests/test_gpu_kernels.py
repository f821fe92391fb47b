"""GPU parity of every libss kernel against the CPU oracle on small shapes
that span several tiles and ragged tails.  Bytes (quantised operands,
packed values, metadata, scales) and INT8 results must be bit-exact; FP8
results must be within the relative tolerance of 1e-2."""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_quantized_b200 as ss
from structured_sparse_quantized_b200 import synth
from _helpers import Q, assert_y_matches, dev, host

pytestmark = pytest.mark.gpu

PATTERNS = ["2:4", "4:6", "6:8", "8:10"]
IN_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _x(M, K, dt, seed=1, scale=1.0):
    return synth.gaussian((M, K), std=scale, seed=seed, dtype=IN_DTYPES[dt])


@pytest.mark.parametrize("pat", ["dense"] + PATTERNS)
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 64), (3, 150), (129, 1000), (16, 4100)])
def test_quant_lift_act(pat, q, dt, M, K):
    X = _x(M, K, dt, seed=M + K)
    Xq_ref, s_ref = oracle.quant_lift_act(X, pat, Q[q])
    Xq, s_x = ss.quant_lift_act(dev(X), pat, q)
    np.testing.assert_array_equal(host(s_x), s_ref)
    np.testing.assert_array_equal(host(Xq), Xq_ref)


@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 64), (5, 150), (130, 1030), (7, 4096)])
def test_prune_act_2to4(q, dt, M, K):
    X = _x(M, K, dt, seed=3 * M + K)
    Xv_ref, Xm_ref, s_ref = oracle.prune_act_2to4(X, Q[q])
    Xv, Xm, s_x = ss.prune_act_2to4(dev(X), q)
    np.testing.assert_array_equal(host(s_x), s_ref)
    K_lp = Xv_ref.shape[1] * 2
    np.testing.assert_array_equal(host(Xm), oracle.meta_to_tiles(Xm_ref, K_lp))
    np.testing.assert_array_equal(host(Xv), Xv_ref)


# Many bf16 rows (several CTAs per SM) at the K values of each register-
# resident variant: 1 warp per row with up to 2, 4, 6, 7 and 8 sixteen-element
# chunks per lane, 2 and 4 warps per row (K up to 16384) with 6, 7 and 8; the
# 6:8 in-register lift with and without a zero tail up to K_lp; and a K that
# takes the two-pass kernel.
@pytest.mark.parametrize("pat", ["dense"] + PATTERNS)
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("M,K", [(1200, 16384), (1200, 14336), (1500, 8192), (1500, 5120),
                                 (3000, 4096), (3000, 3584), (3000, 3072), (3000, 2048),
                                 (3000, 1040), (3000, 1032), (3000, 512)])
def test_quant_lift_act_many_rows(pat, q, M, K):
    X = _x(M, K, "bf16", seed=K)
    Xq_ref, s_ref = oracle.quant_lift_act(X, pat, Q[q])
    Xq, s_x = ss.quant_lift_act(dev(X), pat, q)
    np.testing.assert_array_equal(host(s_x), s_ref)
    np.testing.assert_array_equal(host(Xq), Xq_ref)


@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("M,K", [(5000, 4096), (3001, 4000), (3001, 2056), (700, 1024)])
def test_prune_act_2to4_many_rows(q, M, K):
    X = synth.gaussian_with_heavy_tails(M, K, seed=M)
    Xv_ref, Xm_ref, s_ref = oracle.prune_act_2to4(X, Q[q])
    Xv, Xm, s_x = ss.prune_act_2to4(dev(X), q)
    np.testing.assert_array_equal(host(s_x), s_ref)
    np.testing.assert_array_equal(host(Xm), oracle.meta_to_tiles(Xm_ref, Xv_ref.shape[1] * 2))
    np.testing.assert_array_equal(host(Xv), Xv_ref)


# The single-pass prune kernel (bf16 rows, chunks of up to 4096 elements per
# warp).  Chunks that fill whole steps per lane with no padding (the
# bounds-free form): K = 2048 (2 steps per lane), 4096, 8192 and 16384 (4
# steps, 1, 2 and 4 warps per row).  The bounds-checked form: K = 96 and 160
# (zero-filled padding steps up to K_lp), 1024, 2080, 4032 (padding steps in
# the last step), 6208 and 8320 (2 and 4 warps per row), 8128 (a fifth step
# for the last warp's padding) and 14336.  K = 32768 takes the two-pass kernel.
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("M,K", [(300, 96), (257, 160), (2000, 1024), (1000, 2048), (1000, 2080),
                                 (3000, 4096), (400, 4032), (600, 6208), (300, 8128),
                                 (1000, 8192), (300, 8320), (700, 14336), (600, 16384),
                                 (200, 32768)])
def test_prune_act_2to4_register_rows(q, M, K):
    X = synth.gaussian_with_heavy_tails(M, K, seed=K + 1)
    Xv_ref, Xm_ref, s_ref = oracle.prune_act_2to4(X, Q[q])
    Xv, Xm, s_x = ss.prune_act_2to4(dev(X), q)
    np.testing.assert_array_equal(host(s_x), s_ref)
    np.testing.assert_array_equal(host(Xm), oracle.meta_to_tiles(Xm_ref, Xv_ref.shape[1] * 2))
    np.testing.assert_array_equal(host(Xv), Xv_ref)


@pytest.mark.parametrize("pat", ["dense"] + PATTERNS)
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("N,K", [(1, 64), (64, 150), (130, 1000)])
def test_compress_weight(pat, q, dt, N, K):
    W = _x(N, K, dt, seed=N * 7 + K, scale=0.02)
    Wv_ref, Wm_ref, s_ref = oracle.compress_weight(W, pat, Q[q])
    Wv, Wm, s_w = ss.compress_weight(dev(W), pat, q)
    np.testing.assert_array_equal(host(s_w), s_ref)
    np.testing.assert_array_equal(host(Wv), Wv_ref)
    if pat != "dense":
        np.testing.assert_array_equal(host(Wm), oracle.meta_to_tiles(Wm_ref, Wv_ref.shape[1] * 2))
    assert ss.ss_get_device_status() == ss.SS_OK


def test_compress_weight_with_ties_and_zeros():
    """Exact ties, zero groups and a zero row exercise the tie rule, the
    padding of windows with fewer than two owners, and the zero scale."""
    W = torch.tensor(np.random.default_rng(0).integers(-3, 4, (40, 96)), dtype=torch.float32)
    W[5] = 0.0
    for pat in PATTERNS:
        for q in ["int8", "fp8"]:
            Wv_ref, Wm_ref, s_ref = oracle.compress_weight(W, pat, Q[q])
            Wv, Wm, s_w = ss.compress_weight(dev(W), pat, q)
            np.testing.assert_array_equal(host(s_w), s_ref)
            np.testing.assert_array_equal(host(Wv), Wv_ref)
            np.testing.assert_array_equal(host(Wm),
                                          oracle.meta_to_tiles(Wm_ref, Wv_ref.shape[1] * 2))


@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_prune_act_ties_and_zeros(q):
    """Small integers as bf16: exact ties inside most groups of 4 (the lower
    index wins), all-zero groups, a zero row and -0.0 against +0.0."""
    rng = np.random.default_rng(11)
    X = torch.tensor(rng.integers(-3, 4, (300, 512)), dtype=torch.float32)
    X[7] = 0.0
    X[9, ::3] = -0.0
    X = X.to(torch.bfloat16)
    Xv_ref, Xm_ref, s_ref = oracle.prune_act_2to4(X, Q[q])
    Xv, Xm, s_x = ss.prune_act_2to4(dev(X), q)
    np.testing.assert_array_equal(host(s_x), s_ref)
    np.testing.assert_array_equal(host(Xm), oracle.meta_to_tiles(Xm_ref, Xv_ref.shape[1] * 2))
    np.testing.assert_array_equal(host(Xv), Xv_ref)


def test_nan_weight_reports_data_error():
    W = torch.randn(8, 64)
    W[3, 10] = float("nan")
    ss.compress_weight(dev(W), "6:8", "int8")
    assert ss.ss_get_device_status() == ss.SS_ERR_DATA
    assert ss.ss_get_device_status() == ss.SS_OK        # cleared by the read


# ---------------------------------------------------------------- GEMMs

GEMM_CASES = [  # M, N, K, pattern
    (16, 64, 64, "6:8"),        # the single-linear workload shape
    (1, 130, 300, "2:4"),       # one token, ragged channel tile
    (37, 257, 1000, "4:6"),     # ragged both ways, K not a multiple of 6
    (300, 200, 600, "8:10"),    # two token tiles
    (500, 384, 2048, "6:8"),    # three token tiles, 24 K stages
]


@pytest.mark.parametrize("M,N,K,pat", GEMM_CASES)
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_sparse_gemm_weight_sparse(M, N, K, pat, q, out):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wv, Wm, s_w = oracle.compress_weight(W, pat, Q[q])
    Xq, s_x = oracle.quant_lift_act(X, pat, Q[q])
    _, _, K_lp = oracle.slide_shape(pat, K)
    ob = out == "bf16"
    Y_ref = oracle.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, M, N, K_lp, Q[q],
                               oracle.OUT_BF16 if ob else oracle.OUT_F32)
    Y = ss.sparse_gemm(0, dev(Wv), dev(oracle.meta_to_tiles(Wm, K_lp)), dev(s_w), dev(Xq),
                       dev(s_x), M, N, q, out_dtype=torch.bfloat16 if ob else torch.float32)
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(host(Y), Y_ref, q, ob)


# Shapes run by both sparse kernel shapes (pinned with SS_SPARSE_KERNEL): the
# two-B-tile one (single-buffered accumulators, collector-reused A) and the
# one-B-tile one.  Several tiles per CTA pair, ragged channels and tokens, odd
# stage counts and the narrower B tiles the wave balancing picks.
WIDE_CASES = [  # M, N, K, pattern, sampled token rows (None = all)
    (1000, 520, 1024, "2:4", None),    # ragged both ways, 8 stages
    (2000, 300, 768, "6:8", None),     # 9 stages (odd against the 5-stage ring)
    (4500, 1100, 640, "4:6", None),    # 192-token B tiles, ragged channel tile
    (8192, 2048, 256, "2:4", 384),     # 160-token B tiles, 3 tiles per pair
    (3000, 4096, 512, "8:10", 256),    # 16 channel tiles, 2 tiles per pair
    (8192, 14336, 128, "2:4", 256),    # full 224-token B tiles, one stage, 15 waves
]


@pytest.mark.parametrize("M,N,K,pat,nrows", WIDE_CASES)
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("kernel", ["wide", "narrow"])
def test_sparse_gemm_wide_tiles(M, N, K, pat, nrows, q, kernel, monkeypatch):
    monkeypatch.setenv("SS_SPARSE_KERNEL", kernel)
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wv, Wm, s_w = oracle.compress_weight(W, pat, Q[q])
    Xq, s_x = oracle.quant_lift_act(X, pat, Q[q])
    _, _, K_lp = oracle.slide_shape(pat, K)
    rows = None if nrows is None else synth.sample_rows(M, seed=5, middle=nrows)
    Y_ref = oracle.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, M, N, K_lp, Q[q], oracle.OUT_BF16,
                               m_idx=rows)
    Y = host(ss.sparse_gemm(0, dev(Wv), dev(oracle.meta_to_tiles(Wm, K_lp)), dev(s_w), dev(Xq),
                            dev(s_x), M, N, q))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y if rows is None else Y[rows], Y_ref, q, True)


# Activation-sparse shapes (A = pruned X, token rows) on both kernel shapes.
@pytest.mark.parametrize("M,N,K", [(1000, 520, 1024), (300, 2000, 768), (2049, 4096, 512),
                                   (8192, 1400, 256)])
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("kernel", ["wide", "narrow"])
def test_sparse_gemm_activation_sparse_tiles(M, N, K, q, kernel, monkeypatch):
    monkeypatch.setenv("SS_SPARSE_KERNEL", kernel)
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian_with_heavy_tails(M, K, seed=1)
    Xv, Xm, s_x = oracle.prune_act_2to4(X, Q[q])
    Wq, _, s_w = oracle.compress_weight(W, "dense", Q[q])
    K_lp = oracle.act_2to4_k_lp(K)
    rows = synth.sample_rows(M, seed=3, middle=200)
    Y_ref = oracle.sparse_gemm(1, Xv, Xm, s_x, Wq, s_w, M, N, K_lp, Q[q], oracle.OUT_BF16,
                               m_idx=rows)
    Y = host(ss.sparse_gemm(1, dev(Xv), dev(oracle.meta_to_tiles(Xm, K_lp)), dev(s_x), dev(Wq),
                            dev(s_w), M, N, q))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y[rows], Y_ref, q, True)


@pytest.mark.parametrize("M,N,K", [(130, 64, 256), (257, 300, 1024), (8, 96, 4096)])
@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_sparse_gemm_activation_sparse(M, N, K, q):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian_with_heavy_tails(M, K, seed=1)
    Xv, Xm, s_x = oracle.prune_act_2to4(X, Q[q])
    Wq, _, s_w = oracle.compress_weight(W, "dense", Q[q])
    K_lp = oracle.act_2to4_k_lp(K)
    assert Wq.shape[1] == K_lp
    Y_ref = oracle.sparse_gemm(1, Xv, Xm, s_x, Wq, s_w, M, N, K_lp, Q[q], oracle.OUT_BF16)
    Y = ss.sparse_gemm(1, dev(Xv), dev(oracle.meta_to_tiles(Xm, K_lp)), dev(s_x), dev(Wq),
                       dev(s_w), M, N, q)
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(host(Y), Y_ref, q, True)


@pytest.mark.parametrize("M,N,K", [(16, 64, 64), (1, 130, 300), (300, 257, 1000), (600, 128, 512)])
@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_dense_gemm(M, N, K, q):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wq, _, s_w = oracle.compress_weight(W, "dense", Q[q])
    Xq, s_x = oracle.quant_lift_act(X, "dense", Q[q])
    Y_ref = oracle.dense_gemm(Xq, s_x, Wq, s_w, Q[q], oracle.OUT_BF16)
    Y = ss.dense_gemm(dev(Xq), dev(s_x), dev(Wq), dev(s_w), q)
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(host(Y), Y_ref, q, True)


@pytest.mark.parametrize("pat", PATTERNS)
@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_chained_gpu_path_matches_plain_definition(pat, q):
    """GPU compress -> GPU quant+lift -> GPU sparse GEMM equals the oracle's
    plain path (prune, quantise, naive matmul over the original K): the
    lossless-decomposition identity, end to end on the device."""
    M, N, K = 70, 200, 333
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    plain = oracle.plain_linear(W, X, pat, Q[q], oracle.OUT_BF16)
    Y = ss.linear(dev(X), ss.compress_weight(dev(W), pat, q), pat, q)
    assert_y_matches(host(Y), plain, q, True)


def test_zero_rows_and_channels():
    M, N, K = 20, 140, 256
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    W[7] = 0
    X[3] = 0
    for q in ["int8", "fp8"]:
        packed = ss.compress_weight(dev(W), "6:8", q)
        Y = host(ss.linear(dev(X), packed, "6:8", q)).view(np.uint16)
        assert np.all(Y[3] == 0) and np.all(Y[:, 7] == 0)
        plain = oracle.plain_linear(W, X, "6:8", Q[q], oracle.OUT_BF16)
        assert_y_matches(Y, plain, q, True)


def test_launch_counter_and_status():
    before = ss.ss_kernel_launches()
    X = synth.gaussian((4, 64), seed=2, dtype=torch.bfloat16)
    ss.quant_lift_act(dev(X), "6:8", "int8")
    assert ss.ss_kernel_launches() == before + 1
    assert ss.ss_get_device_status() == ss.SS_OK
