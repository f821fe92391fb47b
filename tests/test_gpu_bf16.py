"""GPU parity of the bf16 tier (2:4 and the sliding patterns with bf16
operands, kind::f16 on the sparse tensor cores) against the CPU oracle.
Stored values (bf16 bits), metadata and the lift are bit-exact; GEMM results
are within the relative tolerance BF16_TOL (fp32 accumulation order)."""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_quantized_b200 as ss
from structured_sparse_quantized_b200 import synth
from _helpers import assert_y_matches, dev, host

pytestmark = pytest.mark.gpu

PATTERNS = ["2:4", "4:6", "6:8", "8:10"]
IN_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _x(M, K, dt, seed=1, scale=1.0):
    return synth.gaussian((M, K), std=scale, seed=seed, dtype=IN_DTYPES[dt])


def _bf(a: np.ndarray) -> torch.Tensor:
    """bf16 bits (uint16) -> bf16 CUDA tensor."""
    return dev(torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16))


def _tiles(Am: np.ndarray, K_lp: int) -> torch.Tensor:
    """Row-layout selectors -> the bf16 tier's device storage."""
    return dev(oracle.meta_to_tiles(Am, K_lp, i16=True))


@pytest.mark.parametrize("pat", ["dense"] + PATTERNS)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 64), (3, 151), (129, 1000), (16, 4100), (700, 4096)])
def test_lift_bf16(pat, dt, M, K):
    X = _x(M, K, dt, seed=M + K)
    ref = oracle.lift_act_bf16(X, pat)
    Xl, s_x = ss.quant_lift_act(dev(X), pat, "bf16")
    assert s_x is None and Xl.dtype == torch.bfloat16
    np.testing.assert_array_equal(host(Xl), ref)


@pytest.mark.parametrize("pat", ["dense"] + PATTERNS)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("N,K", [(1, 64), (64, 150), (130, 1000)])
def test_compress_weight_bf16(pat, dt, N, K):
    W = _x(N, K, dt, seed=N + 2 * K, scale=0.02)
    Wv_ref, Wm_ref = oracle.compress_weight_bf16(W, pat)
    Wv, Wm, s_w = ss.compress_weight(dev(W), pat, "bf16")
    assert s_w is None
    assert ss.ss_get_device_status() == ss.SS_OK
    np.testing.assert_array_equal(host(Wv), Wv_ref)
    if pat != "dense":
        _, _, K_lp = oracle.slide_shape(pat, K)
        np.testing.assert_array_equal(host(Wm), oracle.meta_to_tiles(Wm_ref, K_lp, i16=True))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 64), (5, 150), (130, 1030), (300, 4096)])
def test_prune_act_2to4_bf16(dt, M, K):
    X = _x(M, K, dt, seed=3 * M + K)
    Xv_ref, Xm_ref = oracle.prune_act_2to4_bf16(X)
    Xv, Xm, s_x = ss.prune_act_2to4(dev(X), "bf16")
    assert s_x is None
    K_lp = Xv_ref.shape[1] * 2
    np.testing.assert_array_equal(host(Xm), oracle.meta_to_tiles(Xm_ref, K_lp, i16=True))
    np.testing.assert_array_equal(host(Xv), Xv_ref)


def test_prune_act_bf16_ties_and_zeros():
    """Equal magnitudes keep the lower index; all-zero groups keep 0 and 1."""
    X = torch.tensor([[1.0, -1.0, 1.0, -1.0] * 32,
                      [0.0, 0.0, 0.0, 0.0] * 32,
                      [0.0, 2.0, -2.0, 0.5] * 32], dtype=torch.bfloat16)
    Xv_ref, Xm_ref = oracle.prune_act_2to4_bf16(X)
    Xv, Xm, _ = ss.prune_act_2to4(dev(X), "bf16")
    np.testing.assert_array_equal(host(Xm), oracle.meta_to_tiles(Xm_ref, 128, i16=True))
    np.testing.assert_array_equal(host(Xv), Xv_ref)


GEMM_CASES = [  # M, N, K, pattern
    (16, 64, 64, "6:8"),
    (1, 130, 300, "2:4"),
    (37, 257, 1000, "4:6"),
    (300, 200, 600, "8:10"),
    (500, 384, 2048, "6:8"),     # three token tiles, 24 K stages
]


@pytest.mark.parametrize("M,N,K,pat", GEMM_CASES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_sparse_gemm_bf16_weight_sparse(M, N, K, pat, out):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wv, Wm = oracle.compress_weight_bf16(W, pat)
    Xl = oracle.lift_act_bf16(X, pat)
    _, _, K_lp = oracle.slide_shape(pat, K)
    ob = out == "bf16"
    Y_ref = oracle.sparse_gemm_bf16(0, Wv, Wm, Xl, M, N, K_lp,
                                    oracle.OUT_BF16 if ob else oracle.OUT_F32)
    Y = ss.sparse_gemm(0, _bf(Wv), _tiles(Wm, K_lp), None, _bf(Xl), None, M, N, "bf16",
                       out_dtype=torch.bfloat16 if ob else torch.float32)
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(host(Y), Y_ref, "bf16", ob)


@pytest.mark.parametrize("M,N,K,pat,nrows", [
    (2000, 1100, 1024, "6:8", 256),   # 5 channel tiles x 9 token tiles
    (4096, 4096, 512, "2:4", 256),    # several tiles per CTA pair
])
def test_sparse_gemm_bf16_many_tiles(M, N, K, pat, nrows):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wv, Wm = oracle.compress_weight_bf16(W, pat)
    Xl = oracle.lift_act_bf16(X, pat)
    _, _, K_lp = oracle.slide_shape(pat, K)
    rows = synth.sample_rows(M, seed=5, middle=nrows)
    Y_ref = oracle.sparse_gemm_bf16(0, Wv, Wm, Xl, M, N, K_lp, oracle.OUT_BF16, m_idx=rows)
    Y = host(ss.sparse_gemm(0, _bf(Wv), _tiles(Wm, K_lp), None, _bf(Xl), None, M, N, "bf16"))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y[rows], Y_ref, "bf16", True)


@pytest.mark.parametrize("M,N,K", [(130, 64, 256), (257, 300, 1024), (8, 96, 4096),
                                   (2049, 1400, 512)])
def test_sparse_gemm_bf16_activation_sparse(M, N, K):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian_with_heavy_tails(M, K, seed=1)
    Xv, Xm = oracle.prune_act_2to4_bf16(X)
    Wb, _ = oracle.compress_weight_bf16(W, "dense")
    K_lp = oracle.act_2to4_k_lp(K)
    assert Wb.shape[1] == K_lp
    rows = synth.sample_rows(M, seed=3, middle=200) if M > 1000 else None
    Y_ref = oracle.sparse_gemm_bf16(1, Xv, Xm, Wb, M, N, K_lp, oracle.OUT_BF16, m_idx=rows)
    Y = host(ss.sparse_gemm(1, _bf(Xv), _tiles(Xm, K_lp), None, _bf(Wb), None, M, N, "bf16"))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y if rows is None else Y[rows], Y_ref, "bf16", True)


@pytest.mark.parametrize("M,N,K", [(16, 64, 64), (1, 130, 300), (300, 257, 1000),
                                   (600, 128, 512), (1000, 2000, 768)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_dense_gemm_bf16(M, N, K, out):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wb, _ = oracle.compress_weight_bf16(W, "dense")
    Xb = oracle.lift_act_bf16(X, "dense")
    ob = out == "bf16"
    rows = synth.sample_rows(M, seed=2, middle=200) if M > 600 else None
    Y_ref = oracle.matmul_bf16(Xb, Wb, oracle.OUT_BF16 if ob else oracle.OUT_F32, m_idx=rows)
    Y = host(ss.dense_gemm(_bf(Xb), None, _bf(Wb), None, "bf16",
                           out_dtype=torch.bfloat16 if ob else torch.float32))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y if rows is None else Y[rows], Y_ref, "bf16", ob)


@pytest.mark.parametrize("pat", ["dense"] + PATTERNS)
def test_chained_bf16_path_matches_plain_definition(pat):
    """GPU compress -> GPU lift -> GPU sparse GEMM (bf16 tier) against the
    oracle's plain path: prune, round to bf16, naive matmul over K."""
    M, N, K = 70, 200, 333
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    plain = oracle.plain_linear_bf16(W, X, pat, oracle.OUT_BF16)
    Y = ss.linear(dev(X), ss.compress_weight(dev(W), pat, "bf16"), pat, "bf16")
    assert_y_matches(host(Y), plain, "bf16", True)
