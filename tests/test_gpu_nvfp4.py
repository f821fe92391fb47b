"""GPU parity of the NVFP4 path (pairwise sparse FP4 on kind::mxf4nvf4)
against the CPU oracle: packed E2M1 codes, pair metadata, UE4M3 scales and
global scales bit-exact; GEMM results within 1e-2 relative (fp32
tensor-core accumulation of the same quantised operands)."""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_quantized_b200 as ss
from structured_sparse_quantized_b200 import synth
from _helpers import assert_y_matches, dev, host

pytestmark = pytest.mark.gpu

PAIR_PATTERNS = ["2:4", "4:6", "6:8", "8:10"]
IN_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _x(M, K, dt, seed=1, scale=1.0):
    return synth.gaussian((M, K), std=scale, seed=seed, dtype=IN_DTYPES[dt])


@pytest.mark.parametrize("pat", ["dense"] + PAIR_PATTERNS)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("N,K", [(1, 64), (64, 150), (130, 1000), (300, 4096)])
def test_compress_weight_nvfp4(pat, dt, N, K):
    W = _x(N, K, dt, seed=N + K, scale=0.02)
    Wv, Wm, Ws, g_w = ss.compress_weight_nvfp4(dev(W), pat)
    assert ss.ss_get_device_status() == ss.SS_OK
    _, K_lp = oracle.fp4_shape(pat, K)
    if pat == "dense":
        Wv_ref, Ws_ref, g_ref = oracle.quant_nvfp4(W, "dense", 16)
        g_ref = g_ref[0]
        block = 16
    else:
        Wv_ref, Wm_ref, Ws_ref, g_ref = oracle.compress_weight_nvfp4(W, pat)
        np.testing.assert_array_equal(host(Wm), oracle.meta_to_tiles(Wm_ref, K_lp // 2))
        block = 32
    assert host(g_w)[0] == np.float32(g_ref)
    np.testing.assert_array_equal(host(Wv), Wv_ref)
    np.testing.assert_array_equal(host(Ws), oracle.scales_to_tiles(Ws_ref, K_lp, block))


@pytest.mark.parametrize("pat", ["dense"] + PAIR_PATTERNS)
@pytest.mark.parametrize("block", [16, 32])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 64), (3, 151), (129, 1000), (300, 4096)])
def test_quant_lift_act_nvfp4(pat, block, dt, M, K):
    X = _x(M, K, dt, seed=3 * M + K)
    Xv, Xs, g_x = ss.quant_lift_act_nvfp4(dev(X), pat, block)
    Xv_ref, Xs_ref, g_ref = oracle.quant_nvfp4(X, pat, block)
    _, K_lp = oracle.fp4_shape(pat, K)
    assert host(g_x)[0] == g_ref[0]
    np.testing.assert_array_equal(host(Xv), Xv_ref)
    np.testing.assert_array_equal(host(Xs), oracle.scales_to_tiles(Xs_ref, K_lp, block))


def test_quant_nvfp4_zero_rows_and_negative_zero():
    """All-zero rows give zero scales and codes; a negative value that rounds
    to zero keeps its sign (-0 = code 8) on both sides."""
    X = torch.zeros((4, 64), dtype=torch.float32)
    X[1, 0] = 1.0
    X[1, 1] = -1e-3
    X[2, 5] = -0.0
    Xv, Xs, g_x = ss.quant_lift_act_nvfp4(dev(X), "dense", 16)
    Xv_ref, Xs_ref, g_ref = oracle.quant_nvfp4(X, "dense", 16)
    assert host(g_x)[0] == g_ref[0]
    np.testing.assert_array_equal(host(Xv), Xv_ref)
    np.testing.assert_array_equal(host(Xs), oracle.scales_to_tiles(Xs_ref, 256, 16))


def test_quant_nvfp4_all_zero_tensor():
    """An all-zero activation has amax 0: g = 0, every scale and code 0."""
    X = torch.zeros((130, 96), dtype=torch.bfloat16)
    for pat, block in (("dense", 16), ("6:8", 32)):
        Xv, Xs, g_x = ss.quant_lift_act_nvfp4(dev(X), pat, block)
        assert ss.ss_get_device_status() == ss.SS_OK
        assert host(g_x)[0] == 0.0 and not host(Xv).any() and not host(Xs).any()


@pytest.mark.parametrize("pat,block", [("dense", 16), ("2:4", 32), ("6:8", 32)])
def test_quant_nvfp4_global_scale_is_per_tensor(pat, block):
    """One global scale for the whole activation (the NVFP4 definition), taken
    from its amax: with 1% of channels x20 the outlier rows set g for every
    row, and two calls in a row on different tensors each reduce their own
    (the accumulator restarts at zero)."""
    X = synth.gaussian_with_outliers(300, 1024, seed=4, dtype=torch.bfloat16)
    X_small = (X.float() * 0.125).to(torch.bfloat16)
    for x in (X, X_small):
        Xv, Xs, g_x = ss.quant_lift_act_nvfp4(dev(x), pat, block)
        Xv_ref, Xs_ref, g_ref = oracle.quant_nvfp4(x, pat, block)
        _, K_lp = oracle.fp4_shape(pat, 1024)
        assert host(g_x)[0] == g_ref[0] == np.float32(x.float().abs().max().item()) / np.float32(2688)
        np.testing.assert_array_equal(host(Xv), Xv_ref)
        np.testing.assert_array_equal(host(Xs), oracle.scales_to_tiles(Xs_ref, K_lp, block))


GEMM_CASES = [  # M, N, K, pattern (pairs)
    (16, 64, 64, "2:4"),
    (1, 130, 300, "2:4"),
    (37, 257, 1000, "4:6"),
    (300, 200, 600, "8:10"),
    (500, 384, 2048, "6:8"),
]


def _sparse_operands(M, N, K, pat):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wv, Wm, Ws, g_w = oracle.compress_weight_nvfp4(W, pat)
    Xv, Xs, g_x = oracle.quant_nvfp4(X, pat, 32)
    _, K_lp = oracle.fp4_shape(pat, K)
    return Wv, Wm, Ws, g_w, Xv, Xs, g_x, K_lp


@pytest.mark.parametrize("M,N,K,pat", GEMM_CASES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_sparse_gemm_nvfp4(M, N, K, pat, out):
    Wv, Wm, Ws, g_w, Xv, Xs, g_x, K_lp = _sparse_operands(M, N, K, pat)
    ob = out == "bf16"
    Y_ref = oracle.sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp,
                                     oracle.OUT_BF16 if ob else oracle.OUT_F32)
    packed = (dev(Wv), dev(oracle.meta_to_tiles(Wm, K_lp // 2)),
              dev(oracle.scales_to_tiles(Ws, K_lp, 32)),
              dev(np.array([g_w, 0, 0, 0], dtype=np.float32)))
    act = (dev(Xv), dev(oracle.scales_to_tiles(Xs, K_lp, 32)), dev(g_x))
    Y = ss.sparse_gemm_nvfp4(packed, act, M, N, out_dtype=torch.bfloat16 if ob else torch.float32)
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(host(Y), Y_ref, "fp8", ob)


@pytest.mark.parametrize("M,N,K,pat,nrows", [(2000, 1100, 1024, "6:8", 256),
                                             (4096, 4096, 512, "2:4", 256)])
def test_sparse_gemm_nvfp4_many_tiles(M, N, K, pat, nrows):
    Wv, Wm, Ws, g_w, Xv, Xs, g_x, K_lp = _sparse_operands(M, N, K, pat)
    rows = synth.sample_rows(M, seed=5, middle=nrows)
    Y_ref = oracle.sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp, oracle.OUT_BF16,
                                     m_idx=rows)
    packed = (dev(Wv), dev(oracle.meta_to_tiles(Wm, K_lp // 2)),
              dev(oracle.scales_to_tiles(Ws, K_lp, 32)),
              dev(np.array([g_w, 0, 0, 0], dtype=np.float32)))
    act = (dev(Xv), dev(oracle.scales_to_tiles(Xs, K_lp, 32)), dev(g_x))
    Y = host(ss.sparse_gemm_nvfp4(packed, act, M, N))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y[rows], Y_ref, "fp8", True)


# Sparse CTA-pair tiles (more than 128 weight rows and K_lp > 2048): M = 256
# MMAs over 256-token B tiles with two scale tiles each, ragged in M, N and K.
@pytest.mark.parametrize("M,N,K,pat", [(700, 520, 4096, "2:4"), (300, 300, 3000, "6:8"),
                                       (2100, 1000, 2560, "4:6"), (33, 4096, 4096, "8:10")])
def test_sparse_gemm_nvfp4_pair_tiles(M, N, K, pat):
    Wv, Wm, Ws, g_w, Xv, Xs, g_x, K_lp = _sparse_operands(M, N, K, pat)
    assert K_lp > 2048 and N > 128
    rows = synth.sample_rows(M, seed=6, middle=200) if M > 600 else None
    Y_ref = oracle.sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp, oracle.OUT_BF16,
                                     m_idx=rows)
    packed = (dev(Wv), dev(oracle.meta_to_tiles(Wm, K_lp // 2)),
              dev(oracle.scales_to_tiles(Ws, K_lp, 32)),
              dev(np.array([g_w, 0, 0, 0], dtype=np.float32)))
    act = (dev(Xv), dev(oracle.scales_to_tiles(Xs, K_lp, 32)), dev(g_x))
    Y = host(ss.sparse_gemm_nvfp4(packed, act, M, N))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y if rows is None else Y[rows], Y_ref, "fp8", True)


@pytest.mark.parametrize("M,N,K", [(16, 64, 64), (1, 130, 300), (300, 257, 1000),
                                   (1000, 2000, 768)])
def test_dense_gemm_nvfp4(M, N, K):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wv, Ws, g_w = oracle.quant_nvfp4(W, "dense", 16)
    Xv, Xs, g_x = oracle.quant_nvfp4(X, "dense", 16)
    _, K_p = oracle.fp4_shape("dense", K)
    rows = synth.sample_rows(M, seed=2, middle=200) if M > 600 else None
    Y_ref = oracle.dense_gemm_nvfp4(Xv, Xs, g_x, Wv, Ws, g_w[0], oracle.OUT_BF16, m_idx=rows)
    packed = (dev(Wv), None, dev(oracle.scales_to_tiles(Ws, K_p, 16)),
              dev(np.array([g_w[0], 0, 0, 0], dtype=np.float32)))
    act = (dev(Xv), dev(oracle.scales_to_tiles(Xs, K_p, 16)), dev(g_x))
    Y = host(ss.dense_gemm_nvfp4(act, packed, M, N))
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(Y if rows is None else Y[rows], Y_ref, "fp8", True)


@pytest.mark.parametrize("pat", ["dense"] + PAIR_PATTERNS)
def test_chained_nvfp4_path(pat):
    """GPU compress -> GPU quant + lift -> GPU GEMM against the oracle's chain
    on the same inputs."""
    M, N, K = 70, 200, 333
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    _, K_lp = oracle.fp4_shape(pat, K)
    if pat == "dense":
        Wv, Ws, g_w = oracle.quant_nvfp4(W, "dense", 16)
        Xv, Xs, g_x = oracle.quant_nvfp4(X, "dense", 16)
        ref = oracle.dense_gemm_nvfp4(Xv, Xs, g_x, Wv, Ws, g_w[0], oracle.OUT_BF16)
    else:
        Wv, Wm, Ws, g_w = oracle.compress_weight_nvfp4(W, pat)
        Xv, Xs, g_x = oracle.quant_nvfp4(X, pat, 32)
        ref = oracle.sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp, oracle.OUT_BF16)
    Y = ss.linear_nvfp4(dev(X), ss.compress_weight_nvfp4(dev(W), pat), pat)
    assert_y_matches(host(Y), ref, "fp8", True)


# Many bf16 rows through the activation kernels (the tensor's amax, then one
# thread per window of 8 lifted elements): identity maps and sliding pair
# patterns, rows of 1000 to 8192 elements.
@pytest.mark.parametrize("pat", ["dense", "2:4", "6:8"])
@pytest.mark.parametrize("block", [16, 32])
@pytest.mark.parametrize("M,K", [(3000, 4096), (3000, 3584), (2100, 2048), (2100, 1000),
                                  (1200, 8192)])
def test_quant_lift_act_nvfp4_many_rows(pat, block, M, K):
    X = _x(M, K, "bf16", seed=K + block)
    Xv, Xs, g_x = ss.quant_lift_act_nvfp4(dev(X), pat, block)
    Xv_ref, Xs_ref, g_ref = oracle.quant_nvfp4(X, pat, block)
    _, K_lp = oracle.fp4_shape(pat, K)
    assert host(g_x)[0] == g_ref[0]
    np.testing.assert_array_equal(host(Xv), Xv_ref)
    np.testing.assert_array_equal(host(Xs), oracle.scales_to_tiles(Xs_ref, K_lp, block))


def test_llama_gateup_4of8_nvfp4_full_size():
    """The benchmark's NVFP4 workload at full size (Llama-3.1-8B gate/up,
    M = 8192, N = 14336, K = 4096, pairwise 4:8): GPU compression and
    activation codes, scales and global scales bit-exact against the oracle
    on every row; the GEMM on the first and last 128 and 64 seeded token
    rows within 1e-2."""
    w = synth.WORKLOADS["llama_gateup_4of8_nvfp4"]
    M, N, K, pat = w["M"], w["N"], w["K"], w["pattern"]
    W = synth.make_weight(N, K, w["w_std"], w["in_dtype"])
    X = synth.make_activation(M, K, w["x_kind"], w["in_dtype"])
    _, K_lp = oracle.fp4_shape(pat, K)
    packed = ss.compress_weight_nvfp4(dev(W), pat)
    act = ss.quant_lift_act_nvfp4(dev(X), pat, 32)
    Y = ss.sparse_gemm_nvfp4(packed, act, M, N)
    assert ss.ss_get_device_status() == ss.SS_OK
    Wv, Wm, Ws, g_w = oracle.compress_weight_nvfp4(W, pat)
    assert host(packed[3])[0] == np.float32(g_w)
    np.testing.assert_array_equal(host(packed[0]), Wv)
    np.testing.assert_array_equal(host(packed[1]), oracle.meta_to_tiles(Wm, K_lp // 2))
    np.testing.assert_array_equal(host(packed[2]), oracle.scales_to_tiles(Ws, K_lp, 32))
    Xv, Xs, g_x = oracle.quant_nvfp4(X, pat, 32)
    assert host(act[2])[0] == g_x[0]
    np.testing.assert_array_equal(host(act[0]), Xv)
    np.testing.assert_array_equal(host(act[1]), oracle.scales_to_tiles(Xs, K_lp, 32))
    rows = synth.sample_rows(M, seed=9, middle=64)
    Wd = oracle.decode_sparse_nvfp4(Wv, Wm, Ws, K_lp)
    Xd = oracle.decode_dense_nvfp4(Xv[rows], Xs[rows], K_lp, 32)
    Y_ref = oracle.matmul_nvfp4(Xd, g_x, Wd, np.full(N, g_w, dtype=np.float32), oracle.OUT_BF16)
    assert_y_matches(host(Y)[rows], Y_ref, "fp8", True)
