"""GPU parity of the split-K GEMM that decode-sized problems take (at most 64
tokens and few 128-channel tiles: the K range of each tile is split over
the CTAs of a cluster and reduced through distributed shared memory).
INT8 must stay bit-exact (int32 partials); FP8 and bf16 within 1e-2."""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_quantized_b200 as ss
from structured_sparse_quantized_b200 import synth
from _helpers import Q, assert_y_matches, dev, host

pytestmark = pytest.mark.gpu

# M, N, K, pattern.  Splits: 4096 channels = 32 tiles (S = 4), 1024 = 8 tiles
# (S = 8), 1000 = 8 ragged tiles, 130 = 2 tiles with two K stages (S = 2).
DECODE_CASES = [
    (1, 4096, 4096, "2:4"),
    (16, 4096, 4096, "6:8"),
    (7, 1024, 4096, "6:8"),
    (33, 1000, 640, "4:6"),
    (64, 4096, 2048, "8:10"),
    (1, 130, 300, "2:4"),
]


@pytest.mark.parametrize("M,N,K,pat", DECODE_CASES)
@pytest.mark.parametrize("q", ["int8", "fp8"])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_splitk_weight_sparse(M, N, K, pat, q, out):
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


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (40, 2048, 3000), (16, 1024, 14336)])
@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_splitk_dense(M, N, K, q):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    Wq, _, s_w = oracle.compress_weight(W, "dense", Q[q])
    Xq, s_x = oracle.quant_lift_act(X, "dense", Q[q])
    Y_ref = oracle.dense_gemm(Xq, s_x, Wq, s_w, Q[q], oracle.OUT_BF16)
    Y = ss.dense_gemm(dev(Xq), dev(s_x), dev(Wq), dev(s_w), q)
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(host(Y), Y_ref, q, True)


@pytest.mark.parametrize("M,N,K,pat", [(1, 4096, 4096, "2:4"), (16, 1024, 4096, "6:8"),
                                       (5, 4096, 1000, "dense")])
def test_splitk_bf16(M, N, K, pat):
    W = synth.gaussian((N, K), std=0.02, seed=0, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=1, dtype=torch.bfloat16)
    _, _, K_lp = oracle.slide_shape(pat, K)
    Wv, Wm = oracle.compress_weight_bf16(W, pat)
    Xl = oracle.lift_act_bf16(X, pat)
    bf = lambda a: dev(torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16))
    if pat == "dense":
        Y_ref = oracle.matmul_bf16(Xl, Wv, oracle.OUT_BF16)
        Y = ss.dense_gemm(bf(Xl), None, bf(Wv), None, "bf16")
    else:
        Y_ref = oracle.sparse_gemm_bf16(0, Wv, Wm, Xl, M, N, K_lp, oracle.OUT_BF16)
        Y = ss.sparse_gemm(0, bf(Wv), dev(oracle.meta_to_tiles(Wm, K_lp, i16=True)), None,
                           bf(Xl), None, M, N, "bf16")
    assert ss.ss_get_device_status() == ss.SS_OK
    assert_y_matches(host(Y), Y_ref, "bf16", True)


@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_splitk_matches_one_pass_kernel(q, monkeypatch):
    """The split and the one-pass kernel on the same decode inputs: INT8
    identical bits, FP8 within the tolerance of each other."""
    M, N, K, pat = 9, 4096, 4096, "6:8"
    W = synth.gaussian((N, K), std=0.02, seed=3, dtype=torch.bfloat16)
    X = synth.gaussian((M, K), std=1.0, seed=4, dtype=torch.bfloat16)
    packed = ss.compress_weight(dev(W), pat, q)
    y_split = host(ss.linear(dev(X), packed, pat, q))
    monkeypatch.setenv("SS_SPARSE_KERNEL", "narrow")
    y_one = host(ss.linear(dev(X), packed, pat, q))
    assert_y_matches(y_split, y_one, q, True)
