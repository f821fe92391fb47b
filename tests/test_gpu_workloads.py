"""GPU parity at the full sizes of the benchmark workloads, in the launch
configuration the benchmark times.  Quantised operands, packed weights and
metadata are compared in full (bit-exact); the GEMM output is compared on a
deterministic row sample the oracle computes one row at a time (first and
last rows plus seeded middle rows) -- bit-exact for INT8, within 1e-2
relative for FP8."""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_quantized_b200 as ss
from structured_sparse_quantized_b200 import synth
from _helpers import Q, assert_y_matches, dev, host

pytestmark = pytest.mark.gpu


def _rows(M):
    return synth.sample_rows(M, seed=7, edge=32, middle=64)


def _weight_sparse_case(W, X, pat, q, out_bf16=True, packed_ref=None):
    M, K = X.shape
    N = W.shape[0]
    Wv_ref, Wm_ref, s_w_ref = packed_ref or oracle.compress_weight(W, pat, Q[q])
    Xq_ref, s_x_ref = oracle.quant_lift_act(X, pat, Q[q])
    Wv, Wm, s_w = ss.compress_weight(dev(W), pat, q)
    Xq, s_x = ss.quant_lift_act(dev(X), pat, q)
    np.testing.assert_array_equal(host(s_w), s_w_ref)
    np.testing.assert_array_equal(host(Wv), Wv_ref)
    np.testing.assert_array_equal(host(Wm), oracle.meta_to_tiles(Wm_ref, Wv_ref.shape[1] * 2))
    np.testing.assert_array_equal(host(s_x), s_x_ref)
    np.testing.assert_array_equal(host(Xq), Xq_ref)
    Y = ss.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, M, N, q,
                       out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    assert ss.ss_get_device_status() == ss.SS_OK
    rows = _rows(M)
    _, _, K_lp = oracle.slide_shape(pat, K)
    Y_ref = oracle.sparse_gemm(0, Wv_ref, Wm_ref, s_w_ref, Xq_ref, s_x_ref, M, N, K_lp, Q[q],
                               oracle.OUT_BF16 if out_bf16 else oracle.OUT_F32, m_idx=rows)
    assert_y_matches(host(Y)[rows], Y_ref, q, out_bf16)


def test_linear_6of8_int8_m16():
    w = synth.WORKLOADS["linear_6of8_int8_m16"]
    W = synth.make_weight(w["N"], w["K"], w["w_std"], w["in_dtype"])
    X = synth.make_activation(w["M"], w["K"], w["x_kind"], w["in_dtype"])
    _weight_sparse_case(W, X, "6:8", "int8", out_bf16=False)


@pytest.mark.parametrize("M", [2048, 8192])
def test_llama_q_2of4_int8(M):
    W = synth.make_weight(4096, 4096, 0.02, "bf16")
    X = synth.make_activation(M, 4096, "outlier", "bf16")
    _weight_sparse_case(W, X, "2:4", "int8")


@pytest.fixture(scope="module")
def qwen_weight():
    W = synth.make_weight(18944, 3584, 0.02, "bf16")
    return W, oracle.compress_weight(W, "6:8", oracle.FP8_E4M3)


@pytest.mark.parametrize("M", [1, 16, 128, 1024, 4096, 8192])
def test_qwen_gateup_6of8_fp8(qwen_weight, M):
    W, packed = qwen_weight
    X = synth.make_activation(M, 3584, "gauss", "bf16")
    _weight_sparse_case(W, X, "6:8", "fp8", packed_ref=packed)


def test_online_x_2of4_fp8():
    M, K, N = 8192, 4096, 14336
    W = synth.make_weight(N, K, 0.02, "bf16")
    X = synth.make_activation(M, K, "heavy", "bf16")
    Wq_ref, _, s_w_ref = oracle.compress_weight(W, "dense", oracle.FP8_E4M3)
    Xv_ref, Xm_ref, s_x_ref = oracle.prune_act_2to4(X, oracle.FP8_E4M3)
    Wq, _, s_w = ss.compress_weight(dev(W), "dense", "fp8")
    Xv, Xm, s_x = ss.prune_act_2to4(dev(X), "fp8")
    np.testing.assert_array_equal(host(Wq), Wq_ref)
    np.testing.assert_array_equal(host(s_w), s_w_ref)
    np.testing.assert_array_equal(host(Xv), Xv_ref)
    np.testing.assert_array_equal(host(Xm), oracle.meta_to_tiles(Xm_ref, Xv_ref.shape[1] * 2))
    np.testing.assert_array_equal(host(s_x), s_x_ref)
    Y = ss.sparse_gemm(1, Xv, Xm, s_x, Wq, s_w, M, N, "fp8")
    assert ss.ss_get_device_status() == ss.SS_OK
    rows = _rows(M)
    Y_ref = oracle.sparse_gemm(1, Xv_ref, Xm_ref, s_x_ref, Wq_ref, s_w_ref, M, N, Wq_ref.shape[1],
                               oracle.FP8_E4M3, oracle.OUT_BF16, m_idx=rows)
    assert_y_matches(host(Y)[rows], Y_ref, "fp8", True)
    # the dense comparator on the same weights
    Xq_ref, sx_ref = oracle.quant_lift_act(X, "dense", oracle.FP8_E4M3)
    Xq, sx = ss.quant_lift_act(dev(X), "dense", "fp8")
    np.testing.assert_array_equal(host(Xq), Xq_ref)
    Yd = ss.dense_gemm(Xq, sx, Wq, s_w, "fp8")
    Yd_ref = oracle.dense_gemm(Xq_ref, sx_ref, Wq_ref, s_w_ref, oracle.FP8_E4M3, oracle.OUT_BF16,
                               m_idx=rows)
    assert_y_matches(host(Yd)[rows], Yd_ref, "fp8", True)


@pytest.mark.parametrize("pat", ["dense", "2:4", "4:6", "6:8", "8:10"])
@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_pattern_sweep_llama_q_o(pat, q):
    """One Llama-3.1-8B q/o projection (4096 x 4096) per pattern and dtype at
    M = 2048."""
    M, N, K = 2048, 4096, 4096
    W = synth.make_weight(N, K, 0.02, "bf16")
    X = synth.make_activation(M, K, "gauss", "bf16")
    if pat != "dense":
        _weight_sparse_case(W, X, pat, q)
        return
    Wq_ref, _, s_w_ref = oracle.compress_weight(W, "dense", Q[q])
    Xq_ref, s_x_ref = oracle.quant_lift_act(X, "dense", Q[q])
    Wq, _, s_w = ss.compress_weight(dev(W), "dense", q)
    Xq, s_x = ss.quant_lift_act(dev(X), "dense", q)
    np.testing.assert_array_equal(host(Wq), Wq_ref)
    np.testing.assert_array_equal(host(Xq), Xq_ref)
    Y = ss.dense_gemm(Xq, s_x, Wq, s_w, q)
    rows = _rows(M)
    Y_ref = oracle.dense_gemm(Xq_ref, s_x_ref, Wq_ref, s_w_ref, Q[q], oracle.OUT_BF16, m_idx=rows)
    assert_y_matches(host(Y)[rows], Y_ref, q, True)


# The Llama-3.1-8B layer sweep at the benchmark's M = 16384: every projection
# shape other than q/o, every pattern, INT8 and FP8.  Quantised activations,
# packed weights and metadata are compared in full; Y on the first and last
# 32 rows plus 64 seeded rows.  down with 8:10 INT8 (K_lp = 22944) is the
# widest int32 accumulation of the build and must be bit-exact.
_LAYER_CACHE = {}


def _layer_inputs(proj, M):
    N, K = synth.LLAMA_LAYER[proj]
    key_w, key_x = ("W", proj), ("X", M, K)
    if key_w not in _LAYER_CACHE:
        _LAYER_CACHE[key_w] = synth.make_weight(N, K, 0.02, "bf16")
    if key_x not in _LAYER_CACHE:   # two activations (K = 4096 and 14336): 0.6 GB bf16
        _LAYER_CACHE[key_x] = synth.make_activation(M, K, "gauss", "bf16")
    return _LAYER_CACHE[key_w], _LAYER_CACHE[key_x]


@pytest.mark.parametrize("proj", ["gate_up", "k_v", "down"])
@pytest.mark.parametrize("pat", ["dense", "2:4", "4:6", "6:8", "8:10"])
@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_llama_layer_sweep_m16384(proj, pat, q):
    M = 16384
    W, X = _layer_inputs(proj, M)
    N = W.shape[0]
    if pat != "dense":
        _weight_sparse_case(W, X, pat, q)
        return
    Wq_ref, _, s_w_ref = oracle.compress_weight(W, "dense", Q[q])
    Xq_ref, s_x_ref = oracle.quant_lift_act(X, "dense", Q[q])
    Wq, _, s_w = ss.compress_weight(dev(W), "dense", q)
    Xq, s_x = ss.quant_lift_act(dev(X), "dense", q)
    np.testing.assert_array_equal(host(Wq), Wq_ref)
    np.testing.assert_array_equal(host(s_w), s_w_ref)
    np.testing.assert_array_equal(host(Xq), Xq_ref)
    np.testing.assert_array_equal(host(s_x), s_x_ref)
    Y = ss.dense_gemm(Xq, s_x, Wq, s_w, q)
    assert ss.ss_get_device_status() == ss.SS_OK
    rows = _rows(M)
    Y_ref = oracle.dense_gemm(Xq_ref, s_x_ref, Wq_ref, s_w_ref, Q[q], oracle.OUT_BF16, m_idx=rows)
    assert_y_matches(host(Y)[rows], Y_ref, q, True)
