"""The bounded waits' abort path on the GPU, driven without any fault.

A test hook makes the GEMM producers skip one K stage of their first tile:
nothing is loaded toward that stage's barrier, so the MMA warp's bounded wait
for it can only run out (a wait that nothing satisfies; no copy or MMA is
aimed at it).  With the wait limit shortened to 20 ms the kernel must record
SS_ERR_TIMEOUT, unwind (issued copies land, issued MMAs drain, tensor memory
is freed) and leave the device usable: the status is read once and cleared,
and the same call made again returns the oracle's result."""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_quantized_b200 as ss
from structured_sparse_quantized_b200 import synth
from _helpers import Q, assert_y_matches, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture
def short_waits():
    assert ss.ss_get_device_status() == ss.SS_OK
    ss.ss_debug_set_wait_limit(20_000_000)  # 20 ms
    yield
    ss.ss_debug_skip_stage(-1)
    ss.ss_debug_set_wait_limit(4_000_000_000)


def _run(shape, q, ops):
    if shape == "dense":
        Xq, s_x, Wq, s_w = ops
        return ss.dense_gemm(Xq, s_x, Wq, s_w, q)
    Wv, Wm, s_w, Xq, s_x, M, N = ops
    return ss.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, M, N, q)


@pytest.mark.parametrize("shape", ["narrow", "wide", "dense"])
@pytest.mark.parametrize("q", ["int8", "fp8"])
def test_wait_runs_out_then_next_call_is_clean(shape, q, short_waits, monkeypatch):
    M, N, K = 500, 1024, 2048
    monkeypatch.setenv("SS_SPARSE_KERNEL", "wide" if shape == "wide" else "narrow")
    W = synth.make_weight(N, K, 0.02, "bf16")
    X = synth.make_activation(M, K, "gauss", "bf16")
    pat = "dense" if shape == "dense" else "2:4"
    if shape == "dense":
        Wq, _, s_w = ss.compress_weight(dev(W), "dense", q)
        Xq, s_x = ss.quant_lift_act(dev(X), "dense", q)
        ops = (Xq, s_x, Wq, s_w)
    else:
        Wv, Wm, s_w = ss.compress_weight(dev(W), pat, q)
        Xq, s_x = ss.quant_lift_act(dev(X), pat, q)
        ops = (Wv, Wm, s_w, Xq, s_x, M, N)
    assert ss.ss_get_device_status() == ss.SS_OK

    ss.ss_debug_skip_stage(1)
    _run(shape, q, ops)                       # the launch itself succeeds
    assert ss.ss_get_device_status() == ss.SS_ERR_TIMEOUT
    assert ss.ss_get_device_status() == ss.SS_OK   # read once, then cleared

    ss.ss_debug_skip_stage(-1)
    ss.ss_debug_set_wait_limit(4_000_000_000)
    Y = _run(shape, q, ops)
    assert ss.ss_get_device_status() == ss.SS_OK
    rows = synth.sample_rows(M, seed=3, edge=32, middle=32)
    if shape == "dense":
        Wq_r, _, s_w_r = oracle.compress_weight(W, "dense", Q[q])
        Xq_r, s_x_r = oracle.quant_lift_act(X, "dense", Q[q])
        ref = oracle.dense_gemm(Xq_r, s_x_r, Wq_r, s_w_r, Q[q], oracle.OUT_BF16, m_idx=rows)
    else:
        Wv_r, Wm_r, s_w_r = oracle.compress_weight(W, pat, Q[q])
        Xq_r, s_x_r = oracle.quant_lift_act(X, pat, Q[q])
        ref = oracle.sparse_gemm(0, Wv_r, Wm_r, s_w_r, Xq_r, s_x_r, M, N, Xq_r.shape[1], Q[q],
                                 oracle.OUT_BF16, m_idx=rows)
    assert_y_matches(host(Y)[rows], ref, q, True)


def test_status_exchange_keeps_a_recorded_error_until_read():
    """A NaN weight records SS_ERR_DATA on the device; the status call made
    on another stream after the work has finished still returns it (the word
    is device-wide), and only once."""
    W = torch.zeros((128, 64), dtype=torch.float32)
    W[5, 7] = float("nan")
    ss.compress_weight(dev(W), "2:4", "int8")
    torch.cuda.synchronize()
    other = torch.cuda.Stream()
    assert ss.ss_get_device_status(other) == ss.SS_ERR_DATA
    assert ss.ss_get_device_status(other) == ss.SS_OK
