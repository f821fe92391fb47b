"""Pins for the CPU oracle: each test ties an oracle function to something
other than the oracle itself -- values the pages print (tests/golden, cited
there), the completeness theorem checked by brute force, closed forms, the
OCP FP8 code table, independent library routines (numpy integer/float64
matmul, torch's float8/bfloat16 casts) and error bounds.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

PATTERNS = ["2:4", "4:6", "6:8", "8:10"]


# ---------------------------------------------------------------- shapes

def test_pattern_table_matches_pages():
    """Non-zero ratio keep/group and ideal speedup 2 / (K_lift / K_pad)."""
    for pat, pct, speed in read_golden("pattern_table.txt"):
        keep, group = oracle.pattern(pat)
        K = group * 12
        K_pad, K_lift, _ = oracle.slide_shape(pat, K)
        assert round(100.0 * keep / group, 1) == pytest.approx(float(pct), abs=0.05)
        digits = len(speed.split(".")[1])
        assert round(2.0 / (K_lift / K_pad), digits) == pytest.approx(float(speed))


def test_k_lift_values_from_pages():
    for pat, K, K_lift in read_golden("workload_shapes.txt"):
        _, kl, k_lp = oracle.slide_shape(pat, int(K))
        assert kl == int(K_lift)
        assert k_lp % 128 == 0 and k_lp >= kl and k_lp - kl < 128


@pytest.mark.parametrize("pat", PATTERNS)
def test_k_lift_closed_form(pat):
    keep, group = oracle.pattern(pat)
    Nh = group // 2
    for K in [1, 7, group, 64, 4096, 3584, 14336, 4097]:
        K_pad, K_lift, K_lp = oracle.slide_shape(pat, K)
        assert K_pad == math.ceil(K / group) * group
        # Nh-1 windows of 4 per group of 2Nh: expansion 2(Nh-1)/Nh
        assert K_lift * Nh == K_pad * 2 * (Nh - 1)
        assert K_lp == math.ceil(K_lift / 128) * 128


def test_bit_accounting_matches_pages():
    for kind, vbits, sparse, expect, _ in read_golden("bit_accounting.txt"):
        b = oracle.bits_per_element(int(vbits), bool(int(sparse)))
        other = oracle.bits_per_element(int(expect), False)
        if kind == "equal":
            assert b == pytest.approx(other)
        else:
            assert b > other
    assert oracle.bits_per_element(8, True) == pytest.approx(5.125)


# ---------------------------------------------------------------- windows

def _int_row(values):
    """A row whose absmax is 127 so that the INT8 scale is exactly 1."""
    return np.asarray(values, dtype=np.float32)


def test_worked_example_windows():
    rows = {r[0]: r[1:] for r in read_golden("slide_6of8_example.txt")}
    pat = rows["pattern"][0]
    group = int(rows["group"][0])
    # activation = its own index, plus an absmax-127 tail channel group
    x = _int_row(list(range(1, group + 1)) + [127] + [0] * (group - 1))
    Xq, s_x = oracle.quant_lift_act(x[None, :], pat, oracle.INT8)
    assert s_x[0] == pytest.approx(1.0)
    n_win = int(rows["windows"][0])
    lifted = Xq[0, : 4 * n_win].astype(np.int8)
    expect = []
    win_rows = [r for r in read_golden("slide_6of8_example.txt") if r[0] == "window"]
    assert len(win_rows) == n_win
    for r in win_rows:
        expect.extend(int(p) + 1 for p in r[2:])
    assert lifted.tolist() == expect
    assert len(expect) == int(rows["lifted_length"][0])
    _, K_lift, _ = oracle.slide_shape(pat, group)
    assert K_lift == int(rows["lifted_length"][0])
    assert K_lift / group == pytest.approx(float(rows["expansion"][0]))


def _placements(group, n_kept):
    return itertools.combinations(range(group), n_kept)


@pytest.mark.parametrize("group", [4, 6, 8, 10, 12])
def test_lossless_decomposition_bruteforce(group):
    """Completeness theorem: every placement of at most 2Nh-2 non-zeros in a
    2Nh block decomposes into Nh-1 stride-2 width-4 windows, and the lifted
    integer dot product equals the original one exactly."""
    keep = group - 2
    pat = f"{keep}:{group}"
    rng = np.random.default_rng(group)
    rows_w, rows_x = [], []
    for n_kept in range(0, keep + 1):
        for pos in _placements(group, n_kept):
            w = np.zeros(2 * group, dtype=np.float32)
            vals = rng.integers(1, 127, size=len(pos))
            sign = rng.choice([-1, 1], size=len(pos))
            w[list(pos)] = vals * sign
            w[group] = 127.0           # second group pins the scale to 1
            rows_w.append(w)
            x = rng.integers(-127, 128, size=2 * group).astype(np.float32)
            x[group + 1] = 127.0
            rows_x.append(x)
    W = np.stack(rows_w)
    X = np.stack(rows_x)
    # the window assignment covers every kept position
    mask = oracle.prune_mask(W, keep, group)
    win = oracle.assign_windows(mask, group)
    assert np.all((win >= 0) == mask.astype(bool))
    for j in range((group // 2) - 1):
        per_window = (win.reshape(len(W), -1, group) == j).sum(axis=2)
        assert per_window.max() <= 2
    Wv, Wm, s_w = oracle.compress_weight(W, pat, oracle.INT8)
    Xq, s_x = oracle.quant_lift_act(X, pat, oracle.INT8)
    assert np.all(s_w == 1.0) and np.all(s_x == 1.0)
    _, K_lift, K_lp = oracle.slide_shape(pat, W.shape[1])
    Wd = oracle.decompress_2to4(Wv, Wm, K_lp).astype(np.int8).astype(np.int64)
    Xl = Xq.astype(np.int8).astype(np.int64)
    lifted = (Xl * Wd).sum(axis=1)                     # row-wise dot products
    plain = (X.astype(np.int64) * W.astype(np.int64)).sum(axis=1)
    np.testing.assert_array_equal(lifted, plain)


@pytest.mark.parametrize("group", [4, 6, 8, 10, 12])
def test_one_more_nonzero_does_not_fit(group):
    """Capacity 2(Nh-1) < 2Nh-1: no assignment exists, the oracle reports it."""
    mask = np.zeros((1, group), dtype=np.uint8)
    mask[0, : group - 1] = 1
    with pytest.raises(oracle.OracleError):
        oracle.assign_windows(mask, group)
    Nh = group // 2
    assert 2 * (Nh - 2) < group - 2          # Nh-2 windows never suffice


def test_first_fit_examples():
    """Ascending first-fit on hand-worked 6:8 blocks."""
    cases = {
        (0, 1, 2, 3, 4, 5): [0, 0, 1, 1, 2, 2, -1, -1],
        (2, 3, 4, 5, 6, 7): [-1, -1, 0, 0, 1, 1, 2, 2],
        (0, 1, 2, 3, 6, 7): [0, 0, 1, 1, -1, -1, 2, 2],
        (0, 2, 3, 4, 6, 7): [0, -1, 0, 1, 1, -1, 2, 2],
        (1, 2, 3, 4, 5, 7): [-1, 0, 0, 1, 1, 2, -1, 2],
    }
    for pos, expect in cases.items():
        m = np.zeros((1, 8), dtype=np.uint8)
        m[0, list(pos)] = 1
        assert oracle.assign_windows(m, 8)[0].tolist() == expect


# ---------------------------------------------------------------- pruning

@pytest.mark.parametrize("pat", PATTERNS)
def test_prune_keeps_largest(pat):
    keep, group = oracle.pattern(pat)
    rng = np.random.default_rng(3)
    W = rng.standard_normal((64, group * 9)).astype(np.float32)
    W[::7, ::5] = 0.5                                  # plant exact ties
    W[::7, 1::5] = -0.5
    mask = oracle.prune_mask(W, keep, group)
    a = np.abs(W).reshape(64, -1, group)
    m = mask.reshape(64, -1, group).astype(bool)
    assert np.all(m.sum(axis=2) == keep)
    kept_min = np.where(m, a, np.inf).min(axis=2)
    drop_max = np.where(~m, a, -np.inf).max(axis=2)
    assert np.all(kept_min >= drop_max)
    # among equal magnitudes the lower index is kept first
    for r, g in zip(*np.nonzero(kept_min == drop_max)):
        t = kept_min[r, g]
        ties = np.nonzero(a[r, g] == t)[0]
        kept_ties = [i for i in ties if m[r, g, i]]
        assert kept_ties == list(ties[: len(kept_ties)])


def test_energy_removed_by_2of4_matches_pages():
    target = dict((k, float(v)) for k, v in read_golden("energy.txt"))["elementwise_2of4"]
    X = np.random.default_rng(0).standard_normal((1000, 4000)).astype(np.float32)
    mask = oracle.prune_mask(X, 2, 4)
    removed = (X.astype(np.float64) ** 2 * (1 - mask)).sum() / (X.astype(np.float64) ** 2).sum()
    assert 100 * removed == pytest.approx(target, abs=0.1)


def test_energy_removed_by_pairwise_4of8_matches_pages_and_closed_form():
    target = dict((k, float(v)) for k, v in read_golden("energy.txt"))["pairwise_4of8"]
    X = np.random.default_rng(0).standard_normal((1000, 4000)).astype(np.float32)
    mask = oracle.prune_pairwise_4of8(X)
    removed = (X.astype(np.float64) ** 2 * (1 - mask)).sum() / (X.astype(np.float64) ** 2).sum()
    assert 100 * removed == pytest.approx(target, abs=0.1)
    # closed form: pair energy ~ Exp(mean 2); the two smallest of four have
    # expected sum 2*(1/4 + 1/4 + 1/3) = 5/3 out of 8
    assert removed == pytest.approx(5.0 / 24.0, abs=0.002)


def test_online_prune_2of4_invariants():
    X = torch.randn(40, 260, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    Xf = X.float().numpy()
    for q in (oracle.INT8, oracle.FP8_E4M3):
        Xv, Xm, s_x = oracle.prune_act_2to4(X, q)
        K_lp = oracle.act_2to4_k_lp(260)
        assert Xv.shape == (40, K_lp // 2) and Xm.shape == (40, K_lp // 8)
        dense = oracle.decompress_2to4(Xv, Xm, K_lp)[:, :260]
        mask = oracle.prune_mask(Xf, 2, 4)[:, :260]
        # exactly the pruned positions are non-zero-capable, the rest are 0
        assert np.all(dense[~mask.astype(bool)] == 0)
        # the row absmax is always kept and maps to the top code
        amax = np.abs(Xf).argmax(axis=1)
        codes = dense[np.arange(40), amax]
        if q == oracle.INT8:
            assert np.all(np.abs(codes.view(np.int8).astype(int)) == 127)
        else:
            assert np.all(codes & 0x7F == 0x7E)
        np.testing.assert_allclose(s_x, np.abs(Xf).max(axis=1) / (127 if q == 0 else 448),
                                   rtol=1e-7)


def test_nibbles_are_legal():
    legal = {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}
    W = np.random.default_rng(1).standard_normal((33, 150)).astype(np.float32)
    for pat in PATTERNS:
        _, Wm, _ = oracle.compress_weight(W, pat, oracle.INT8)
        nib = np.concatenate([Wm & 0xF, Wm >> 4]).ravel()
        assert set(np.unique(nib).tolist()) <= legal


# ---------------------------------------------------------------- formats

def test_e4m3_ocp_table():
    for code, value in read_golden("e4m3_ocp.txt"):
        c = int(code, 16)
        assert oracle.e4m3_to_float(c) == float(value)
        assert oracle.e4m3_from_float(float(value)) == c
    assert math.isnan(oracle.e4m3_to_float(0x7F))


def test_e4m3_matches_torch_cast_in_range():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_to_float(c) == codes[c]
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(4000) * 50,
        rng.standard_normal(2000) * 0.01,
        (codes[np.isfinite(codes)][:-1] + codes[np.isfinite(codes)][1:]) / 2,  # midpoints
    ]).astype(np.float32)
    vals = vals[np.abs(vals) <= 448]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_from_float(v) for v in vals], dtype=np.uint8)
    # torch keeps the sign of zero the same way
    np.testing.assert_array_equal(got, ref)


def test_e4m3_saturates():
    assert oracle.e4m3_from_float(449.0) == 0x7E
    assert oracle.e4m3_from_float(1e9) == 0x7E
    assert oracle.e4m3_from_float(-1e9) == 0xFE
    assert oracle.e4m3_from_float(464.0) == 0x7E


def test_bf16_matches_torch():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(5000) * 100,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8])]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.uint16).numpy()
    got = np.array([oracle.bf16_from_float(x) for x in v], dtype=np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_int8_quantisation_textbook_cases():
    inv, s = oracle.scale_from_absmax(127.0, oracle.INT8)
    assert inv == 1.0 and s == 1.0
    assert oracle.quantize_value(2.5, inv, oracle.INT8) == 2          # ties to even
    assert oracle.quantize_value(3.5, inv, oracle.INT8) == 4
    assert np.uint8(oracle.quantize_value(-2.5, inv, oracle.INT8)).view(np.int8) == -2
    assert np.uint8(oracle.quantize_value(-127.0, inv, oracle.INT8)).view(np.int8) == -127
    inv, s = oracle.scale_from_absmax(0.0, oracle.INT8)
    assert inv == 0.0 and s == 0.0
    # absmax maps to +-127 for many magnitudes, never to -128
    for a in np.random.default_rng(4).uniform(1e-3, 1e3, 200).astype(np.float32):
        inv, s = oracle.scale_from_absmax(float(a), oracle.INT8)
        assert oracle.quantize_value(float(a), inv, oracle.INT8) == 127
        assert np.uint8(oracle.quantize_value(-float(a), inv, oracle.INT8)).view(np.int8) == -127
        inv8, _ = oracle.scale_from_absmax(float(a), oracle.FP8_E4M3)
        assert oracle.quantize_value(float(a), inv8, oracle.FP8_E4M3) == 0x7E


# ---------------------------------------------------------------- matmul

def test_int8_matmul_matches_numpy():
    rng = np.random.default_rng(5)
    A = rng.integers(-127, 128, (37, 300)).astype(np.int8)
    B = rng.integers(-127, 128, (21, 300)).astype(np.int8)
    acc = oracle.matmul_acc(oracle.INT8, A.view(np.uint8), B.view(np.uint8))
    np.testing.assert_array_equal(acc, A.astype(np.int64) @ B.astype(np.int64).T)


def test_fp8_matmul_matches_numpy_float64():
    rng = np.random.default_rng(6)
    A = rng.integers(0, 256, (17, 200), dtype=np.uint8)
    B = rng.integers(0, 256, (9, 200), dtype=np.uint8)
    A[(A & 0x7F) == 0x7F] = 0x3C
    B[(B & 0x7F) == 0x7F] = 0x3C
    acc = oracle.matmul_acc(oracle.FP8_E4M3, A, B)
    ref = oracle.e4m3_decode_array(A) @ oracle.e4m3_decode_array(B).T
    np.testing.assert_allclose(acc, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("pat", PATTERNS + ["dense"])
@pytest.mark.parametrize("q", [oracle.INT8, oracle.FP8_E4M3])
def test_method_equals_plain_path(pat, q):
    """Path (ii) (decompose, lift, pack, sparse matmul over K_lp) equals path
    (i) (prune, quantise, naive matmul over the original K): exactly for
    INT8, and to double-rounding for E4M3."""
    rng = np.random.default_rng(8)
    K = 150                              # not a multiple of 4, 6, 8 or 10
    W = torch.from_numpy(rng.standard_normal((40, K)).astype(np.float32) * 0.02).to(torch.bfloat16)
    X = torch.from_numpy(rng.standard_normal((23, K)).astype(np.float32)).to(torch.bfloat16)
    plain = oracle.plain_linear(W, X, pat, q, oracle.OUT_F32)
    Wv, Wm, s_w = oracle.compress_weight(W, pat, q)
    Xq, s_x = oracle.quant_lift_act(X, pat, q)
    _, _, K_lp = oracle.slide_shape(pat, K)
    if pat == "dense":
        method = oracle.dense_gemm(Xq, s_x, Wv, s_w, q, oracle.OUT_F32)
    else:
        method = oracle.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, 23, 40, K_lp, q, oracle.OUT_F32)
    if q == oracle.INT8:
        np.testing.assert_array_equal(method, plain)
    else:
        np.testing.assert_allclose(method, plain, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("pat", ["2:4", "6:8", "8:10"])
@pytest.mark.parametrize("q", [oracle.INT8, oracle.FP8_E4M3])
def test_result_within_quantisation_error_bound(pat, q):
    """Y approximates X . prune(W)^T (fp64) within the bound set by the two
    quantisers: |err| <= sum_k |x_k| e_w + |w_k| e_x + e_x e_w, with e the
    largest rounding error of one quantised value, plus bf16 output rounding."""
    rng = np.random.default_rng(9)
    K = 96
    keep, group = oracle.pattern(pat)
    W = rng.standard_normal((24, K)).astype(np.float32)
    X = rng.standard_normal((12, K)).astype(np.float32)
    mask = oracle.prune_mask(W, keep, group)[:, :K].astype(bool)
    ref = X.astype(np.float64) @ np.where(mask, W, 0).astype(np.float64).T
    Wv, Wm, s_w = oracle.compress_weight(W, pat, q)
    Xq, s_x = oracle.quant_lift_act(X, pat, q)
    _, _, K_lp = oracle.slide_shape(pat, K)
    Y = oracle.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, 12, 24, K_lp, q, oracle.OUT_BF16)
    Yf = oracle.bf16_bits_to_float(Y).astype(np.float64)
    if q == oracle.INT8:
        ex = s_x[:, None] / 2.0 * np.ones((1, K))
        ew = s_w[:, None] / 2.0 * np.ones((1, K))
    else:   # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 (normals)
        ex = np.abs(X) * 2.0 ** -4 + s_x[:, None] * 2.0 ** -9
        ew = np.abs(W) * 2.0 ** -4 + s_w[:, None] * 2.0 ** -9
    Wa = np.abs(np.where(mask, W, 0))
    bound = (np.abs(X) @ (ew * mask).T + ex @ Wa.T + ex @ (ew * mask).T)
    bound = bound + np.abs(ref) * 2.0 ** -8 + 1e-6
    assert np.all(np.abs(Yf - ref) <= bound)
    # and the result is close, not just inside a worst-case bound
    rel = np.linalg.norm(Yf - ref) / np.linalg.norm(ref)
    assert rel < (0.02 if q == oracle.INT8 else 0.06)
    if q == oracle.INT8:
        assert np.median(bound) < 0.2 * np.median(np.abs(ref)) + 1.0


# ---------------------------------------------------------------- bf16 tier

def _bf16_vals(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_float(bits).astype(np.float64)


def test_bf16_matmul_matches_numpy_float64():
    """Products of bf16 values are exact in double: the oracle's sum equals a
    float64 library matmul of the decoded values up to summation order."""
    rng = np.random.default_rng(21)
    X = torch.from_numpy(rng.standard_normal((19, 260)).astype(np.float32)).to(torch.bfloat16)
    W = torch.from_numpy(rng.standard_normal((11, 260)).astype(np.float32)).to(torch.bfloat16)
    Xb = X.view(torch.uint16).numpy()
    Wb = W.view(torch.uint16).numpy()
    Y = oracle.matmul_bf16(Xb, Wb, oracle.OUT_F32)
    ref = (_bf16_vals(Xb) @ _bf16_vals(Wb).T).astype(np.float32)
    np.testing.assert_allclose(Y, ref, rtol=1e-6, atol=1e-6)
    # bf16 output is the RNE rounding of the fp32 result
    Yb = oracle.matmul_bf16(Xb, Wb, oracle.OUT_BF16)
    np.testing.assert_array_equal(
        Yb, torch.from_numpy(Y).to(torch.bfloat16).view(torch.uint16).numpy())


def test_bf16_small_integers_exact():
    """With small-integer operands every partial sum is an integer well inside
    binary32: the result is the exact integer product."""
    rng = np.random.default_rng(22)
    X = rng.integers(-8, 9, (13, 96)).astype(np.float32)
    W = rng.integers(-8, 9, (7, 96)).astype(np.float32)
    Xb = oracle.lift_act_bf16(X, "dense")
    Wb, _ = oracle.compress_weight_bf16(W, "dense")
    Y = oracle.matmul_bf16(Xb, Wb, oracle.OUT_F32)
    np.testing.assert_array_equal(Y, (X.astype(np.int64) @ W.astype(np.int64).T).astype(np.float32))


@pytest.mark.parametrize("pat", PATTERNS)
def test_bf16_decompress_is_lifted_pruned_weight(pat):
    """Unpacking the compressed bf16 weight gives, window by window, the pruned
    weight's values at the positions the window map assigns (zero elsewhere);
    summed back over the windows that cover each k it gives prune(W) exactly."""
    rng = np.random.default_rng(23)
    K = 150
    keep, group = oracle.pattern(pat)
    W = rng.standard_normal((9, K)).astype(np.float32)
    Wv, Wm = oracle.compress_weight_bf16(W, pat)
    _, K_lift, K_lp = oracle.slide_shape(pat, K)
    Wl = oracle.decompress_2to4_bf16(Wv, Wm, K_lp)
    Wl_vals = _bf16_vals(Wl)
    # every window holds at most 2 nonzeros (2:4 on the lifted axis)
    assert np.all((Wl_vals.reshape(9, -1, 4) != 0).sum(-1) <= 2)
    # fold the lifted axis back onto k with the window map of the pages
    Nh = group // 2
    back = np.zeros((9, K + group), dtype=np.float64)
    for w in range(K_lift // 4):
        g, j = divmod(w, Nh - 1)
        for t in range(4):
            back[:, g * group + 2 * j + t] += Wl_vals[:, 4 * w + t]
    mask = oracle.prune_mask(W, keep, group)[:, :K].astype(bool)
    Wp = np.where(mask, W, 0)
    Wp_b = _bf16_vals(torch.from_numpy(Wp).to(torch.bfloat16).view(torch.uint16).numpy())
    np.testing.assert_array_equal(back[:, :K], Wp_b)
    assert np.all(back[:, K:] == 0)
    assert np.all(Wl_vals[:, K_lift:] == 0)


@pytest.mark.parametrize("pat", PATTERNS + ["dense"])
def test_bf16_method_equals_plain_path(pat):
    """Decompose + lift + pack + sparse matmul over K_lp equals prune + naive
    matmul over K: exactly on small integers, to summation order otherwise."""
    rng = np.random.default_rng(24)
    K = 150
    keep, group = oracle.pattern(pat)
    _, _, K_lp = oracle.slide_shape(pat, K)

    def method(W, X):
        Wv, Wm = oracle.compress_weight_bf16(W, pat)
        Xl = oracle.lift_act_bf16(X, pat)
        if pat == "dense":
            return oracle.matmul_bf16(Xl, Wv, oracle.OUT_F32)
        return oracle.sparse_gemm_bf16(0, Wv, Wm, Xl, X.shape[0], W.shape[0], K_lp,
                                       oracle.OUT_F32)

    Wi = rng.integers(-6, 7, (40, K)).astype(np.float32)
    Xi = rng.integers(-6, 7, (23, K)).astype(np.float32)
    # distinct magnitudes inside each group keep the top-k choice unique
    Wi = Wi + np.sign(Wi) * (np.arange(K) % 7)[None, :].astype(np.float32) / 8
    np.testing.assert_array_equal(method(Wi, Xi), oracle.plain_linear_bf16(Wi, Xi, pat, oracle.OUT_F32))
    W = rng.standard_normal((40, K)).astype(np.float32)
    X = rng.standard_normal((23, K)).astype(np.float32)
    np.testing.assert_allclose(method(W, X), oracle.plain_linear_bf16(W, X, pat, oracle.OUT_F32),
                               rtol=1e-6, atol=1e-6)
    # and the sparse-activation operand role (A = lifted X, compressed) agrees
    if pat != "dense":
        Xv, Xm = oracle.compress_weight_bf16(X, "2:4")
        Wl = oracle.lift_act_bf16(W, "2:4")
        K4 = oracle.slide_shape("2:4", K)[2]
        Y1 = oracle.sparse_gemm_bf16(1, Xv, Xm, Wl, 23, 40, K4, oracle.OUT_F32)
        Y0 = oracle.sparse_gemm_bf16(0, *oracle.compress_weight_bf16(W, "2:4"),
                                     oracle.lift_act_bf16(X, "2:4"), 23, 40, K4, oracle.OUT_F32)
        Xp = np.where(oracle.prune_mask(X, 2, 4)[:, :K].astype(bool), X, 0)
        Wp = np.where(oracle.prune_mask(W, 2, 4)[:, :K].astype(bool), W, 0)
        np.testing.assert_allclose(Y1, oracle.plain_linear_bf16(W, Xp, "dense", oracle.OUT_F32),
                                   rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(Y0, oracle.plain_linear_bf16(Wp, X, "dense", oracle.OUT_F32),
                                   rtol=1e-6, atol=1e-6)
