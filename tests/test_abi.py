"""CPU checks of the C-ABI library: it loads, exports every function that
include/ss.h declares, and its host-only logic (pattern parsing, shapes,
argument validation before any launch) behaves as documented.  No compute
call runs here: there is no GPU on this machine."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import structured_sparse_quantized_b200 as ss

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from structured_sparse_quantized_b200 import _build
    _build.build()
    return ss.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "ss.h"), encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ss_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["ss_compress_weight", "ss_quant_lift_act", "ss_prune_act_2to4", "ss_sparse_gemm",
              "ss_dense_gemm", "ss_slide_shape", "ss_parse_pattern", "ss_get_device_status"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # same names in the Python binding
    for name in declared_functions():
        assert hasattr(ss, name), name


def test_parse_pattern():
    assert ss.ss_parse_pattern("2:4") == (2, 4)
    assert ss.ss_parse_pattern("4:6") == (4, 6)
    assert ss.ss_parse_pattern("6:8") == (6, 8)
    assert ss.ss_parse_pattern("8:10") == (8, 10)
    assert ss.ss_parse_pattern("dense") == (0, 0)
    for bad in ["3:4", "6:9", "", "2:4:6", "10:12"]:
        with pytest.raises(ss.SSError) as e:
            ss.ss_parse_pattern(bad)
        assert e.value.status == ss.SS_ERR_INVALID_ARG


@pytest.mark.parametrize("pat", ["dense", "2:4", "4:6", "6:8", "8:10"])
def test_slide_shape_matches_oracle(pat):
    for K in [1, 5, 64, 150, 3584, 4096, 14336, 4097]:
        assert ss.ss_slide_shape(pat, K) == oracle.slide_shape(pat, K)
    for K in [1, 3, 4, 130, 4096]:
        assert ss.ss_act_2to4_shape(K) == oracle.act_2to4_k_lp(K)


def test_status_strings():
    assert ss.ss_status_string(ss.SS_OK) == "SS_OK"
    assert ss.ss_status_string(ss.SS_ERR_TIMEOUT) == "SS_ERR_TIMEOUT"
    assert ss.ss_status_string(99) == "SS_ERR_UNKNOWN"


def test_argument_errors_return_before_any_launch(L):
    """Validation runs before the device is touched: these return at once."""
    vp = ctypes.c_void_p
    good = vp(0x10000)          # never dereferenced: every call below fails first
    odd = vp(0x10008)
    pat = ss.ss_pattern(6, 8)
    # GEMM: K_lp not a multiple of 128, zero sizes, NULL pointers, bad dtype
    assert L.ss_sparse_gemm(0, good, good, good, good, good, 16, 64, 100, 0, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm(0, good, good, good, good, good, 0, 64, 128, 0, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm(2, good, good, good, good, good, 16, 64, 128, 0, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm(0, None, good, good, good, good, 16, 64, 128, 0, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm(0, good, good, good, good, good, 16, 64, 128, 5, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm(0, odd, good, good, good, good, 16, 64, 128, 0, good, 1, None) \
        == ss.SS_ERR_ALIGNMENT
    assert L.ss_sparse_gemm(0, good, good, good, good, good, 16, 64, 128, 3, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    # scales are required by the 8-bit tiers and unused (NULL allowed) by bf16
    assert L.ss_sparse_gemm(0, good, good, None, good, good, 16, 64, 128, 1, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm(0, good, good, None, good, None, 16, 64, 128, ss.SS_BF16, odd, 1,
                            None) == ss.SS_ERR_ALIGNMENT
    assert L.ss_dense_gemm(good, None, good, None, 16, 64, 128, 0, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_dense_gemm(good, None, odd, None, 16, 64, 128, ss.SS_BF16, good, 1, None) \
        == ss.SS_ERR_ALIGNMENT
    assert L.ss_quant_lift_act(good, 1, 16, 64, pat, 0, good, None, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_quant_lift_act(odd, 1, 16, 64, pat, ss.SS_BF16, good, None, None) \
        == ss.SS_ERR_ALIGNMENT
    assert L.ss_prune_act_2to4(good, 1, 16, 64, ss.SS_BF16, good, odd, None, None) \
        == ss.SS_ERR_ALIGNMENT
    assert L.ss_compress_weight(good, 1, 64, 64, pat, 0, good, good, None, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_compress_weight(odd, 1, 64, 64, pat, ss.SS_BF16, good, good, None, None) \
        == ss.SS_ERR_ALIGNMENT
    assert L.ss_dense_gemm(good, good, good, good, 16, 64, 96, 0, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_dense_gemm(good, good, odd, good, 16, 64, 128, 0, good, 1, None) \
        == ss.SS_ERR_ALIGNMENT
    # activation kernels
    assert L.ss_quant_lift_act(good, 1, 16, 0, pat, 0, good, good, None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_quant_lift_act(good, 3, 16, 64, pat, 0, good, good, None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_quant_lift_act(good, 1, 16, 64, ss.ss_pattern(3, 4), 0, good, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_quant_lift_act(odd, 1, 16, 64, pat, 0, good, good, None) == ss.SS_ERR_ALIGNMENT
    assert L.ss_prune_act_2to4(good, 1, -1, 64, 0, good, good, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_prune_act_2to4(good, 1, 16, 64, 0, good, odd, good, None) == ss.SS_ERR_ALIGNMENT
    # weight compression: Wm required unless dense; rows too long for one CTA
    assert L.ss_compress_weight(good, 1, 64, 64, pat, 0, good, None, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_compress_weight(good, 1, 64, 1 << 20, pat, 0, good, good, good, None) \
        == ss.SS_ERR_UNSUPPORTED


@pytest.mark.parametrize("pat", ["dense", "2:4", "4:6", "6:8", "8:10"])
def test_fp4_shape_matches_oracle(pat):
    for K in [1, 2, 7, 64, 300, 1000, 4096, 4097, 14336]:
        assert ss.ss_fp4_shape(pat, K) == oracle.fp4_shape(pat, K)


def test_fp4_scale_bytes(L):
    """Tile-major scales: 128-row tiles, one byte per block of 16 or 32."""
    assert ss.ss_fp4_scale_bytes(1, 256, 16) == 128 * 16
    assert ss.ss_fp4_scale_bytes(129, 512, 32) == 256 * 16
    assert ss.ss_fp4_scale_bytes(300, 4096, 32) == 384 * 128
    for rows, K_lp, block in [(0, 256, 16), (1, 100, 16), (1, 128, 16), (1, 256, 8),
                              (-1, 256, 32)]:
        assert ss.ss_fp4_scale_bytes(rows, K_lp, block) == 0


def test_nvfp4_argument_errors_return_before_any_launch(L):
    """The NVFP4 calls validate shapes, pointers, dtypes and alignment before
    the device is touched."""
    vp = ctypes.c_void_p
    good = vp(0x10000)          # never dereferenced: every call below fails first
    odd = vp(0x10008)
    pat = ss.ss_pattern(6, 8)
    dense = ss.ss_pattern(0, 0)
    # weight: Wm required unless dense, bad dtype, bad size, misaligned
    assert L.ss_compress_weight_nvfp4(good, 1, 64, 64, pat, good, None, good, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_compress_weight_nvfp4(good, 2, 64, 64, pat, good, good, good, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_compress_weight_nvfp4(good, 1, 0, 64, dense, good, None, good, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_compress_weight_nvfp4(odd, 1, 64, 64, pat, good, good, good, good, None) \
        == ss.SS_ERR_ALIGNMENT
    assert L.ss_compress_weight_nvfp4(good, 1, 64, 64, ss.ss_pattern(3, 4), good, good, good,
                                      good, None) == ss.SS_ERR_INVALID_ARG
    # activation: block 16 or 32 only, NULL outputs, misaligned
    assert L.ss_quant_lift_act_nvfp4(good, 1, 16, 64, pat, 8, good, good, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_quant_lift_act_nvfp4(good, 1, 16, 64, pat, 32, good, None, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_quant_lift_act_nvfp4(good, 1, 0, 64, pat, 32, good, good, good, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_quant_lift_act_nvfp4(good, 1, 16, 64, pat, 32, good, good, odd, None) \
        == ss.SS_ERR_ALIGNMENT
    # GEMMs: K_lp a positive multiple of 256, metadata required for the sparse
    # one, out dtype, alignment
    assert L.ss_sparse_gemm_nvfp4(good, good, good, good, good, good, good, 16, 64, 128, good, 1,
                                  None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm_nvfp4(good, None, good, good, good, good, good, 16, 64, 256, good, 1,
                                  None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm_nvfp4(good, good, good, good, good, good, good, 0, 64, 256, good, 1,
                                  None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm_nvfp4(good, good, good, good, good, good, good, 16, 64, 256, good, 2,
                                  None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_sparse_gemm_nvfp4(good, good, good, good, odd, good, good, 16, 64, 256, good, 1,
                                  None) == ss.SS_ERR_ALIGNMENT
    assert L.ss_dense_gemm_nvfp4(good, good, good, good, good, good, 16, 64, 384, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_dense_gemm_nvfp4(good, good, None, good, good, good, 16, 64, 256, good, 1, None) \
        == ss.SS_ERR_INVALID_ARG
    assert L.ss_dense_gemm_nvfp4(good, good, good, good, good, good, 16, 64, 256, odd, 1, None) \
        == ss.SS_ERR_ALIGNMENT


@pytest.mark.parametrize("rows,K_lp", [(1, 128), (130, 384), (256, 1024), (300, 128)])
def test_metadata_storage_layout(L, rows, K_lp):
    """Tile-major selector storage: every byte sits where ss.h's formula puts
    it, padding rows are zero, and the buffer size is ss_meta_bytes()."""
    rng = np.random.default_rng(rows + K_lp)
    Am = rng.integers(0, 256, (rows, K_lp // 8), dtype=np.uint8)
    At = oracle.meta_to_tiles(Am, K_lp)
    assert At.shape == ss.meta_shape(rows, K_lp)
    assert At.size == ss.ss_meta_bytes(rows, K_lp)
    flat = At.reshape(-1)
    r, b = np.meshgrid(np.arange(rows), np.arange(K_lp // 8), indexing="ij")
    off = ((r // 128) * (K_lp // 128) + b // 16) * 2048 + (r % 128) * 16 + b % 16
    np.testing.assert_array_equal(flat[off], Am)
    mask = np.ones(flat.size, dtype=bool)
    mask[off.reshape(-1)] = False
    assert not flat[mask].any()                          # padding rows
    np.testing.assert_array_equal(oracle.meta_from_tiles(At, rows, K_lp), Am)


@pytest.mark.parametrize("rows,K_lp", [(16, 128), (130, 256), (300, 384)])
def test_metadata_storage_layout_bf16(rows, K_lp):
    """The bf16 tier's storage: the tile-major offset of ss.h taken at row
    (r & ~8) | (b & 2) << 2 and byte (b & ~2) | (r & 8) >> 2 -- rows r and
    r + 8 exchange the 2-byte halves of each 4-byte word."""
    rng = np.random.default_rng(rows * K_lp)
    Am = rng.integers(0, 256, (rows, K_lp // 8), dtype=np.uint8)
    At = oracle.meta_to_tiles(Am, K_lp, i16=True)
    assert At.shape == ss.meta_shape(rows, K_lp)
    flat = At.reshape(-1)
    r, b = np.meshgrid(np.arange(rows), np.arange(K_lp // 8), indexing="ij")
    r2 = (r & ~8) | ((b & 2) << 2)
    b2 = (b & ~2) | ((r & 8) >> 2)
    off = ((r2 // 128) * (K_lp // 128) + b2 // 16) * 2048 + (r2 % 128) * 16 + b2 % 16
    np.testing.assert_array_equal(flat[off], Am)
    mask = np.ones(flat.size, dtype=bool)
    mask[off.reshape(-1)] = False
    assert not flat[mask].any()
    np.testing.assert_array_equal(oracle.meta_from_tiles(At, rows, K_lp, i16=True), Am)
    # rows 0..7 keep the first half of each word and hold row r + 8's first half second
    if rows >= 16:
        np.testing.assert_array_equal(At[0, 0, 3, 0:2], Am[3, 0:2])
        np.testing.assert_array_equal(At[0, 0, 3, 2:4], Am[11, 0:2])
        np.testing.assert_array_equal(At[0, 0, 11, 0:2], Am[3, 2:4])


def test_meta_bytes_rejects_bad_shapes(L):
    assert ss.ss_meta_bytes(0, 128) == 0
    assert ss.ss_meta_bytes(5, 100) == 0
    assert ss.ss_meta_bytes(5, 0) == 0


def test_debug_hooks_reject_bad_arguments_before_the_device(L):
    """The test hooks validate their argument before touching the device:
    a wait limit outside 1 ms .. 60 s and a stage below -1 are refused."""
    assert L.ss_debug_set_wait_limit(999_999) == ss.SS_ERR_INVALID_ARG
    assert L.ss_debug_set_wait_limit(60_000_000_001) == ss.SS_ERR_INVALID_ARG
    assert L.ss_debug_skip_stage(-2) == ss.SS_ERR_INVALID_ARG


def test_stored_traffic_is_tied_to_the_sources():
    """bench.py reports a stored DRAM-traffic figure only while the CUDA
    sources hash as they did when it was captured."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    h = bench.csrc_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    for key, tr in bench.TRAFFIC.items():
        assert set(tr) == {"bytes", "profile", "sources", "csrc_hash"}, key
        assert len(bench.csrc_hash(tr["sources"])) == 16
        assert os.path.exists(os.path.join(ROOT, tr["profile"])), tr["profile"]
        assert tr["bytes"] > 0
