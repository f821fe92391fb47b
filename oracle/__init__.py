"""CPU oracle for structured-sparse quantized matmul -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it.

This module is argument marshalling around ``ssref.c`` (plain C, see the
citations there): numpy arrays in, numpy arrays out.  Inputs given as bf16 are
upcast to fp32 exactly before they reach the C code.

Pins (tests that tie each function to something other than itself) live in
``tests/test_oracle_*.py``; every function below has at least one.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

INT8 = 0
FP8_E4M3 = 1
BF16 = 2
NVFP4 = 3
OUT_F32 = 0
OUT_BF16 = 1

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        sig = {
            "ssref_slide_shape": [i32, i32, i64, p, p, p],
            "ssref_prune_mask": [p, i64, i64, i32, i32, p],
            "ssref_prune_pairwise_4of8": [p, i64, i64, p],
            "ssref_assign_windows": [p, i64, i64, i32, p],
            "ssref_compress_weight": [p, i64, i64, i32, i32, i32, p, p, p],
            "ssref_quant_lift_act": [p, i64, i64, i32, i32, i32, p, p],
            "ssref_prune_act_2to4": [p, i64, i64, i32, p, p, p],
            "ssref_decompress_2to4": [p, p, i64, i64, p],
            "ssref_matmul_q": [i32, p, p, p, p, i64, i64, i64, p, i64, i32, p],
            "ssref_matmul_acc": [i32, p, p, i64, i64, i64, p, p],
            "ssref_sparse_gemm": [i32, p, p, p, p, p, i64, i64, i64, i32, p, i64, i32, p],
            "ssref_quantize_value": [ctypes.c_float, ctypes.c_float, i32, p],
            "ssref_scale_from_absmax": [ctypes.c_float, i32, p, p],
            "ssref_compress_weight_bf16": [p, i64, i64, i32, i32, p, p],
            "ssref_lift_act_bf16": [p, i64, i64, i32, i32, p],
            "ssref_decompress_2to4_bf16": [p, p, i64, i64, p],
            "ssref_matmul_bf16": [p, p, i64, i64, i64, p, i64, i32, p],
            "ssref_sparse_gemm_bf16": [i32, p, p, p, i64, i64, i64, p, i64, i32, p],
            "ssref_fp4_shape": [i32, i32, i64, p, p],
            "ssref_prune_pairs": [p, i64, i64, i32, i32, p],
            "ssref_compress_weight_nvfp4": [p, i64, i64, i32, i32, p, p, p, p],
            "ssref_quant_nvfp4": [p, i64, i64, i32, i32, i32, p, p, p],
            "ssref_nvfp4_act_page": [p, i64, i64, i32, i32, p, p],
            "ssref_decode_sparse_nvfp4": [p, p, p, i64, i64, p],
            "ssref_decode_dense_nvfp4": [p, p, i64, i64, i32, p],
            "ssref_matmul_nvfp4": [p, p, p, p, i64, i64, i64, p, i64, i32, p],
        }
        for name, args in sig.items():
            fn = getattr(_lib, name)
            fn.argtypes = args
            fn.restype = i32
        _lib.ssref_e4m3_from_float.argtypes = [ctypes.c_float]
        _lib.ssref_e4m3_from_float.restype = ctypes.c_uint8
        _lib.ssref_e4m3_to_double.argtypes = [ctypes.c_uint8]
        _lib.ssref_e4m3_to_double.restype = ctypes.c_double
        _lib.ssref_bf16_from_float.argtypes = [ctypes.c_float]
        _lib.ssref_bf16_from_float.restype = ctypes.c_uint16
        _lib.ssref_bits_per_element.argtypes = [i32, i32]
        _lib.ssref_bits_per_element.restype = ctypes.c_double
        _lib.ssref_e2m1_from_float.argtypes = [ctypes.c_float]
        _lib.ssref_e2m1_from_float.restype = ctypes.c_uint8
        _lib.ssref_e2m1_to_double.argtypes = [ctypes.c_uint8]
        _lib.ssref_e2m1_to_double.restype = ctypes.c_double
        _lib.ssref_nvfp4_global.argtypes = [ctypes.c_float]
        _lib.ssref_nvfp4_global.restype = ctypes.c_float
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(st: int, what: str):
    if st != 0:
        raise OracleError(f"{what}: oracle status {st}")


def _f32(x) -> np.ndarray:
    """fp32 contiguous view; torch bf16/fp32 tensors are upcast exactly."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").float().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def pattern(p: str) -> tuple[int, int]:
    """'6:8' -> (6, 8); 'dense' -> (0, 0)."""
    if p == "dense":
        return 0, 0
    keep, group = (int(v) for v in p.split(":"))
    return keep, group


def slide_shape(p: str, K: int) -> tuple[int, int, int]:
    keep, group = pattern(p)
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ssref_slide_shape(keep, group, K, ctypes.byref(a), ctypes.byref(b),
                                   ctypes.byref(c)), "slide_shape")
    return a.value, b.value, c.value


def bits_per_element(value_bits: int, sparse_2to4: bool) -> float:
    return lib().ssref_bits_per_element(value_bits, int(sparse_2to4))


def e4m3_from_float(v: float) -> int:
    return int(lib().ssref_e4m3_from_float(float(v)))


def e4m3_to_float(b: int) -> float:
    return float(lib().ssref_e4m3_to_double(int(b)))


def e4m3_decode_array(a: np.ndarray) -> np.ndarray:
    table = np.array([e4m3_to_float(b) for b in range(256)], dtype=np.float64)
    return table[np.asarray(a, dtype=np.uint8)]


def bf16_from_float(v: float) -> int:
    return int(lib().ssref_bf16_from_float(float(v)))


def scale_from_absmax(a: float, qdtype: int) -> tuple[float, float]:
    inv, s = ctypes.c_float(), ctypes.c_float()
    _check(lib().ssref_scale_from_absmax(float(a), qdtype, ctypes.byref(inv), ctypes.byref(s)),
           "scale")
    return inv.value, s.value


def quantize_value(x: float, inv: float, qdtype: int) -> int:
    out = ctypes.c_uint8()
    _check(lib().ssref_quantize_value(float(x), float(inv), qdtype, ctypes.byref(out)), "quant")
    return out.value


def prune_mask(W, keep: int, group: int) -> np.ndarray:
    W = _f32(W)
    rows, K = W.shape
    K_pad = -(-K // group) * group
    mask = np.zeros((rows, K_pad), dtype=np.uint8)
    _check(lib().ssref_prune_mask(_ptr(W), rows, K, keep, group, _ptr(mask)), "prune_mask")
    return mask


def prune_pairwise_4of8(W) -> np.ndarray:
    W = _f32(W)
    rows, K = W.shape
    mask = np.zeros((rows, K), dtype=np.uint8)
    _check(lib().ssref_prune_pairwise_4of8(_ptr(W), rows, K, _ptr(mask)), "pairwise")
    return mask


def assign_windows(mask: np.ndarray, group: int) -> np.ndarray:
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    rows, K_pad = mask.shape
    win = np.zeros((rows, K_pad), dtype=np.int8)
    _check(lib().ssref_assign_windows(_ptr(mask), rows, K_pad, group, _ptr(win)),
           "assign_windows")
    return win


def compress_weight(W, p: str, qdtype: int):
    """-> (Wv, Wm, s_w); Wm is None for 'dense'."""
    W = _f32(W)
    N, K = W.shape
    keep, group = pattern(p)
    _, _, K_lp = slide_shape(p, K)
    if group == 0:
        Wv = np.zeros((N, K_lp), dtype=np.uint8)
        Wm = None
    else:
        Wv = np.zeros((N, K_lp // 2), dtype=np.uint8)
        Wm = np.zeros((N, K_lp // 8), dtype=np.uint8)
    s_w = np.zeros(N, dtype=np.float32)
    _check(lib().ssref_compress_weight(_ptr(W), N, K, keep, group, qdtype, _ptr(Wv), _ptr(Wm),
                                       _ptr(s_w)), "compress_weight")
    return Wv, Wm, s_w


def quant_lift_act(X, p: str, qdtype: int):
    """-> (Xq_lift [M, K_lp], s_x [M])."""
    X = _f32(X)
    M, K = X.shape
    keep, group = pattern(p)
    _, _, K_lp = slide_shape(p, K)
    Xq = np.zeros((M, K_lp), dtype=np.uint8)
    s_x = np.zeros(M, dtype=np.float32)
    _check(lib().ssref_quant_lift_act(_ptr(X), M, K, keep, group, qdtype, _ptr(Xq), _ptr(s_x)),
           "quant_lift_act")
    return Xq, s_x


def act_2to4_k_lp(K: int) -> int:
    return -(-(-(-K // 4) * 4) // 128) * 128


def prune_act_2to4(X, qdtype: int):
    """-> (Xv [M, K_lp/2], Xm [M, K_lp/8], s_x [M])."""
    X = _f32(X)
    M, K = X.shape
    K_lp = act_2to4_k_lp(K)
    Xv = np.zeros((M, K_lp // 2), dtype=np.uint8)
    Xm = np.zeros((M, K_lp // 8), dtype=np.uint8)
    s_x = np.zeros(M, dtype=np.float32)
    _check(lib().ssref_prune_act_2to4(_ptr(X), M, K, qdtype, _ptr(Xv), _ptr(Xm), _ptr(s_x)),
           "prune_act_2to4")
    return Xv, Xm, s_x


def decompress_2to4(Av: np.ndarray, Am: np.ndarray, K_lp: int) -> np.ndarray:
    Av = np.ascontiguousarray(Av, dtype=np.uint8)
    Am = np.ascontiguousarray(Am, dtype=np.uint8)
    rows = Av.shape[0]
    A = np.zeros((rows, K_lp), dtype=np.uint8)
    _check(lib().ssref_decompress_2to4(_ptr(Av), _ptr(Am), rows, K_lp, _ptr(A)), "decompress")
    return A


def _rows(m_idx, M):
    if m_idx is None:
        return None, M
    m_idx = np.ascontiguousarray(m_idx, dtype=np.int64)
    return m_idx, len(m_idx)


def _out(R, N, out_dtype):
    return np.zeros((R, N), dtype=np.float32 if out_dtype == OUT_F32 else np.uint16)


def matmul_q(qdtype: int, Xq, s_x, Wq, s_w, out_dtype: int, m_idx=None):
    """Y = dequant(Xq . Wq^T); bf16 output comes back as raw uint16 bits."""
    Xq = np.ascontiguousarray(Xq, dtype=np.uint8)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, K = Xq.shape
    N = Wq.shape[0]
    m_idx, R = _rows(m_idx, M)
    Y = _out(R, N, out_dtype)
    _check(lib().ssref_matmul_q(qdtype, _ptr(Xq), _ptr(s_x), _ptr(Wq), _ptr(s_w), M, N, K,
                                _ptr(m_idx), R, out_dtype, _ptr(Y)), "matmul_q")
    return Y


def matmul_acc(qdtype: int, Xq, Wq):
    """Raw accumulators: int64 for INT8, float64 for E4M3."""
    Xq = np.ascontiguousarray(Xq, dtype=np.uint8)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    M, K = Xq.shape
    N = Wq.shape[0]
    if qdtype == INT8:
        acc = np.zeros((M, N), dtype=np.int64)
        _check(lib().ssref_matmul_acc(qdtype, _ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), None),
               "matmul_acc")
    else:
        acc = np.zeros((M, N), dtype=np.float64)
        _check(lib().ssref_matmul_acc(qdtype, _ptr(Xq), _ptr(Wq), M, N, K, None, _ptr(acc)),
               "matmul_acc")
    return acc


def sparse_gemm(sparse_operand: int, Av, Am, s_a, B, s_b, M: int, N: int, K_lp: int,
                qdtype: int, out_dtype: int, m_idx=None):
    Av = np.ascontiguousarray(Av, dtype=np.uint8)
    Am = np.ascontiguousarray(Am, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_b = np.ascontiguousarray(s_b, dtype=np.float32)
    m_idx, R = _rows(m_idx, M)
    Y = _out(R, N, out_dtype)
    _check(lib().ssref_sparse_gemm(sparse_operand, _ptr(Av), _ptr(Am), _ptr(s_a), _ptr(B),
                                   _ptr(s_b), M, N, K_lp, qdtype, _ptr(m_idx), R, out_dtype,
                                   _ptr(Y)), "sparse_gemm")
    return Y


def dense_gemm(Xq, s_x, Wq, s_w, qdtype: int, out_dtype: int, m_idx=None):
    return matmul_q(qdtype, Xq, s_x, Wq, s_w, out_dtype, m_idx)


def plain_linear(W, X, p: str, qdtype: int, out_dtype: int, m_idx=None):
    """Path (i): prune W, quantise both operands, naive matmul over the
    original (zero-padded) K -- no decomposition, no lifting."""
    W = _f32(W)
    X = _f32(X)
    N, K = W.shape
    keep, group = pattern(p)
    if group:
        mask = prune_mask(W, keep, group)[:, :K]
        Wp = np.where(mask.astype(bool), W, np.float32(0))
    else:
        Wp = W
    Wq, _, s_w = compress_weight(Wp, "dense", qdtype)
    Xq, s_x = quant_lift_act(X, "dense", qdtype)
    return matmul_q(qdtype, Xq, s_x, Wq, s_w, out_dtype, m_idx)


def bf16_bits_to_float(y: np.ndarray) -> np.ndarray:
    return (np.asarray(y, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ storage layout

def _swap_r8_halves(At: np.ndarray) -> np.ndarray:
    """Inside each 2 KB block [128 rows][16 bytes], exchange row bit 3 with
    byte bit 1: the 2-byte half h of 4-byte word c of row 16a + 8x + r goes to
    row 16a + 8h + r, half x of word c (its own inverse)."""
    rt, kt = At.shape[:2]
    # [rt, kt, a, x, r, c, h, byte]
    v = At.reshape(rt, kt, 8, 2, 8, 4, 2, 2)
    return np.ascontiguousarray(v.transpose(0, 1, 2, 6, 4, 5, 3, 7).reshape(rt, kt, 128, 16))


def meta_to_tiles(Am: np.ndarray, K_lp: int, i16: bool = False) -> np.ndarray:
    """Row-layout selectors [rows, K_lp/8] -> the library's tile-major storage
    [ceil(rows/128), K_lp/128, 128, 16]: block (row tile, K tile) holds the 16
    selector bytes of 128 lifted K for each of the tile's 128 rows; padding
    rows are zero.  With i16 (the bf16 tier) the 2-byte halves of rows r and
    r + 8 of each 16-row group are exchanged as well (_swap_r8_halves).  A
    pure relabelling of bytes (no arithmetic), used to hand oracle metadata to
    the GPU and to compare the GPU's metadata with it."""
    Am = np.ascontiguousarray(Am, dtype=np.uint8)
    rows, nb = Am.shape
    assert nb == K_lp // 8 and K_lp % 128 == 0
    rt = (rows + 127) // 128
    padded = np.zeros((rt * 128, nb), dtype=np.uint8)
    padded[:rows] = Am
    # [row tile, row in tile, K tile, byte in K tile] -> [row tile, K tile, row, byte]
    At = np.ascontiguousarray(padded.reshape(rt, 128, K_lp // 128, 16).transpose(0, 2, 1, 3))
    return _swap_r8_halves(At) if i16 else At


def meta_from_tiles(At: np.ndarray, rows: int, K_lp: int, i16: bool = False) -> np.ndarray:
    """Inverse of meta_to_tiles: tile-major storage -> [rows, K_lp/8]."""
    At = np.ascontiguousarray(At, dtype=np.uint8)
    rt = (rows + 127) // 128
    At = At.reshape(rt, K_lp // 128, 128, 16)
    if i16:
        At = _swap_r8_halves(At)
    return np.ascontiguousarray(At.transpose(0, 2, 1, 3).reshape(rt * 128, K_lp // 8)[:rows])


# ---------------------------------------------------------------- bf16 tier

def compress_weight_bf16(W, p: str):
    """-> (Wv uint16 bf16 bits, Wm); Wv is [N, K_lp] for 'dense', else [N, K_lp/2]."""
    W = _f32(W)
    N, K = W.shape
    keep, group = pattern(p)
    _, _, K_lp = slide_shape(p, K)
    if group == 0:
        Wv = np.zeros((N, K_lp), dtype=np.uint16)
        Wm = None
    else:
        Wv = np.zeros((N, K_lp // 2), dtype=np.uint16)
        Wm = np.zeros((N, K_lp // 8), dtype=np.uint8)
    _check(lib().ssref_compress_weight_bf16(_ptr(W), N, K, keep, group, _ptr(Wv), _ptr(Wm)),
           "compress_weight_bf16")
    return Wv, Wm


def lift_act_bf16(X, p: str):
    """-> Xl [M, K_lp] uint16 bf16 bits."""
    X = _f32(X)
    M, K = X.shape
    keep, group = pattern(p)
    _, _, K_lp = slide_shape(p, K)
    Xl = np.zeros((M, K_lp), dtype=np.uint16)
    _check(lib().ssref_lift_act_bf16(_ptr(X), M, K, keep, group, _ptr(Xl)), "lift_act_bf16")
    return Xl


def decompress_2to4_bf16(Av: np.ndarray, Am: np.ndarray, K_lp: int) -> np.ndarray:
    Av = np.ascontiguousarray(Av, dtype=np.uint16)
    Am = np.ascontiguousarray(Am, dtype=np.uint8)
    rows = Av.shape[0]
    A = np.zeros((rows, K_lp), dtype=np.uint16)
    _check(lib().ssref_decompress_2to4_bf16(_ptr(Av), _ptr(Am), rows, K_lp, _ptr(A)),
           "decompress_bf16")
    return A


def matmul_bf16(X, W, out_dtype: int, m_idx=None):
    """Y = round_f32(X . W^T) over bf16 bits, double accumulation."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    W = np.ascontiguousarray(W, dtype=np.uint16)
    M, K = X.shape
    N = W.shape[0]
    m_idx, R = _rows(m_idx, M)
    Y = _out(R, N, out_dtype)
    _check(lib().ssref_matmul_bf16(_ptr(X), _ptr(W), M, N, K, _ptr(m_idx), R, out_dtype,
                                   _ptr(Y)), "matmul_bf16")
    return Y


def sparse_gemm_bf16(sparse_operand: int, Av, Am, B, M: int, N: int, K_lp: int,
                     out_dtype: int, m_idx=None):
    Av = np.ascontiguousarray(Av, dtype=np.uint16)
    Am = np.ascontiguousarray(Am, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    m_idx, R = _rows(m_idx, M)
    Y = _out(R, N, out_dtype)
    _check(lib().ssref_sparse_gemm_bf16(sparse_operand, _ptr(Av), _ptr(Am), _ptr(B), M, N, K_lp,
                                        _ptr(m_idx), R, out_dtype, _ptr(Y)), "sparse_gemm_bf16")
    return Y


def plain_linear_bf16(W, X, p: str, out_dtype: int, m_idx=None):
    """Prune W, round both operands to bf16, naive matmul over the original K."""
    W = _f32(W)
    X = _f32(X)
    keep, group = pattern(p)
    if group:
        mask = prune_mask(W, keep, group)[:, :W.shape[1]]
        W = np.where(mask.astype(bool), W, np.float32(0))
    Wb, _ = compress_weight_bf16(W, "dense")
    Xb = lift_act_bf16(X, "dense")
    return matmul_bf16(Xb, Wb, out_dtype, m_idx)


def prune_act_2to4_bf16(X):
    """Online 2:4 prune of an activation in the bf16 tier -> (Xv bf16 bits,
    Xm).  With no scale, this is the 2:4 weight compression applied to the
    token rows: the same magnitude ranking, tie rule and packing."""
    return compress_weight_bf16(X, "2:4")



# ---------------------------------------------------------------- NVFP4 (pairs)

def e2m1_from_float(v: float) -> int:
    return int(lib().ssref_e2m1_from_float(float(v)))


def e2m1_to_float(c: int) -> float:
    return float(lib().ssref_e2m1_to_double(int(c)))


def nvfp4_global(amax: float) -> float:
    return float(lib().ssref_nvfp4_global(float(amax)))


def fp4_shape(p: str, K: int) -> tuple[int, int]:
    """(K_lift, K_lp) in elements for pattern p counted in pairs."""
    keep, group = pattern(p)
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ssref_fp4_shape(keep, group, K, ctypes.byref(a), ctypes.byref(b)), "fp4_shape")
    return a.value, b.value


def prune_pairs(W, keep: int, group: int) -> np.ndarray:
    """Pair mask [rows, P_pad] (P = ceil(K/2) pairs)."""
    W = _f32(W)
    rows, K = W.shape
    P = (K + 1) // 2
    P_pad = -(-P // group) * group
    mask = np.zeros((rows, P_pad), dtype=np.uint8)
    _check(lib().ssref_prune_pairs(_ptr(W), rows, K, keep, group, _ptr(mask)), "prune_pairs")
    return mask


def compress_weight_nvfp4(W, p: str):
    """-> (Wv [N, K_lp/4] bytes, Wm [N, K_lp/16], Ws [N, K_lp/32] UE4M3, g_w)."""
    W = _f32(W)
    N, K = W.shape
    keep, group = pattern(p)
    _, K_lp = fp4_shape(p, K)
    Wv = np.zeros((N, K_lp // 4), dtype=np.uint8)
    Wm = np.zeros((N, K_lp // 16), dtype=np.uint8)
    Ws = np.zeros((N, K_lp // 32), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    _check(lib().ssref_compress_weight_nvfp4(_ptr(W), N, K, keep, group, _ptr(Wv), _ptr(Wm),
                                             _ptr(Ws), _ptr(g)), "compress_weight_nvfp4")
    return Wv, Wm, Ws, float(g[0])


def quant_nvfp4(X, p: str, block: int):
    """Dense NVFP4 matrix (lifted on pairs for a pattern) with one global
    scale for the whole tensor -> (Xv [rows, K_lp/2] bytes, Xs [rows,
    K_lp/block] UE4M3, g [1])."""
    X = _f32(X)
    rows, K = X.shape
    keep, group = pattern(p)
    _, K_lp = fp4_shape(p, K)
    Xv = np.zeros((rows, K_lp // 2), dtype=np.uint8)
    Xs = np.zeros((rows, K_lp // block), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    _check(lib().ssref_quant_nvfp4(_ptr(X), rows, K, keep, group, block, _ptr(Xv), _ptr(Xs),
                                   _ptr(g)), "quant_nvfp4")
    return Xv, Xs, g


def nvfp4_act_page(X, p: str):
    """The activation as the NVFP4 definition has it (16-element groups along
    the original K, one global scale), decoded without the global scale and
    lifted to K_lp -> (Xlift [rows, K_lp] float64, g [1])."""
    X = _f32(X)
    rows, K = X.shape
    keep, group = pattern(p)
    _, K_lp = fp4_shape(p, K)
    Xl = np.zeros((rows, K_lp), dtype=np.float64)
    g = np.zeros(1, dtype=np.float32)
    _check(lib().ssref_nvfp4_act_page(_ptr(X), rows, K, keep, group, _ptr(Xl), _ptr(g)),
           "nvfp4_act_page")
    return Xl, g


def decode_sparse_nvfp4(Av, Am, As, K_lp: int) -> np.ndarray:
    Av = np.ascontiguousarray(Av, dtype=np.uint8)
    rows = Av.shape[0]
    A = np.zeros((rows, K_lp), dtype=np.float64)
    _check(lib().ssref_decode_sparse_nvfp4(_ptr(Av), _ptr(np.ascontiguousarray(Am, np.uint8)),
                                           _ptr(np.ascontiguousarray(As, np.uint8)), rows, K_lp,
                                           _ptr(A)), "decode_sparse_nvfp4")
    return A


def decode_dense_nvfp4(Xv, Xs, K_lp: int, block: int) -> np.ndarray:
    Xv = np.ascontiguousarray(Xv, dtype=np.uint8)
    rows = Xv.shape[0]
    X = np.zeros((rows, K_lp), dtype=np.float64)
    _check(lib().ssref_decode_dense_nvfp4(_ptr(Xv), _ptr(np.ascontiguousarray(Xs, np.uint8)),
                                          rows, K_lp, block, _ptr(X)), "decode_dense_nvfp4")
    return X


def matmul_nvfp4(Xd, g_x, Wd, g_w, out_dtype: int, m_idx=None):
    """Y = ((float)(Xd . Wd^T) * g_x) * g_w[n] over decoded operands (g_x one
    value for the tensor, or one per row)."""
    Xd = np.ascontiguousarray(Xd, dtype=np.float64)
    Wd = np.ascontiguousarray(Wd, dtype=np.float64)
    M, K = Xd.shape
    g_x = np.ascontiguousarray(np.broadcast_to(np.asarray(g_x, dtype=np.float32).reshape(-1), (M,)))
    g_w = np.ascontiguousarray(g_w, dtype=np.float32)
    N = Wd.shape[0]
    m_idx, R = _rows(m_idx, M)
    Y = _out(R, N, out_dtype)
    _check(lib().ssref_matmul_nvfp4(_ptr(Xd), _ptr(g_x), _ptr(Wd), _ptr(g_w), M, N, K,
                                    _ptr(m_idx), R, out_dtype, _ptr(Y)), "matmul_nvfp4")
    return Y


def sparse_gemm_nvfp4(Wv, Wm, Ws, g_w: float, Xv, Xs, g_x, M: int, N: int, K_lp: int,
                      out_dtype: int, m_idx=None):
    """The sparse NVFP4 product: decoded W (2 kept pairs per window of 4,
    16-value blocks) against decoded lifted X (32-element blocks)."""
    Wd = decode_sparse_nvfp4(Wv, Wm, Ws, K_lp)
    Xd = decode_dense_nvfp4(Xv, Xs, K_lp, 32)
    return matmul_nvfp4(Xd, g_x, Wd, np.full(N, g_w, dtype=np.float32), out_dtype, m_idx)


def sparse_gemm_nvfp4_page(Wv, Wm, Ws, g_w: float, X, p: str, out_dtype: int, m_idx=None):
    """The same product with the activation quantised as the NVFP4 definition
    has it (nvfp4_act_page: 16-element groups along the original K)."""
    N = Wv.shape[0]
    K_lp = Wv.shape[1] * 4
    Xl, g_x = nvfp4_act_page(X, p)
    Wd = decode_sparse_nvfp4(Wv, Wm, Ws, K_lp)
    return matmul_nvfp4(Xl, g_x, Wd, np.full(N, g_w, dtype=np.float32), out_dtype, m_idx)


def dense_gemm_nvfp4(Xv, Xs, g_x, Wv, Ws, g_w, out_dtype: int, m_idx=None):
    """The dense NVFP4 comparator (16-element blocks on both operands)."""
    K_lp = Xv.shape[1] * 2
    Xd = decode_dense_nvfp4(Xv, Xs, K_lp, 16)
    Wd = decode_dense_nvfp4(Wv, Ws, K_lp, 16)
    g_w = np.ascontiguousarray(g_w, dtype=np.float32)
    return matmul_nvfp4(Xd, g_x, Wd, np.broadcast_to(g_w, (Wd.shape[0],)).copy(), out_dtype,
                        m_idx)


def scales_to_tiles(S: np.ndarray, K_lp: int, block: int) -> np.ndarray:
    """Row-layout UE4M3 scales [rows, K_lp/block] -> the library's tile-major
    storage: 512-byte blocks of 128 rows x 4 consecutive scales, inside a
    block byte (r % 32) * 16 + ((r % 128) / 32) * 4 + j % 4 (the source shape
    of the tensor-memory copy); rows padded to 128 with zeros.  A pure
    relabelling of bytes."""
    S = np.ascontiguousarray(S, dtype=np.uint8)
    rows, nblk = S.shape
    assert nblk == K_lp // block and nblk % 4 == 0
    rt = (rows + 127) // 128
    P = np.zeros((rt * 128, nblk), dtype=np.uint8)
    P[:rows] = S
    # [rt, q (row/32 % 4), l (row % 32), kb (j/4), s (j%4)] -> [rt, kb, l, q, s]
    T = P.reshape(rt, 4, 32, nblk // 4, 4).transpose(0, 3, 2, 1, 4)
    return np.ascontiguousarray(T).reshape(-1)
