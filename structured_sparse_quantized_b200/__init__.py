"""structured_sparse_quantized_b200 -- Python binding of libss.

Quantized (INT8 / FP8-E4M3, and the unscaled BF16 tier) matmul on the
Blackwell sparse tensor cores for
structured-sparse weights: hardware 2:4 and the milder (2Nh-2):2Nh patterns
(4:6, 6:8, 8:10) brought to 2:4 by SlideSparse's sliding-window
decomposition.  Every step runs in the CUDA kernels of ``libss.so`` (see
``include/ss.h``); this module only marshals arguments: torch tensors supply
device memory and streams, and each ``ss_*`` function here calls the C
function of the same name.  There is no CPU fallback: if ``libss.so`` is
missing, or the device is not sm_100, calls raise ``SSError``.

Low-level calls (same names and argument order as the C ABI, outputs
preallocated by the caller):
    ss_parse_pattern, ss_slide_shape, ss_act_2to4_shape, ss_compress_weight,
    ss_quant_lift_act, ss_prune_act_2to4, ss_sparse_gemm, ss_dense_gemm,
    ss_get_device_status, ss_status_string, ss_kernel_launches, ss_meta_bytes,
    ss_debug_set_wait_limit, ss_debug_skip_stage (test hooks),
    ss_fp4_shape, ss_fp4_scale_bytes, ss_compress_weight_nvfp4,
    ss_quant_lift_act_nvfp4, ss_sparse_gemm_nvfp4, ss_dense_gemm_nvfp4
Convenience wrappers that allocate their outputs with torch:
    compress_weight, quant_lift_act, prune_act_2to4, sparse_gemm, dense_gemm,
    linear, and for NVFP4 compress_weight_nvfp4, quant_lift_act_nvfp4,
    sparse_gemm_nvfp4, dense_gemm_nvfp4, linear_nvfp4
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libss.so")

SS_OK = 0
SS_ERR_INVALID_ARG = 1
SS_ERR_UNSUPPORTED = 2
SS_ERR_ALIGNMENT = 3
SS_ERR_ARCH = 4
SS_ERR_CUDA = 5
SS_ERR_TIMEOUT = 6
SS_ERR_DATA = 7

SS_IN_F32, SS_IN_BF16 = 0, 1
SS_INT8, SS_FP8_E4M3, SS_BF16 = 0, 1, 2
SS_OUT_F32, SS_OUT_BF16 = 0, 1

QDTYPES = {"int8": SS_INT8, "fp8": SS_FP8_E4M3, "e4m3": SS_FP8_E4M3, "bf16": SS_BF16}


class SSError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {ss_status_string(status)} ({status})")
        self.status = status


class ss_pattern(ctypes.Structure):
    _fields_ = [("keep", ctypes.c_int32), ("group", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libss.so (built by ``python -m structured_sparse_quantized_b200._build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libss.so is not built ({LIB_PATH}); run "
                           "`python -m structured_sparse_quantized_b200._build`")
    L = ctypes.CDLL(LIB_PATH)
    i64, i32, p, f = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_float
    pat = ss_pattern
    sigs = {
        "ss_parse_pattern": [ctypes.c_char_p, ctypes.POINTER(pat)],
        "ss_slide_shape": [pat, i64, ctypes.POINTER(i64), ctypes.POINTER(i64),
                           ctypes.POINTER(i64)],
        "ss_act_2to4_shape": [i64, ctypes.POINTER(i64)],
        "ss_compress_weight": [p, i32, i64, i64, pat, i32, p, p, p, p],
        "ss_quant_lift_act": [p, i32, i64, i64, pat, i32, p, p, p],
        "ss_prune_act_2to4": [p, i32, i64, i64, i32, p, p, p, p],
        "ss_sparse_gemm": [i32, p, p, p, p, p, i64, i64, i64, i32, p, i32, p],
        "ss_dense_gemm": [p, p, p, p, i64, i64, i64, i32, p, i32, p],
        "ss_get_device_status": [p],
        "ss_debug_set_wait_limit": [ctypes.c_uint64],
        "ss_debug_skip_stage": [i32],
        "ss_fp4_shape": [pat, i64, ctypes.POINTER(i64), ctypes.POINTER(i64)],
        "ss_compress_weight_nvfp4": [p, i32, i64, i64, pat, p, p, p, p, p],
        "ss_quant_lift_act_nvfp4": [p, i32, i64, i64, pat, i32, p, p, p, p],
        "ss_sparse_gemm_nvfp4": [p, p, p, p, p, p, p, i64, i64, i64, p, i32, p],
        "ss_dense_gemm_nvfp4": [p, p, p, p, p, p, i64, i64, i64, p, i32, p],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = i32
    L.ss_status_string.argtypes = [i32]
    L.ss_status_string.restype = ctypes.c_char_p
    L.ss_kernel_launches.argtypes = []
    L.ss_kernel_launches.restype = i64
    L.ss_meta_bytes.argtypes = [i64, i64]
    L.ss_meta_bytes.restype = i64
    L.ss_fp4_scale_bytes.argtypes = [i64, i64, i32]
    L.ss_fp4_scale_bytes.restype = i64
    del f
    _lib = L
    return L


def ss_status_string(status: int) -> str:
    return lib().ss_status_string(int(status)).decode()


def ss_kernel_launches() -> int:
    return int(lib().ss_kernel_launches())


def _check(status: int, where: str) -> None:
    if status != SS_OK:
        raise SSError(status, where)


# ------------------------------------------------------------------ marshalling

def _pattern(p) -> ss_pattern:
    if isinstance(p, ss_pattern):
        return p
    out = ss_pattern()
    _check(lib().ss_parse_pattern(str(p).encode(), ctypes.byref(out)), "ss_parse_pattern")
    return out


def _qdtype(q) -> int:
    return QDTYPES[q] if isinstance(q, str) else int(q)


def _dev(t: torch.Tensor | None, name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _in_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SS_IN_BF16
    if t.dtype == torch.float32:
        return SS_IN_F32
    raise ValueError(f"input dtype {t.dtype} not supported (float32 or bfloat16)")


def _out_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SS_OUT_BF16
    if t.dtype == torch.float32:
        return SS_OUT_F32
    raise ValueError(f"output dtype {t.dtype} not supported (float32 or bfloat16)")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


# ------------------------------------------------------------------ C ABI, 1:1

def ss_parse_pattern(s: str) -> tuple[int, int]:
    p = _pattern(s)
    return p.keep, p.group


def ss_slide_shape(pattern, K: int) -> tuple[int, int, int]:
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ss_slide_shape(_pattern(pattern), int(K), ctypes.byref(a), ctypes.byref(b),
                                ctypes.byref(c)), "ss_slide_shape")
    return a.value, b.value, c.value


def ss_act_2to4_shape(K: int) -> int:
    a = ctypes.c_int64()
    _check(lib().ss_act_2to4_shape(int(K), ctypes.byref(a)), "ss_act_2to4_shape")
    return a.value


def ss_meta_bytes(rows: int, K_lp: int) -> int:
    return int(lib().ss_meta_bytes(int(rows), int(K_lp)))


def meta_shape(rows: int, K_lp: int) -> tuple:
    """Shape of a tile-major metadata buffer: [row tiles, K tiles, 128, 16]
    (one 2 KB block of 2:4 selectors per 128 rows x 128 lifted K)."""
    return ((rows + 127) // 128, K_lp // 128, 128, 16)


def ss_compress_weight(W, pattern, q, Wv, Wm, s_w, stream=None) -> None:
    N, K = W.shape
    _check(lib().ss_compress_weight(_dev(W, "W"), _in_dtype(W), N, K, _pattern(pattern),
                                    _qdtype(q), _dev(Wv, "Wv"), _dev(Wm, "Wm"),
                                    _dev(s_w, "s_w"), _stream(stream)), "ss_compress_weight")


def ss_quant_lift_act(X, pattern, q, Xq_lift, s_x, stream=None) -> None:
    M, K = X.shape
    _check(lib().ss_quant_lift_act(_dev(X, "X"), _in_dtype(X), M, K, _pattern(pattern),
                                   _qdtype(q), _dev(Xq_lift, "Xq_lift"), _dev(s_x, "s_x"),
                                   _stream(stream)), "ss_quant_lift_act")


def ss_prune_act_2to4(X, q, Xv, Xm, s_x, stream=None) -> None:
    M, K = X.shape
    _check(lib().ss_prune_act_2to4(_dev(X, "X"), _in_dtype(X), M, K, _qdtype(q),
                                   _dev(Xv, "Xv"), _dev(Xm, "Xm"), _dev(s_x, "s_x"),
                                   _stream(stream)), "ss_prune_act_2to4")


def ss_sparse_gemm(sparse_operand: int, Av, Am, s_a, B, s_b, M: int, N: int, K_lp: int, q, Y,
                   stream=None) -> None:
    _check(lib().ss_sparse_gemm(int(sparse_operand), _dev(Av, "Av"), _dev(Am, "Am"),
                                _dev(s_a, "s_a"), _dev(B, "B"), _dev(s_b, "s_b"), int(M), int(N),
                                int(K_lp), _qdtype(q), _dev(Y, "Y"), _out_dtype(Y),
                                _stream(stream)), "ss_sparse_gemm")


def ss_dense_gemm(Xq, s_x, Wq, s_w, M: int, N: int, K_p: int, q, Y, stream=None) -> None:
    _check(lib().ss_dense_gemm(_dev(Xq, "Xq"), _dev(s_x, "s_x"), _dev(Wq, "Wq"),
                               _dev(s_w, "s_w"), int(M), int(N), int(K_p), _qdtype(q),
                               _dev(Y, "Y"), _out_dtype(Y), _stream(stream)), "ss_dense_gemm")


def ss_get_device_status(stream=None) -> int:
    return int(lib().ss_get_device_status(_stream(stream)))


def ss_debug_set_wait_limit(ns: int) -> None:
    """Test hook: device-side waits give up after `ns` nanoseconds (4 s default)."""
    _check(lib().ss_debug_set_wait_limit(int(ns)), "ss_debug_set_wait_limit")


def ss_debug_skip_stage(kb: int) -> None:
    """Test hook: GEMM producers skip K stage `kb` of their first tile (-1: off)."""
    _check(lib().ss_debug_skip_stage(int(kb)), "ss_debug_skip_stage")


# ------------------------------------------------------------------ allocating wrappers
# Stored values are uint8 codes for the 8-bit tiers and bfloat16 for the bf16
# tier, which has no scales (its s_* entries are None).

def _vals_dtype(q) -> torch.dtype:
    return torch.bfloat16 if _qdtype(q) == SS_BF16 else torch.uint8


def _scales(n: int, q, dev):
    return None if _qdtype(q) == SS_BF16 else torch.empty(n, dtype=torch.float32, device=dev)


def compress_weight(W: torch.Tensor, pattern, q, stream=None):
    """-> (Wv, Wm, s_w); Wm is None for 'dense'."""
    N, K = W.shape
    p = _pattern(pattern)
    _, _, K_lp = ss_slide_shape(p, K)
    dev = W.device
    vd = _vals_dtype(q)
    if p.group == 0:
        Wv = torch.empty((N, K_lp), dtype=vd, device=dev)
        Wm = None
    else:
        Wv = torch.empty((N, K_lp // 2), dtype=vd, device=dev)
        Wm = torch.empty(meta_shape(N, K_lp), dtype=torch.uint8, device=dev)
    s_w = _scales(N, q, dev)
    ss_compress_weight(W, p, q, Wv, Wm, s_w, stream)
    return Wv, Wm, s_w


def quant_lift_act(X: torch.Tensor, pattern, q, stream=None, out=None):
    M, K = X.shape
    p = _pattern(pattern)
    _, _, K_lp = ss_slide_shape(p, K)
    if out is None:
        out = (torch.empty((M, K_lp), dtype=_vals_dtype(q), device=X.device),
               _scales(M, q, X.device))
    ss_quant_lift_act(X, p, q, out[0], out[1], stream)
    return out


def prune_act_2to4(X: torch.Tensor, q, stream=None, out=None):
    M, K = X.shape
    K_lp = ss_act_2to4_shape(K)
    if out is None:
        out = (torch.empty((M, K_lp // 2), dtype=_vals_dtype(q), device=X.device),
               torch.empty(meta_shape(M, K_lp), dtype=torch.uint8, device=X.device),
               _scales(M, q, X.device))
    ss_prune_act_2to4(X, q, out[0], out[1], out[2], stream)
    return out


def sparse_gemm(sparse_operand: int, Av, Am, s_a, B, s_b, M: int, N: int, q,
                out_dtype=torch.bfloat16, stream=None, out=None):
    K_lp = Av.shape[1] * 2
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=Av.device)
    ss_sparse_gemm(sparse_operand, Av, Am, s_a, B, s_b, M, N, K_lp, q, out, stream)
    return out


def dense_gemm(Xq, s_x, Wq, s_w, q, out_dtype=torch.bfloat16, stream=None, out=None):
    M, K_p = Xq.shape
    N = Wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=Xq.device)
    ss_dense_gemm(Xq, s_x, Wq, s_w, M, N, K_p, q, out, stream)
    return out


def linear(X: torch.Tensor, packed, pattern, q, out_dtype=torch.bfloat16, stream=None):
    """Y = X W^T through the weight-sparse path: quant+lift, then the sparse
    GEMM (or the dense GEMM for pattern 'dense').  `packed` = compress_weight()."""
    Wv, Wm, s_w = packed
    M = X.shape[0]
    N = Wv.shape[0]
    Xq, s_x = quant_lift_act(X, pattern, q, stream)
    if _pattern(pattern).group == 0:
        return dense_gemm(Xq, s_x, Wv, s_w, q, out_dtype, stream)
    return sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, M, N, q, out_dtype, stream)


# ------------------------------------------------------------------ NVFP4 (pairwise sparse FP4)
# Patterns count pairs of adjacent elements ("2:4" = the hardware's pairwise
# 4:8).  Values are packed E2M1 codes (uint8, two per byte), local scales
# UE4M3 bytes in the tile-major layout of ss_fp4_scale_bytes, global scales
# fp32 (one per weight tensor, one per token).

def ss_fp4_shape(pattern, K: int) -> tuple[int, int]:
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().ss_fp4_shape(_pattern(pattern), int(K), ctypes.byref(a), ctypes.byref(b)),
           "ss_fp4_shape")
    return a.value, b.value


def ss_fp4_scale_bytes(rows: int, K_lp: int, block: int) -> int:
    return int(lib().ss_fp4_scale_bytes(int(rows), int(K_lp), int(block)))


def ss_compress_weight_nvfp4(W, pattern, Wv, Wm, Ws, g_w, stream=None) -> None:
    N, K = W.shape
    _check(lib().ss_compress_weight_nvfp4(_dev(W, "W"), _in_dtype(W), N, K, _pattern(pattern),
                                          _dev(Wv, "Wv"), _dev(Wm, "Wm"), _dev(Ws, "Ws"),
                                          _dev(g_w, "g_w"), _stream(stream)),
           "ss_compress_weight_nvfp4")


def ss_quant_lift_act_nvfp4(X, pattern, block: int, Xv, Xs, g_x, stream=None) -> None:
    M, K = X.shape
    _check(lib().ss_quant_lift_act_nvfp4(_dev(X, "X"), _in_dtype(X), M, K, _pattern(pattern),
                                         int(block), _dev(Xv, "Xv"), _dev(Xs, "Xs"),
                                         _dev(g_x, "g_x"), _stream(stream)),
           "ss_quant_lift_act_nvfp4")


def ss_sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M: int, N: int, K_lp: int, Y,
                         stream=None) -> None:
    _check(lib().ss_sparse_gemm_nvfp4(_dev(Wv, "Wv"), _dev(Wm, "Wm"), _dev(Ws, "Ws"),
                                      _dev(g_w, "g_w"), _dev(Xv, "Xv"), _dev(Xs, "Xs"),
                                      _dev(g_x, "g_x"), int(M), int(N), int(K_lp), _dev(Y, "Y"),
                                      _out_dtype(Y), _stream(stream)), "ss_sparse_gemm_nvfp4")


def ss_dense_gemm_nvfp4(Xv, Xs, g_x, Wv, Ws, g_w, M: int, N: int, K_p: int, Y,
                        stream=None) -> None:
    _check(lib().ss_dense_gemm_nvfp4(_dev(Xv, "Xv"), _dev(Xs, "Xs"), _dev(g_x, "g_x"),
                                     _dev(Wv, "Wv"), _dev(Ws, "Ws"), _dev(g_w, "g_w"), int(M),
                                     int(N), int(K_p), _dev(Y, "Y"), _out_dtype(Y),
                                     _stream(stream)), "ss_dense_gemm_nvfp4")


def compress_weight_nvfp4(W: torch.Tensor, pattern, stream=None):
    """-> (Wv, Wm, Ws, g_w); Wm is None for 'dense' (blocks of 16)."""
    N, K = W.shape
    p = _pattern(pattern)
    _, K_lp = ss_fp4_shape(p, K)
    dev = W.device
    if p.group == 0:
        Wv = torch.empty((N, K_lp // 2), dtype=torch.uint8, device=dev)
        Wm = None
        Ws = torch.empty(ss_fp4_scale_bytes(N, K_lp, 16), dtype=torch.uint8, device=dev)
    else:
        Wv = torch.empty((N, K_lp // 4), dtype=torch.uint8, device=dev)
        Wm = torch.empty(meta_shape(N, K_lp // 2), dtype=torch.uint8, device=dev)
        Ws = torch.empty(ss_fp4_scale_bytes(N, K_lp, 32), dtype=torch.uint8, device=dev)
    g_w = torch.empty(4, dtype=torch.float32, device=dev)   # [0] is the global scale
    ss_compress_weight_nvfp4(W, p, Wv, Wm, Ws, g_w, stream)
    return Wv, Wm, Ws, g_w


def quant_lift_act_nvfp4(X: torch.Tensor, pattern, block: int, stream=None, out=None):
    """-> (Xv [M, K_lp/2] uint8, Xs scale bytes, g_x: [0] is the tensor's global scale)."""
    M, K = X.shape
    p = _pattern(pattern)
    _, K_lp = ss_fp4_shape(p, K)
    if out is None:
        out = (torch.empty((M, K_lp // 2), dtype=torch.uint8, device=X.device),
               torch.empty(ss_fp4_scale_bytes(M, K_lp, block), dtype=torch.uint8, device=X.device),
               torch.empty(4, dtype=torch.float32, device=X.device))
    ss_quant_lift_act_nvfp4(X, p, block, out[0], out[1], out[2], stream)
    return out


def sparse_gemm_nvfp4(packed, act, M: int, N: int, out_dtype=torch.bfloat16, stream=None,
                      out=None):
    Wv, Wm, Ws, g_w = packed
    Xv, Xs, g_x = act
    K_lp = Xv.shape[1] * 2
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=Xv.device)
    ss_sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp, out, stream)
    return out


def dense_gemm_nvfp4(act, packed, M: int, N: int, out_dtype=torch.bfloat16, stream=None,
                     out=None):
    Xv, Xs, g_x = act
    Wv, _, Ws, g_w = packed
    K_p = Xv.shape[1] * 2
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=Xv.device)
    ss_dense_gemm_nvfp4(Xv, Xs, g_x, Wv, Ws, g_w, M, N, K_p, out, stream)
    return out


def linear_nvfp4(X: torch.Tensor, packed, pattern, out_dtype=torch.bfloat16, stream=None):
    """Y = X W^T in NVFP4: quantisation with one global scale for X + pair
    lift (blocks of 32 for a sparse weight, 16 for a dense one), then the
    block-scaled GEMM."""
    dense = _pattern(pattern).group == 0
    act = quant_lift_act_nvfp4(X, pattern, 16 if dense else 32, stream)
    M, N = X.shape[0], packed[0].shape[0]
    if dense:
        return dense_gemm_nvfp4(act, packed, M, N, out_dtype, stream)
    return sparse_gemm_nvfp4(packed, act, M, N, out_dtype, stream)
