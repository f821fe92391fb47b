"""Shared helpers for the GPU parity tests (host side only)."""
import numpy as np
import torch

import oracle

Q = {"int8": oracle.INT8, "fp8": oracle.FP8_E4M3, "bf16": oracle.BF16}
FP8_TOL = 1e-2
# bf16 tier: exact products, fp32 accumulation in the tensor core's order
# against the oracle's double sum rounded once.  Reordering the sum of K
# products changes it by at most about K * 2^-24 * sum|x w| (2^-10 of the
# largest |y| at K = 16384 for Gaussian data), and bf16 output can then move
# by one unit in the last place (2^-8 relative): 1e-2 covers both.
BF16_TOL = 1e-2


def dev(a) -> torch.Tensor:
    """numpy / CPU tensor -> contiguous CUDA tensor (uint8 stays uint8)."""
    if isinstance(a, np.ndarray):
        a = torch.from_numpy(np.ascontiguousarray(a))
    return a.contiguous().cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.uint16).numpy()
    return t.numpy()


def y_to_float(y: np.ndarray, out_bf16: bool) -> np.ndarray:
    return oracle.bf16_bits_to_float(y) if out_bf16 else y.astype(np.float32)


def fp8_rel_error(y: np.ndarray, r: np.ndarray) -> float:
    """max_i |y_i - r_i| / max(|r_i|, 1e-2 * max_j |r_j|): relative error with
    a floor so that entries near zero do not make it undefined."""
    y = y.astype(np.float64)
    r = r.astype(np.float64)
    floor = 1e-2 * max(np.abs(r).max(), 1e-30)
    return float((np.abs(y - r) / np.maximum(np.abs(r), floor)).max())


def assert_y_matches(y_gpu: np.ndarray, y_ref: np.ndarray, q: str, out_bf16: bool):
    if q == "int8":
        np.testing.assert_array_equal(y_gpu, y_ref)   # bit-exact
    else:
        tol = BF16_TOL if q == "bf16" else FP8_TOL
        err = fp8_rel_error(y_to_float(y_gpu, out_bf16), y_to_float(y_ref, out_bf16))
        assert err <= tol, f"{q} relative error {err:.3e} > {tol}"
