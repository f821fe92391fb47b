"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module only draws random numbers in the shapes and value distributions
of the workloads; it holds none of the method's arithmetic (no pruning,
quantisation, lifting or packing), so the CUDA path and the CPU oracle can
both take their inputs from it without sharing any computation.

The workloads stand in for the Llama-3.1-8B and Qwen2.5-7B projection layers
that the SlideSparse pages and the "add 2:4 or drop a precision tier" study
measure on real activations; no weights or datasets are used.
"""
from __future__ import annotations

import numpy as np
import torch


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def gaussian(shape, std: float = 1.0, seed: int = 0, dtype=torch.float32) -> torch.Tensor:
    """i.i.d. N(0, std^2), drawn in fp32 and rounded to `dtype` (RNE for bf16)."""
    a = _rng(seed).standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    return torch.from_numpy(a).to(dtype)


def outlier_channels(K: int, frac: float, seed: int) -> np.ndarray:
    """Indices of round(frac*K) channels (at least one), chosen by seed."""
    n = max(1, int(round(frac * K)))
    return np.sort(_rng(seed + 1000).choice(K, size=n, replace=False))


def gaussian_with_outliers(M: int, K: int, scale: float = 20.0, frac: float = 0.01,
                           seed: int = 1, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0,1) activations with `frac` of the K channels multiplied by `scale`."""
    a = _rng(seed).standard_normal(size=(M, K), dtype=np.float32)
    a[:, outlier_channels(K, frac, seed)] *= np.float32(scale)
    return torch.from_numpy(a).to(dtype)


def gaussian_with_heavy_tails(M: int, K: int, nu: float = 3.0, frac: float = 0.01,
                              seed: int = 1, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0,1) activations whose `frac` of channels are Student-t(nu) instead."""
    g = _rng(seed)
    a = g.standard_normal(size=(M, K), dtype=np.float32)
    ch = outlier_channels(K, frac, seed)
    a[:, ch] = g.standard_t(nu, size=(M, len(ch))).astype(np.float32)
    return torch.from_numpy(a).to(dtype)


def sample_rows(M: int, seed: int = 7, edge: int = 128, middle: int = 256) -> np.ndarray:
    """Deterministic output-row sample for full-size parity: the first and
    last `edge` rows plus `middle` seeded rows (all rows when M is small)."""
    if M <= 2 * edge + middle:
        return np.arange(M, dtype=np.int64)
    mid = _rng(seed).choice(np.arange(edge, M - edge), size=middle, replace=False)
    rows = np.concatenate([np.arange(edge), np.sort(mid), np.arange(M - edge, M)])
    return rows.astype(np.int64)


# Workloads: weight W[N, K] and activation X[M, K].  W ~ N(0, 0.02) (fp32
# N(0, 1) for the single-linear case), X ~ N(0, 1); seed 0 for W, 1 for X.
WORKLOADS = {
    "linear_6of8_int8_m16": dict(M=16, K=64, N=64, pattern="6:8", qdtype="int8",
                                 in_dtype="f32", w_std=1.0, out="f32", x_kind="gauss"),
    "llama_q_2of4_int8": dict(M=8192, K=4096, N=4096, pattern="2:4", qdtype="int8",
                              in_dtype="bf16", w_std=0.02, out="bf16", x_kind="outlier"),
    "qwen_gateup_6of8_fp8": dict(M=8192, K=3584, N=18944, pattern="6:8", qdtype="fp8",
                                 in_dtype="bf16", w_std=0.02, out="bf16", x_kind="gauss"),
    "online_x_2of4_fp8": dict(M=8192, K=4096, N=14336, pattern="2:4", qdtype="fp8",
                              in_dtype="bf16", w_std=0.02, out="bf16", x_kind="heavy"),
    # the 16-bit tier of the precision-tier study: 2:4 + bf16 on the
    # Llama-3.1-8B q_proj shape (compared with dense bf16 and dense FP8)
    "llama_q_2of4_bf16": dict(M=8192, K=4096, N=4096, pattern="2:4", qdtype="bf16",
                              in_dtype="bf16", w_std=0.02, out="bf16", x_kind="outlier"),
    # Blackwell's sparse FP4: pairwise 4:8 (pattern 2:4 counted in pairs) in
    # NVFP4 on the Llama-3.1-8B gate/up shape, against dense NVFP4
    "llama_gateup_4of8_nvfp4": dict(M=8192, K=4096, N=14336, pattern="2:4", qdtype="nvfp4",
                                    in_dtype="bf16", w_std=0.02, out="bf16", x_kind="gauss"),
}

# Llama-3.1-8B layer projections (N, K) for the pattern sweep.
LLAMA_LAYER = {"q_o": (4096, 4096), "k_v": (1024, 4096), "gate_up": (14336, 4096),
               "down": (4096, 14336)}

# The sweep's workloads (one per projection; pattern and qdtype are varied on
# the bench command line): Gaussian W std 0.02, Gaussian X, bf16 out.
for _proj, (_n, _k) in LLAMA_LAYER.items():
    WORKLOADS[f"llama_layer_{_proj}"] = dict(M=16384, K=_k, N=_n, pattern="6:8", qdtype="int8",
                                            in_dtype="bf16", w_std=0.02, out="bf16",
                                            x_kind="gauss")


def make_weight(N: int, K: int, std: float, in_dtype: str, seed: int = 0) -> torch.Tensor:
    return gaussian((N, K), std=std, seed=seed,
                    dtype=torch.float32 if in_dtype == "f32" else torch.bfloat16)


def make_activation(M: int, K: int, kind: str, in_dtype: str, seed: int = 1) -> torch.Tensor:
    dt = torch.float32 if in_dtype == "f32" else torch.bfloat16
    if kind == "outlier":
        return gaussian_with_outliers(M, K, seed=seed, dtype=dt)
    if kind == "heavy":
        return gaussian_with_heavy_tails(M, K, seed=seed, dtype=dt)
    return gaussian((M, K), std=1.0, seed=seed, dtype=dt)
