#!/usr/bin/env python
"""Benchmark of the structured-sparse quantized matmul hot path on B200.

One step = one pass of the path over one batch of synthetic input already
resident in HBM:
  weight-sparse workloads:  ss_quant_lift_act (per-token quant + lift)
                            -> ss_sparse_gemm (sparse tensor cores + dequant)
  online-activation workload: ss_prune_act_2to4 -> ss_sparse_gemm (sparse X)
The dense comparator (ss_quant_lift_act dense -> ss_dense_gemm, same
construction) is timed in the same run on the same inputs.  For the bf16
tier (--qdtype bf16 or a *_bf16 workload) the step is the lift and the
kind::f16 sparse GEMM, and the dense FP8 path is timed as well: the pages'
"2x tier" compares 2:4 + 16-bit against dense 8-bit.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--m M]
    python bench.py --impl reference ...   # the CPU oracle, timed on the host

Metric: dense-equivalent TOPS = 2 M N K / step time (K the original,
unpadded reduction length), summed over ranks; also the speedup over the own
dense path and the GEMM's fraction of the sparse tensor-core peak.  L2 is
flushed (a 256 MiB read) before every timed step; the flush is outside the
timed events.  Multi-GPU runs are weak-scaled independent replicas (the path
has no exchange step): no collective touches the data path.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)

from structured_sparse_quantized_b200 import synth  # noqa: E402

METRIC = "dense-equiv TOPS & speedup vs own dense GEMM at prefill M; % sparse TC peak"
UNIT = "TOPS (dense-equivalent)"
# The default line: the largest single-GPU configuration, one Llama-3.1-8B
# gate/up projection (N = 14336, K = 4096) at M = 16384 tokens, 6:8 INT8.
DEFAULT_WORKLOAD = "llama_layer_gate_up"
# Side lines on the same run: 2:4 INT8 on the q_proj shape and the SlideSparse
# 6:8 FP8 headline shape (Qwen2.5-7B gate/up), both at M = 8192.
ALSO_WORKLOADS = (("llama_q_2of4_int8", 8192), ("qwen_gateup_6of8_fp8", 8192))
FLUSH_BYTES = 256 << 20
IDEAL = {"2:4": 2.0, "4:6": 1.5, "6:8": 4.0 / 3.0, "8:10": 1.25}

# DRAM bytes per launch of the dominant kernel (dram__bytes_read.sum +
# dram__bytes_write.sum of one sparse-GEMM launch) from one ncu capture.
# Keyed by (workload, M, pattern, qdtype) as run; each entry names the
# profile summary it comes from, the sources that make up that kernel (its
# device code and the host code that picks its shape) and their hash at
# capture time (csrc_hash).  A stored figure is reported only while those
# sources still hash the same; otherwise "traffic" is null.
GEMM_SOURCES = ("ss_api.cu", "ss_common.cuh", "ss_gemm.cuh", "ss_gemm_wide.cuh")
TRAFFIC = {
    ("llama_layer_gate_up", 16384, "6:8", "int8"): {
        "bytes": (290.75e6 + 430.85e6 + 290.91e6 + 427.64e6) / 2,
        "profile": "profiles/gemm_llama_gateup_6of8_int8_m16384.md",
        "sources": GEMM_SOURCES,
        "csrc_hash": "53a72fd05f31a017"},
}


def csrc_hash(files=None) -> str:
    """sha256 (first 16 hex digits) of the named CUDA sources (all of them
    when files is None)."""
    import hashlib
    d = os.path.join(HERE, "structured_sparse_quantized_b200", "csrc")
    names = sorted(files) if files else sorted(n for n in os.listdir(d)
                                               if n.endswith((".cu", ".cuh")))
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def load_peaks():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", 0) or 0),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------- distributed plumbing

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64,
                         device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock, max clock and throttle reasons through NVML while the
    timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
               "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None
        self.period = period_s
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": "no NVML samples"}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- the path

class Path:
    """Inputs, packed weights and outputs of one workload, resident on the device."""

    def __init__(self, name: str, M: int, device: torch.device):
        import structured_sparse_quantized_b200 as ss
        self.ss = ss
        w = dict(synth.WORKLOADS[name])
        self.name, self.w = name, w
        self.M, self.N, self.K = M, w["N"], w["K"]
        self.pat, self.q = w["pattern"], w["qdtype"]
        self.online = name.startswith("online")
        self.out_dtype = torch.float32 if w["out"] == "f32" else torch.bfloat16
        W = synth.make_weight(self.N, self.K, w["w_std"], w["in_dtype"]).to(device)
        self.X_host = synth.make_activation(M, self.K, w["x_kind"], w["in_dtype"])
        self.X = self.X_host.to(device)
        # offline: compress weights (sparse and the dense comparator's)
        self.fp4 = self.q == "nvfp4"
        if self.fp4:  # pairwise sparse NVFP4 against dense NVFP4 (patterns count pairs)
            if self.online:
                raise ValueError("the NVFP4 path is weight-sparse only")
            self.dense_w = ss.compress_weight_nvfp4(W, "dense")
            self.sparse_w = ss.compress_weight_nvfp4(W, self.pat)
            _, self.K_lp = ss.ss_fp4_shape(self.pat, self.K)
            _, self.K_p = ss.ss_fp4_shape("dense", self.K)
            self.act = ss.quant_lift_act_nvfp4(self.X, self.pat, 32)
            self.dense_act = ss.quant_lift_act_nvfp4(self.X, "dense", 16)
            # row blocks of the end-to-end run are separate calls, each with
            # its own tensor-wide global scale (16-byte aligned slots)
            self.g_blocks = torch.zeros(4 * ((M + 127) // 128), dtype=torch.float32,
                                        device=device)
            self.Y = torch.empty((M, self.N), dtype=self.out_dtype, device=device)
            del W
            torch.cuda.synchronize()
            if ss.ss_get_device_status() != ss.SS_OK:
                raise RuntimeError("device status not clean after set-up")
            return
        self.dense_w = ss.compress_weight(W, "dense", self.q)
        if self.online:
            self.K_lp = ss.ss_act_2to4_shape(self.K)
            self.act = ss.prune_act_2to4(self.X, self.q)
        else:
            self.sparse_w = ss.compress_weight(W, self.pat, self.q)
            _, _, self.K_lp = ss.ss_slide_shape(self.pat, self.K)
            self.act = ss.quant_lift_act(self.X, self.pat, self.q)
        self.dense_act = ss.quant_lift_act(self.X, "dense", self.q)
        self.Y = torch.empty((M, self.N), dtype=self.out_dtype, device=device)
        del W
        torch.cuda.synchronize()
        if ss.ss_get_device_status() != ss.SS_OK:
            raise RuntimeError("device status not clean after set-up")

    # one step of the sparse path; ev = (start, mid, end) events or None
    def sparse_step(self, ev=None, X=None):
        ss = self.ss
        X = self.X if X is None else X
        if ev:
            ev[0].record()
        if self.fp4:
            ss.quant_lift_act_nvfp4(X, self.pat, 32, out=self.act)
            if ev and ev[1] is not None:
                ev[1].record()
            ss.sparse_gemm_nvfp4(self.sparse_w, self.act, self.M, self.N, out=self.Y)
        elif self.online:
            ss.prune_act_2to4(X, self.q, out=self.act)
            if ev and ev[1] is not None:
                ev[1].record()
            Xv, Xm, s_x = self.act
            Wq, _, s_w = self.dense_w
            ss.sparse_gemm(1, Xv, Xm, s_x, Wq, s_w, self.M, self.N, self.q, out=self.Y)
        else:
            ss.quant_lift_act(X, self.pat, self.q, out=self.act)
            if ev and ev[1] is not None:
                ev[1].record()
            Wv, Wm, s_w = self.sparse_w
            Xq, s_x = self.act
            ss.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, self.M, self.N, self.q, out=self.Y)
        if ev:
            ev[2].record()

    def sparse_rows(self, X_rows, r0: int, r1: int):
        """The sparse path on token rows r0..r1 (a multiple of 128 apart) of
        this workload, on the current stream: X_rows in, Y rows r0..r1 out."""
        ss = self.ss
        m = r1 - r0
        rows = lambda t: None if t is None else t[r0:r1]  # bf16 tier: no scales
        if self.fp4:
            Xv, Xs, _ = self.act
            nblk = self.K_lp // 32  # tile-major scales: 128-row tiles are contiguous
            g = self.g_blocks[4 * (r0 // 128):4 * (r0 // 128) + 4]
            part = (Xv[r0:r1], Xs[r0 * nblk:r1 * nblk], g)
            ss.quant_lift_act_nvfp4(X_rows, self.pat, 32, out=part)
            ss.sparse_gemm_nvfp4(self.sparse_w, part, m, self.N, out=self.Y[r0:r1])
        elif self.online:
            Xv, Xm, s_x = self.act
            part = (Xv[r0:r1], Xm[r0 // 128:r1 // 128], rows(s_x))
            ss.prune_act_2to4(X_rows, self.q, out=part)
            Wq, _, s_w = self.dense_w
            ss.sparse_gemm(1, part[0], part[1], part[2], Wq, s_w, m, self.N, self.q,
                           out=self.Y[r0:r1])
        else:
            Xq, s_x = self.act
            part = (Xq[r0:r1], rows(s_x))
            ss.quant_lift_act(X_rows, self.pat, self.q, out=part)
            Wv, Wm, s_w = self.sparse_w
            ss.sparse_gemm(0, Wv, Wm, s_w, part[0], part[1], m, self.N, self.q,
                           out=self.Y[r0:r1])

    def dense_step(self, ev=None):
        ss = self.ss
        if ev:
            ev[0].record()
        if self.fp4:
            ss.quant_lift_act_nvfp4(self.X, "dense", 16, out=self.dense_act)
            if ev and ev[1] is not None:
                ev[1].record()
            ss.dense_gemm_nvfp4(self.dense_act, self.dense_w, self.M, self.N, out=self.Y)
            if ev:
                ev[2].record()
            return
        ss.quant_lift_act(self.X, "dense", self.q, out=self.dense_act)
        if ev and ev[1] is not None:
            ev[1].record()
        Xq, s_x = self.dense_act
        Wq, _, s_w = self.dense_w
        ss.dense_gemm(Xq, s_x, Wq, s_w, self.q, out=self.Y)
        if ev:
            ev[2].record()

    # algorithmic work
    def dense_equiv_ops(self):
        return 2.0 * self.M * self.N * self.K

    def sparse_gemm_ops(self):
        return 2.0 * self.M * self.N * self.K_lp      # lifted logical MACs x 2

    def dense_gemm_ops(self):
        if self.fp4:
            return 2.0 * self.M * self.N * self.K_p
        return 2.0 * self.M * self.N * self.dense_w[0].shape[1]

    def act_kernel_bytes(self):
        esz = self.X.element_size()
        if self.fp4:  # codes, one UE4M3 scale per 32, one global scale (X read once)
            return self.M * (esz * self.K + self.K_lp // 2 + self.K_lp // 32) + 4
        vb, sb = (2, 0) if self.q == "bf16" else (1, 4)   # value bytes, scale bytes
        if self.online:
            return self.M * (esz * self.K + vb * self.K_lp // 2 + self.K_lp // 8 + sb)
        return self.M * (esz * self.K + vb * self.K_lp + sb)

    def dense_act_bytes(self):
        if self.fp4:
            return self.M * (self.X.element_size() * self.K + self.K_p // 2 + self.K_p // 16) + 4
        vb, sb = (2, 0) if self.q == "bf16" else (1, 4)
        return self.M * (self.X.element_size() * self.K + vb * self.dense_act[0].shape[1] + sb)

    # peaks: dense bf16 measured; 8-bit dense = 2x, FP4 dense = 4x, 2:4 sparse
    # = 2x dense (NVIDIA's nominal ratios)
    def dense_peak(self, bf16_peak: float) -> float:
        return bf16_peak * {"bf16": 1.0, "nvfp4": 4.0}.get(self.q, 2.0)

    def sparse_peak(self, bf16_peak: float) -> float:
        return 2.0 * self.dense_peak(bf16_peak)


class DenseFp8:
    """Dense FP8 comparator of a bf16-tier workload (per-token quant + dense
    E4M3 GEMM, the like-for-like 8-bit path) on the same W and X."""

    def __init__(self, path: "Path"):
        ss = path.ss
        self.ss, self.path = ss, path
        W = synth.make_weight(path.N, path.K, path.w["w_std"], path.w["in_dtype"]).to(path.X.device)
        self.w = ss.compress_weight(W, "dense", "fp8")
        self.act = ss.quant_lift_act(path.X, "dense", "fp8")
        del W

    def step(self, ev=None):
        ss, p = self.ss, self.path
        if ev:
            ev[0].record()
        ss.quant_lift_act(p.X, "dense", "fp8", out=self.act)
        if ev and ev[1] is not None:
            ev[1].record()
        Xq, s_x = self.act
        Wq, _, s_w = self.w
        ss.dense_gemm(Xq, s_x, Wq, s_w, "fp8", out=p.Y)
        if ev:
            ev[2].record()


def flush_l2(buf):
    """Evict L2 by reading a buffer twice its size.  A read leaves only clean
    lines behind, so the next kernel does not pay for writing back dirty
    flush data; dirty lines of the previous step are written back here,
    outside the timed events."""
    return buf.sum(dtype=torch.int64)


def time_loop(fn, steps, warmup, flush, split=True):
    """Per-step CUDA-event times (ms) of fn(ev) with an L2 flush before each
    step, outside the events.  With split, an event between the activation
    kernel and the GEMM also times each part; without it the step has only
    its start and end events, so nothing on the stream separates the two
    kernels and the GEMM may start early (programmatic dependent launch)."""
    for _ in range(warmup):
        flush_l2(flush)
        fn(None)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    if not split:
        for e in evs:
            e[1] = None
    torch.cuda.synchronize()
    for i in range(steps):
        flush_l2(flush)
        fn(evs[i])
    torch.cuda.synchronize()
    total = [e[0].elapsed_time(e[2]) for e in evs]
    if not split:
        return total, None, None
    first = [e[0].elapsed_time(e[1]) for e in evs]
    second = [e[1].elapsed_time(e[2]) for e in evs]
    return total, first, second


def measure(path: Path, steps: int, warmup: int, dist: Dist, peaks: dict):
    ss = path.ss
    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
    dist.barrier()
    torch.cuda.synchronize()
    launches0 = ss.ss_kernel_launches()
    with ClockSampler(torch.cuda.current_device()) as clk:
        sp_total, _, _ = time_loop(path.sparse_step, steps, warmup, flush, split=False)
    # every step (warm-up or timed) launches the same kernels
    launches = (ss.ss_kernel_launches() - launches0) * steps // (steps + warmup)
    dn_total, _, _ = time_loop(path.dense_step, steps, warmup, flush, split=False)
    # the per-kernel split (an event between the two kernels) in separate runs
    _, sp_act, sp_gemm = time_loop(path.sparse_step, steps, warmup, flush)
    _, dn_act, dn_gemm = time_loop(path.dense_step, steps, warmup, flush)
    torch.cuda.synchronize()
    dist.barrier()
    status = ss.ss_get_device_status()
    if status != ss.SS_OK:
        raise RuntimeError(f"device status {ss.ss_status_string(status)} after timing")
    mean = statistics.fmean
    t_step = dist.max(mean(sp_total))
    t_dense = dist.max(mean(dn_total))
    r = {
        "t_step_ms": t_step, "t_dense_step_ms": t_dense,
        "t_act_ms": mean(sp_act), "t_gemm_ms": mean(sp_gemm),
        "t_dense_act_ms": mean(dn_act), "t_dense_gemm_ms": mean(dn_gemm),
        "launches": launches, "clocks": clk.summary(),
    }
    sparse_peak = path.sparse_peak(peaks["bf16_tflops"])
    dense_peak = path.dense_peak(peaks["bf16_tflops"])
    r["sparse_gemm_tflops"] = path.sparse_gemm_ops() / (r["t_gemm_ms"] * 1e-3) / 1e12
    r["dense_gemm_tflops"] = path.dense_gemm_ops() / (r["t_dense_gemm_ms"] * 1e-3) / 1e12
    r["sparse_peak"] = sparse_peak
    r["dense_peak"] = dense_peak
    r["act_gbs"] = path.act_kernel_bytes() / (r["t_act_ms"] * 1e-3) / 1e9
    r["dense_act_gbs"] = path.dense_act_bytes() / (r["t_dense_act_ms"] * 1e-3) / 1e9
    if path.q == "bf16":
        f8 = DenseFp8(path)
        f8_total, _, _ = time_loop(f8.step, steps, warmup, flush, split=False)
        _, _, f8_gemm = time_loop(f8.step, steps, warmup, flush)
        r["t_fp8_step_ms"] = dist.max(mean(f8_total))
        r["t_fp8_gemm_ms"] = mean(f8_gemm)
        del f8
    return r


def e2e(path: Path, steps: int, warmup: int, dist: Dist, chunks: int = 8):
    """Same metric through the public API with host buffers: pinned X copied
    in, path run, Y copied out, all inside the timed events.  The step's
    tokens go in `chunks` row blocks on three streams, so the copy of block
    c+1 in, the path on block c and the copy of block c-1 out overlap."""
    X_pin = path.X_host.pin_memory()
    Y_pin = torch.empty(path.Y.shape, dtype=path.Y.dtype).pin_memory()
    X_dev = torch.empty_like(path.X)
    M = path.M
    if M % (128 * chunks) != 0:
        chunks = 1
    mc = M // chunks
    streams = [torch.cuda.Stream() for _ in range(3)]  # copy in, compute, copy out
    e_in = [torch.cuda.Event() for _ in range(chunks)]
    e_done = [torch.cuda.Event() for _ in range(chunks)]

    def step(ev):
        cur = torch.cuda.current_stream()
        if ev:
            ev[0].record(cur)
        for st in streams:
            st.wait_stream(cur)
        for c in range(chunks):
            r0, r1 = c * mc, (c + 1) * mc
            with torch.cuda.stream(streams[0]):
                X_dev[r0:r1].copy_(X_pin[r0:r1], non_blocking=True)
                e_in[c].record()
            with torch.cuda.stream(streams[1]):
                streams[1].wait_event(e_in[c])
                path.sparse_rows(X_dev[r0:r1], r0, r1)
                e_done[c].record()
            with torch.cuda.stream(streams[2]):
                streams[2].wait_event(e_done[c])
                Y_pin[r0:r1].copy_(path.Y[r0:r1], non_blocking=True)
        for st in streams:
            cur.wait_stream(st)
        if ev:
            ev[1].record(cur)
            ev[2].record(cur)

    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")
    total, _, _ = time_loop(step, steps, warmup, flush)
    t = dist.max(statistics.fmean(total))
    h2d = X_pin.numel() * X_pin.element_size()
    d2h = Y_pin.numel() * Y_pin.element_size()
    return t, h2d, d2h


# ---------------------------------------------------------------- CPU oracle (baseline arm)

def oracle_sample(name: str, M: int, budget_s: float):
    """Time the CPU oracle on a bounded row sample of the workload: the
    per-token quantisation (+ lift / online prune) of the sampled rows and
    their sparse GEMM rows.  The weight compression is offline on both arms
    and is not timed.  Returns (TOPS dense-equivalent, rows, seconds, cores)."""
    import oracle
    w = synth.WORKLOADS[name]
    N, K = w["N"], w["K"]
    bf16 = w["qdtype"] == "bf16"
    fp4 = w["qdtype"] == "nvfp4"
    q = {"int8": oracle.INT8, "fp8": oracle.FP8_E4M3, "bf16": oracle.BF16,
         "nvfp4": oracle.NVFP4}[w["qdtype"]]
    out = oracle.OUT_F32 if w["out"] == "f32" else oracle.OUT_BF16
    W = synth.make_weight(N, K, w["w_std"], w["in_dtype"])
    online = name.startswith("online")
    pat = "dense" if online else w["pattern"]
    if fp4:
        packed = oracle.compress_weight_nvfp4(W, pat)
    elif bf16:
        packed = oracle.compress_weight_bf16(W, pat)
    else:
        packed = oracle.compress_weight(W, pat, q)
    X = synth.make_activation(M, K, w["x_kind"], w["in_dtype"])

    def run(rows):
        Xs = X[rows]
        t0 = time.perf_counter()
        if fp4:
            Wv, Wm, Ws, g_w = packed
            Xv, Xsc, g_x = oracle.quant_nvfp4(Xs, pat, 32)
            oracle.sparse_gemm_nvfp4(Wv, Wm, Ws, g_w, Xv, Xsc, g_x, len(rows), N,
                                     Xv.shape[1] * 2, out)
        elif bf16 and online:
            Xv, Xm = oracle.prune_act_2to4_bf16(Xs)
            Wb, _ = packed
            oracle.sparse_gemm_bf16(1, Xv, Xm, Wb, len(rows), N, Wb.shape[1], out)
        elif bf16:
            Wv, Wm = packed
            Xl = oracle.lift_act_bf16(Xs, pat)
            oracle.sparse_gemm_bf16(0, Wv, Wm, Xl, len(rows), N, Xl.shape[1], out)
        elif online:
            Xv, Xm, s_x = oracle.prune_act_2to4(Xs, q)
            Wq, _, s_w = packed
            oracle.sparse_gemm(1, Xv, Xm, s_x, Wq, s_w, len(rows), N, Wq.shape[1], q, out)
        else:
            Wv, Wm, s_w = packed
            Xq, s_x = oracle.quant_lift_act(Xs, w["pattern"], q)
            oracle.sparse_gemm(0, Wv, Wm, s_w, Xq, s_x, len(rows), N, Xq.shape[1], q, out)
        return time.perf_counter() - t0

    n = min(M, 8)
    t = run(np.arange(n))
    while t < budget_s / 4 and n < M:
        n = min(M, max(n * 2, int(n * budget_s / max(t, 1e-3) / 2)))
        t = run(np.arange(n))
    tops = 2.0 * n * N * K / t / 1e12
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return tops, n, t, cores


# ---------------------------------------------------------------- main

def base_line(args, workload, M, n_gpus):
    return {"metric": METRIC, "unit": UNIT, "n_gpus": n_gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "data": "synthetic",
            "config": {"workload": workload, "M": M, "N": synth.WORKLOADS[workload]["N"],
                       "K": synth.WORKLOADS[workload]["K"],
                       "pattern": synth.WORKLOADS[workload]["pattern"],
                       "qdtype": synth.WORKLOADS[workload]["qdtype"],
                       "parallelism": f"replicas x{n_gpus}", "l2": "flushed (256 MiB read) "
                       "before every timed step"}}


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    import oracle  # noqa: F401  (test infrastructure; the reference arm only)
    M = args.m
    vals, rows, secs = [], 0, 0.0
    cores = 1
    for _ in range(args.warmup):
        oracle_sample(args.workload, M, budget_s=1.0)
    for _ in range(args.steps):
        tops, rows, secs, cores = oracle_sample(args.workload, M, budget_s=args.ref_budget)
        vals.append(tops)
    v = statistics.fmean(vals)
    line = base_line(args, args.workload, M, 1)
    line.update({"impl": "reference", "value": v, "ms_per_step": secs * 1e3,
                 "dtype": synth.WORKLOADS[args.workload]["qdtype"],
                 "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                  "cpu_model": cpu_model(),
                                  "sample": f"{rows} of {M} token rows per step (quant/lift or "
                                            f"online prune + sparse GEMM rows); weight "
                                            f"compression offline, untimed"},
                 "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0,
                         "d2h_bytes_per_step": 0}})
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ss", choices=["ss", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--m", type=int, default=None)
    ap.add_argument("--no-also", action="store_true", help="skip the side measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--ref-budget", type=float, default=6.0)
    ap.add_argument("--pattern", default=None, choices=["2:4", "4:6", "6:8", "8:10"],
                    help="override the workload's pattern (the Llama-layer sweep)")
    ap.add_argument("--qdtype", default=None, choices=["int8", "fp8", "bf16", "nvfp4"],
                    help="override the workload's quantised type")
    args = ap.parse_args()
    if args.pattern or args.qdtype:
        w = dict(synth.WORKLOADS[args.workload])
        w["pattern"] = args.pattern or w["pattern"]
        w["qdtype"] = args.qdtype or w["qdtype"]
        synth.WORKLOADS[args.workload] = w
    if args.m is None:
        args.m = synth.WORKLOADS[args.workload]["M"]
    args.warmup = max(args.warmup, 3)
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    peaks = load_peaks()
    path = Path(args.workload, args.m, torch.device("cuda", dist.local))
    r = measure(path, args.steps, args.warmup, dist, peaks)
    t_e2e, h2d, d2h = e2e(path, max(3, args.steps // 3), args.warmup, dist)
    n = dist.world
    value = n * path.dense_equiv_ops() / (r["t_step_ms"] * 1e-3) / 1e12
    line = base_line(args, args.workload, args.m, n)
    wl = synth.WORKLOADS[args.workload]
    tr = TRAFFIC.get((args.workload, args.m, wl["pattern"], wl["qdtype"]))
    traffic = tr["bytes"] if tr and tr["csrc_hash"] == csrc_hash(tr["sources"]) else None
    line.update({
        "value": value, "ms_per_step": r["t_step_ms"],
        "dtype": path.q,
        "speedup_vs_own_dense": r["t_dense_step_ms"] / r["t_step_ms"],
        "gemm_speedup_vs_own_dense": r["t_dense_gemm_ms"] / r["t_gemm_ms"],
        "ideal_speedup": IDEAL[path.pat],
        "pct_sparse_tc_peak": 100.0 * r["sparse_gemm_tflops"] / r["sparse_peak"],
        "kernels": {
            "act": {"name": "prune_act_2to4" if path.online else "quant_lift_act",
                    "us": r["t_act_ms"] * 1e3, "gbs": r["act_gbs"],
                    "frac_hbm": r["act_gbs"] / peaks["hbm_gbs"]},
            "sparse_gemm": {"us": r["t_gemm_ms"] * 1e3, "tflops": r["sparse_gemm_tflops"]},
            "dense_act": {"us": r["t_dense_act_ms"] * 1e3, "gbs": r["dense_act_gbs"]},
            "dense_gemm": {"us": r["t_dense_gemm_ms"] * 1e3, "tflops": r["dense_gemm_tflops"],
                           "frac_dense_peak": r["dense_gemm_tflops"] / r["dense_peak"]},
        },
        "roofline": {"bound": "tensor", "kernel": "sparse_gemm",
                     "achieved": r["sparse_gemm_tflops"], "peak": r["sparse_peak"],
                     "unit": "TFLOP/s", "frac": r["sparse_gemm_tflops"] / r["sparse_peak"],
                     "peak_source": f"{peaks['source']} bf16 burst x"
                                    f"{r['sparse_peak'] / peaks['bf16_tflops']:.0f}"
                                    + {"bf16": " (2:4 x2)", "nvfp4": " (FP4 x4, 2:4 x2)"}.get(
                                        path.q, " (8-bit x2, 2:4 x2)"),
                     "traffic": traffic,
                     "traffic_source": ({"profile": tr["profile"], "csrc_hash": tr["csrc_hash"]}
                                        if traffic is not None else None)},
        "e2e": {"value": n * path.dense_equiv_ops() / (t_e2e * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    })
    if path.q == "bf16":  # the 2x tier: 2:4 + bf16 against dense FP8
        line["vs_dense_fp8"] = {"speedup": r["t_fp8_step_ms"] / r["t_step_ms"],
                                "gemm_speedup": r["t_fp8_gemm_ms"] / r["t_gemm_ms"],
                                "fp8_step_us": r["t_fp8_step_ms"] * 1e3,
                                "fp8_gemm_us": r["t_fp8_gemm_ms"] * 1e3}
    if not args.no_also and dist.world == 1:
        del path
        torch.cuda.empty_cache()
        line["also"] = []
        for name, m in ALSO_WORKLOADS:
            if name == args.workload:
                continue
            p2 = Path(name, m, torch.device("cuda", dist.local))
            r2 = measure(p2, max(5, args.steps // 2), args.warmup, dist, peaks)
            line["also"].append({
                "workload": name, "M": m, "pattern": p2.pat, "qdtype": p2.q,
                "value": p2.dense_equiv_ops() / (r2["t_step_ms"] * 1e-3) / 1e12,
                "speedup_vs_own_dense": r2["t_dense_step_ms"] / r2["t_step_ms"],
                "gemm_speedup_vs_own_dense": r2["t_dense_gemm_ms"] / r2["t_gemm_ms"],
                "ideal_speedup": IDEAL[p2.pat],
                "pct_sparse_tc_peak": 100.0 * r2["sparse_gemm_tflops"] / r2["sparse_peak"],
                "act_gbs": r2["act_gbs"], "act_frac_hbm": r2["act_gbs"] / peaks["hbm_gbs"],
                "sparse_gemm_us": r2["t_gemm_ms"] * 1e3,
                "dense_gemm_us": r2["t_dense_gemm_ms"] * 1e3,
            })
            del p2
            torch.cuda.empty_cache()
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
        tops, rows, secs, cores = oracle_sample(args.workload, args.m, budget_s=10.0)
        line["cpu_baseline"] = {"value": tops, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "cpu_model": cpu_model(),
                                "sample": f"{rows} of {args.m} token rows of the same workload "
                                          f"({secs:.1f} s; weight compression offline, "
                                          f"untimed)"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
