"""Benchmark: one step of the NVFP4 linear with RHT (8192x14336x4096) on B200.

A step is the whole hot path for that workload, in the library's kernels:
  amax(RHT(A)) -> NVFP4 1x16 quantize of RHT(A)          (bsq_quant_nvfp4)
  amax(RHT(W)) -> NVFP4 16x16 quantize of RHT(W)         (bsq_quant_nvfp4)
  C = A W^T, tcgen05 block-scaled GEMM, bf16 output       (bsq_gemm_blockscaled)
value = 2*M*N*K / step time (TFLOP/s, whole job over all ranks).  Inputs (A
and W in bf16, 176 MiB) are larger than L2, so no flush is needed.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With N > 1 it runs under torchrun, one independent replica per GPU (weak
scaling, no collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, N, K = 8192, 14336, 4096
RHT_SEED = 2
METRIC = "NVFP4 GEMM TFLOPS (% of 9 PF FP4); quantize GB/s (% of HBM peak), 1×B200"
WORKLOAD = "nvfp4_linear_rht: A 8192x4096 N(0,1) w/ 0.5% channels x100, W 14336x4096 N(0,0.02), 16x16 RHT seed 2"
NOMINAL_FP4_OVER_BF16 = 4.0   # 9 PF / 2.25 PF dense (B200 table on the pages)
NOMINAL_FP8_OVER_BF16 = 2.0   # 4.5 PF / 2.25 PF
FALLBACK_HBM, FALLBACK_BF16 = 6650.0, 1590.0


def ncu_traffic(profile, sources):
    """DRAM bytes per launch recorded from an ncu capture in profiles/, or None
    when the kernel's sources changed since the capture (the summary records
    the sha256 of the sources it was taken with)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    t = re.search(r"^traffic_bytes_per_launch:\s*(\d+)", text, re.M)
    h = re.search(r"^source_sha256[^:]*:\s*([0-9a-f]{64})", text, re.M)
    if not t or not h:
        return None
    d = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, src), "rb") as f:
            d.update(f.read())
    return int(t.group(1)) if d.hexdigest() == h.group(1) else None


def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks (every rank calls it, same order)."""
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_step: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank runs one full step (weak scaling),
    timed by the slowest rank."""
    return world * flops_per_step / (ms_per_step * 1e-3) / 1e12


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM, FALLBACK_BF16, "fallback"


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every ~2 ms."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

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
            time.sleep(0.002)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------- oracle
def cpu_oracle_step(rows_a=1024, rows_w=2048, threads=1):
    """The oracle on a bounded sample of the workload: the first rows_a rows of
    A and rows_w rows of W quantized (amax + RHT + NVFP4), then their GEMM in
    binary64.  threads == 1: the serial C oracle throughout (its scalar
    binary64 GEMM loop); threads > 1: the oracle's row bands on that many
    threads and its BLAS binary64 GEMM.  Returns (seconds, flops of the
    sample)."""
    import numpy as np
    from fp8_math_b200 import workloads as W
    from oracle import oracle as ora
    A, Wt, seed = W.nvfp4_linear_rht(M=rows_a, N=rows_w, K=K)
    mask = ora.rht_sign_mask(seed)
    xa, xw = W.bf16_bits(A), W.bf16_bits(Wt)
    t0 = time.perf_counter()
    qa = ora.quant_nvfp4(xa, rht_mask=mask, threads=threads)
    qw = ora.quant_nvfp4(xw, block_2d=True, rht_mask=mask, threads=threads)
    da, dw = ora.dequant(0, *qa, threads=threads), ora.dequant(0, *qw, threads=threads)
    if threads > 1:
        ora.gemm_f64_blas(da, dw)
    else:
        ora.gemm_f64(da, dw)
    dt = time.perf_counter() - t0
    del np
    return dt, 2.0 * rows_a * rows_w * K


def cpu_baseline_line():
    """The oracle timed twice on the host: single-threaded on a 1024x2048
    slice, and on every core this process may use on the whole of A and 4096
    rows of W."""
    from oracle import oracle as ora
    ora.build()
    cores = ora.ncores()
    dt1, fl1 = cpu_oracle_step(1024, 2048, threads=1)
    dtn, fln = cpu_oracle_step(M, 4096, threads=cores)
    return {"value": fln / dtn / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"amax+RHT+NVFP4 quantize of all {M} rows of A and the first 4096 rows of W (K={K}), then "
                      f"their {M}x4096x{K} binary64 GEMM; the oracle's row bands on {cores} threads and its BLAS "
                      "GEMM",
            "seconds": dtn,
            "single_core": {"value": fl1 / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1, "seconds": dt1,
                            "sample": "the first 1024 rows of A and 2048 rows of W, then their 1024x2048x4096 "
                                      "binary64 GEMM; the serial C oracle (scalar GEMM loop)"}}


def reference_arm(args, rank):
    if rank != 0:
        return
    sys.path.insert(0, ROOT)
    from oracle import oracle as ora
    ora.build()
    cores = ora.ncores()
    rows_a, rows_w = 1024, 1024
    for _ in range(args.warmup):
        cpu_oracle_step(rows_a=rows_a, rows_w=rows_w, threads=cores)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, fl = cpu_oracle_step(rows_a=rows_a, rows_w=rows_w, threads=cores)
        times.append(dt)
        flops = fl
    tot = sum(times)
    value = flops * args.steps / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: amax+RHT+NVFP4 quantize of {rows_a} rows of A and {rows_w} rows of W "
                                   f"(K=4096), then their {rows_a}x{rows_w}x4096 binary64 GEMM; the oracle's row "
                                   f"bands on {cores} threads and its BLAS GEMM"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- per-row measurements
def measure_rows(hbm, fp4_peak, fp8_peak, reps=10, only=None):
    """Times every step of the hot path on its own workload at full size.
    Each call runs on a cold L2: before it, L2 is flushed by writing a 256 MiB
    buffer and then reading another one (L2 is write-back, so after the write
    alone up to 126 MB of dirty lines would be written back inside the timed
    call; the read replaces them by clean lines).  The CUDA event clock here
    ticks in steps of about 2 us, too coarse for one short call, so a row's
    time is a difference of two event-timed batches on the stream: `reps`
    times (flush, call) minus `reps` times (flush), divided by `reps`, each
    batch the median of three.  Returns a list of dicts; a row that fails
    records its error instead of stopping the bench."""
    import torch

    from fp8_math_b200 import api, bsq
    from fp8_math_b200 import workloads as W

    dev = torch.device("cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def batch(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            flush.zero_()
            flush_r.sum()
            if fn is not None:
                fn()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) * 1e3

    def timed(fn):
        for _ in range(3):
            fn()
        with_fn, without = [], []
        for _ in range(3):
            with_fn.append(batch(fn, reps))
            without.append(batch(None, reps))
        if bsq.bsq_check() != bsq.BSQ_OK:
            raise RuntimeError("device error")
        return max(statistics.median(with_fn) - statistics.median(without), 0.0) / reps

    rows = []

    def wants(*names):
        """Whether any of these rows is selected (inputs are built only then)."""
        return only is None or any(only in n for n in names)

    def looped(fn, n=50):
        # n back-to-back calls between one event pair, no flush: the time per
        # call of a loop, host launch overhead included when it is the bound
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) * 1e3 / n

    def row(name, workload, fn, nbytes=None, flops=None, peak_kind=None, loop=False):
        if only and only not in name:
            return
        try:
            us = looped(fn) if loop else timed(fn)
            r = {"row": name, "workload": workload, "us": round(us, 2)}
            if flops is not None:
                peak = fp4_peak if peak_kind == "fp4" else fp8_peak
                tf = flops / (us * 1e-6) / 1e12
                r.update({"value": round(tf, 1), "unit": "TFLOP/s",
                          "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak,
                                       "frac": round(tf / peak, 3)}})
            else:
                gbs = nbytes / (us * 1e-6) / 1e9
                r.update({"value": round(gbs, 1), "unit": "GB/s",
                          "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                                       "frac": round(gbs / hbm, 3), "bytes": int(nbytes)}})
            rows.append(r)
        except Exception as e:  # noqa: BLE001 -- recorded, not fatal
            rows.append({"row": name, "workload": workload, "error": str(e)[:200]})

    if wants("a1 amax (RHT)", "a2+a5 NVFP4 1x16 quantize (amax + RHT fused)", "a3+a5 NVFP4 16x16 quantize (amax + RHT fused)", "a5 RHT standalone (bf16 -> bf16)", "a8 NVFP4 GEMM bf16",
             "f3 NVFP4 1x16 quantize SR (amax + RHT fused, next row)"):
        # -- NVFP4 linear with RHT, A 8192x4096, W 14336x4096 (the timed step's calls, one at a time)
        A_h, W_h, seed = W.nvfp4_linear_rht()
        mask = bsq.bsq_rht_sign_mask(seed)
        A, Wd = A_h.to(dev), W_h.to(dev)
        M2, K2 = A.shape
        N2 = Wd.shape[0]
        am = torch.empty(1, device=dev)
        row("a1 amax (RHT)", "A 8192x4096 bf16", lambda: bsq.bsq_amax(A, M2, K2, K2, 1, mask, None, am),
            nbytes=M2 * K2 * 2)
        qa = api.quant_nvfp4(A, rht_mask=mask)
        row("a2+a5 NVFP4 1x16 quantize (amax + RHT fused)", "A 8192x4096",
            lambda: api.quant_nvfp4(A, rht_mask=mask, out=qa), nbytes=M2 * K2 * (2 + 2 + 0.5 + 1 / 16))
        qw = api.quant_nvfp4(Wd, block_2d=True, rht_mask=mask)
        row("a3+a5 NVFP4 16x16 quantize (amax + RHT fused)", "W 14336x4096",
            lambda: api.quant_nvfp4(Wd, block_2d=True, rht_mask=mask, out=qw), nbytes=N2 * K2 * (2 + 2 + 0.5 + 1 / 16))
        qsr = api.quant_nvfp4_sr(A, rht_mask=mask, seed=2)
        row("f3 NVFP4 1x16 quantize SR (amax + RHT fused, next row)", "A 8192x4096",
            lambda: api.quant_nvfp4_sr(A, rht_mask=mask, seed=2, out=qsr), nbytes=M2 * K2 * (2 + 2 + 0.5 + 1 / 16))
        del qsr
        y = torch.empty_like(A)
        row("a5 RHT standalone (bf16 -> bf16)", "A 8192x4096", lambda: api.rht(A, mask, out=y), nbytes=M2 * K2 * 4)
        C2 = torch.empty(M2, N2, dtype=torch.bfloat16, device=dev)
        row("a8 NVFP4 GEMM bf16", "8192x14336x4096",
            lambda: api.gemm(0, qa[0], qa[1], qw[0], qw[1], M2, N2, K2, gsA=qa[2], gsB=qw[2], out=C2),
            flops=2 * M2 * N2 * K2, peak_kind="fp4")
        del y, C2
    if wants("a2+a3+a8 small linear step (latency)", "a2+a3+a8 small linear step as one CUDA graph (latency)"):
        # -- the small NVFP4 linear, A 128x256, W 256x256 (latency)
        As, Ws = W.nvfp4_linear_small()
        As, Ws = As.to(dev), Ws.to(dev)
        qas, qws = api.quant_nvfp4(As), api.quant_nvfp4(Ws, block_2d=True)
        Cs = torch.empty(128, 256, dtype=torch.float32, device=dev)

        def small_step():
            api.quant_nvfp4(As, out=qas)
            api.quant_nvfp4(Ws, block_2d=True, out=qws)
            api.gemm(0, qas[0], qas[1], qws[0], qws[1], 128, 256, 256, gsA=qas[2], gsB=qws[2], out=Cs)
        row("a2+a3+a8 small linear step (latency)", "A 128x256, W 256x256, fp32 out", small_step,
            nbytes=(128 + 256) * 256 * 2)
        if wants("a2+a3+a8 small linear step as one CUDA graph (latency)"):
            # the same five launches captured once and replayed as one graph
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                small_step()
            stream.wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                small_step()
            row("a2+a3+a8 small linear step as one CUDA graph (latency)", "A 128x256, W 256x256, fp32 out",
                graph.replay, nbytes=(128 + 256) * 256 * 2)
            # in a loop the host's launch work sets the pace of the eager calls
            row("a2+a3+a8 small linear step as one CUDA graph (latency), 50 in a loop",
                "A 128x256, W 256x256, fp32 out; per step", graph.replay, nbytes=(128 + 256) * 256 * 2, loop=True)
            row("a2+a3+a8 small linear step (latency), 50 eager calls in a loop", "A 128x256, W 256x256, fp32 out; per step",
                small_step, nbytes=(128 + 256) * 256 * 2, loop=True)
            del graph
    if wants("a6 MXFP8 row quantize RNE", "a6 MXFP8 row quantize SR (Philox)", "a7 requant-transpose SR",
             "f3 MXFP4 quantize RNE (next row)", "f3 MXFP4 quantize SR (next row)"):
        # -- MXFP8 4096x4096 Student-t: RNE and SR, requant-transpose
        X1 = W.mxfp8_requant().to(dev)
        M1, K1 = X1.shape
        q1 = api.quant_mxfp8(X1)
        row("a6 MXFP8 row quantize RNE", "X 4096x4096", lambda: api.quant_mxfp8(X1, out=q1),
            nbytes=M1 * K1 * (2 + 1 + 1 / 32))
        q1s = api.quant_mxfp8(X1, sr=True, seed=1)
        row("a6 MXFP8 row quantize SR (Philox)", "X 4096x4096", lambda: api.quant_mxfp8(X1, sr=True, seed=1, out=q1s),
            nbytes=M1 * K1 * (2 + 1 + 1 / 32))
        qt = api.requant_transpose(q1s[0], q1s[1], sr=True, seed=1)
        row("a7 requant-transpose SR", "4096x4096 MXFP8 -> column-wise",
            lambda: api.requant_transpose(q1s[0], q1s[1], sr=True, seed=1, out=qt), nbytes=2 * M1 * K1 * (1 + 1 / 32))
        q4 = api.quant_mxfp4(X1)
        row("f3 MXFP4 quantize RNE (next row)", "X 4096x4096", lambda: api.quant_mxfp4(X1, out=q4),
            nbytes=M1 * K1 * (2 + 0.5 + 1 / 32))
        row("f3 MXFP4 quantize SR (next row)", "X 4096x4096", lambda: api.quant_mxfp4(X1, sr=True, seed=1, out=q4),
            nbytes=M1 * K1 * (2 + 0.5 + 1 / 32))
        del X1, q1, q1s, qt, q4
    if wants("a6 MXFP8 row quantize SR", "a6 MXFP8 column quantize SR", "a8 MXFP8 GEMM dgrad (bf16 out)", "a8 MXFP8 GEMM wgrad (fp32 out)", "a8 NVFP4 rollout GEMM (swap-AB, HBM-bound)",
             "f2 MXFP8 row + column SR in one pass (next row)", "f2 NVFP4 -> MXFP8 column-wise requantize SR (next row)"):
        # -- MXFP8 backward (dY 8192x14336, W 14336x4096, X 8192x4096) + NVFP4 rollout
        dY, W4, X4, A_roll = W.mxfp8_backward()
        dY, W4, X4 = dY.to(dev), W4.to(dev), X4.to(dev)
        M4, N4 = dY.shape
        K4 = W4.shape[1]
        qdr = api.quant_mxfp8(dY, sr=True, seed=4, stream_id=0)
        row("a6 MXFP8 row quantize SR", "dY 8192x14336", lambda: api.quant_mxfp8(dY, sr=True, seed=4, out=qdr),
            nbytes=M4 * N4 * (2 + 1 + 1 / 32))
        qdc = api.quant_mxfp8(dY, colwise=True, sr=True, seed=4, stream_id=1)
        row("a6 MXFP8 column quantize SR", "dY 8192x14336 -> [14336, 8192]",
            lambda: api.quant_mxfp8(dY, colwise=True, sr=True, seed=4, stream_id=1, out=qdc),
            nbytes=M4 * N4 * (2 + 1 + 1 / 32))
        qrc = api.quant_mxfp8_rowcol(dY, sr=True, seed=4, stream_id_row=0, stream_id_col=1)
        row("f2 MXFP8 row + column SR in one pass (next row)", "dY 8192x14336 -> [8192, 14336] and [14336, 8192]",
            lambda: api.quant_mxfp8_rowcol(dY, sr=True, seed=4, stream_id_row=0, stream_id_col=1, out=qrc),
            nbytes=M4 * N4 * (2 + 2 * (1 + 1 / 32)))
        del qrc
        qwc = api.quant_mxfp8(W4, colwise=True, sr=True, seed=4, stream_id=2)
        qw4 = api.quant_nvfp4(W4, block_2d=True)
        qwr = api.requant_nvfp4_mxfp8(qw4[0], qw4[1], qw4[2], sr=True, seed=4, stream_id=2)
        row("f2 NVFP4 -> MXFP8 column-wise requantize SR (next row)", "W 14336x4096 NVFP4 16x16 -> [4096, 14336]",
            lambda: api.requant_nvfp4_mxfp8(qw4[0], qw4[1], qw4[2], sr=True, seed=4, stream_id=2, out=qwr),
            nbytes=N4 * K4 * (0.5 + 1 / 16 + 1 + 1 / 32))
        del qw4, qwr
        qxc = api.quant_mxfp8(X4, colwise=True, sr=True, seed=4, stream_id=3)
        Cd = torch.empty(M4, K4, dtype=torch.bfloat16, device=dev)
        row("a8 MXFP8 GEMM dgrad (bf16 out)", "8192x4096x14336",
            lambda: api.gemm(1, qdr[0], qdr[1], qwc[0], qwc[1], M4, K4, N4, out=Cd), flops=2 * M4 * K4 * N4,
            peak_kind="fp8")
        del Cd
        Cw = torch.empty(N4, K4, dtype=torch.float32, device=dev)
        row("a8 MXFP8 GEMM wgrad (fp32 out)", "14336x4096x8192",
            lambda: api.gemm(1, qdc[0], qdc[1], qxc[0], qxc[1], N4, K4, M4, out=Cw), flops=2 * N4 * K4 * M4,
            peak_kind="fp8")
        del Cw, qdr, qdc, qxc, dY, X4
        qar = api.quant_nvfp4(A_roll.to(dev))
        qwr = api.quant_nvfp4(W4, block_2d=True)
        Cr = torch.empty(64, N4, dtype=torch.bfloat16, device=dev)
        row("a8 NVFP4 rollout GEMM (swap-AB, HBM-bound)", "64x14336x4096",
            lambda: api.gemm(0, qar[0], qar[1], qwr[0], qwr[1], 64, N4, K4, gsA=qar[2], gsB=qwr[2], out=Cr),
            nbytes=N4 * K4 // 2 + N4 * K4 // 16 + 64 * K4 // 2 + 64 * K4 // 16 + 64 * N4 * 2)
        del Cr, qar, qwr, W4, qwc
    if wants("a4 NVFP4 Four Over Six quantize (gathered, expert groups)", "a9 grouped NVFP4 GEMM up", "a9 grouped NVFP4 GEMM down",
             "a4 NVFP4 Four Over Six quantize, each token once then moved to its routed rows",
             "a9+a4 grouped up GEMM, then amax + 4/6 quantize of H (two kernels)",
             "f1 grouped up GEMM with the 4/6 NVFP4 quantize in its epilogue (next row)"):
        # -- MoE forward, 16384 tokens, 64 experts, top-8 (gathered 4/6 quantize, grouped up and down)
        moe = W.moe_forward()
        T3, H3 = moe.X.shape
        E3, F3, _ = moe.W_up.shape
        ri = torch.from_numpy(moe.row_index).to(dev)
        offs = torch.from_numpy(moe.row_offsets).to(dev)
        sfo = torch.from_numpy(moe.sf_row_offsets).to(dev)
        Mt, sf_rows = int(moe.row_offsets[-1]), int(moe.sf_row_offsets[-1])
        Xd = moe.X.to(dev)
        qx = api.quant_nvfp4(Xd, four_over_six=True, row_index=ri, groups=(offs, sfo, sf_rows))
        row("a4 NVFP4 Four Over Six quantize (gathered, expert groups)", "X 16384x4096 -> 131072 routed rows",
            lambda: api.quant_nvfp4(Xd, four_over_six=True, row_index=ri, groups=(offs, sfo, sf_rows), out=qx),
            nbytes=Mt * H3 * (2 + 2 + 0.5 + 1 / 16))

        ws = torch.empty(bsq.bsq_quant_nvfp4_gather_workspace(T3, H3), dtype=torch.uint8, device=dev)
        row("a4 NVFP4 Four Over Six quantize, each token once then moved to its routed rows",
            "X 16384x4096 -> 131072 routed rows",
            lambda: api.quant_nvfp4_gather(Xd, ri, four_over_six=True, groups=(offs, sfo, sf_rows), out=qx,
                                           workspace=ws),
            nbytes=T3 * H3 * 2 + Mt * H3 * (0.5 + 1 / 16))
        del ws

        def experts(Wx):
            E, N, K = Wx.shape
            codes = torch.empty(E, N, K // 2, dtype=torch.uint8, device=dev)
            sfb = torch.zeros(E * bsq.bsq_sf_bytes(N, K // 16), dtype=torch.uint8, device=dev)
            gsb = torch.empty(E, dtype=torch.float32, device=dev)
            per = bsq.bsq_sf_bytes(N, K // 16)
            for e in range(E):
                we = Wx[e].to(dev)
                api.quant_nvfp4(we, block_2d=True, out=(codes[e], sfb[e * per:(e + 1) * per], gsb[e:e + 1]))
            return codes, sfb, gsb
        up = experts(moe.W_up)
        Cup = torch.empty(Mt, F3, dtype=torch.bfloat16, device=dev)
        row("a9 grouped NVFP4 GEMM up", f"{Mt} routed rows x {F3} x {H3}, 64 experts",
            lambda: api.grouped_gemm(0, offs, sfo, qx[0], qx[1], up[0], up[1], Mt, F3, H3, gsA=qx[2], gsB=up[2],
                                     out=Cup), flops=2 * Mt * F3 * H3, peak_kind="fp4")
        qh = api.quant_nvfp4(Cup, four_over_six=True, groups=(offs, sfo, sf_rows))

        def up_then_quantize():
            api.grouped_gemm(0, offs, sfo, qx[0], qx[1], up[0], up[1], Mt, F3, H3, gsA=qx[2], gsB=up[2], out=Cup)
            api.quant_nvfp4(Cup, four_over_six=True, groups=(offs, sfo, sf_rows), out=qh)
        row("a9+a4 grouped up GEMM, then amax + 4/6 quantize of H (two kernels)",
            f"{Mt} routed rows x {F3} x {H3} -> NVFP4 H", up_then_quantize, flops=2 * Mt * F3 * H3, peak_kind="fp4")
        fq = (torch.empty(Mt, F3 // 2, dtype=torch.uint8, device=dev),
              torch.zeros(api.sf_bytes(sf_rows, F3 // 16), dtype=torch.uint8, device=dev),
              torch.empty(1, dtype=torch.float32, device=dev), None)
        row("f1 grouped up GEMM with the 4/6 NVFP4 quantize in its epilogue (next row)",
            f"{Mt} routed rows x {F3} x {H3} -> NVFP4 H",
            lambda: api.grouped_gemm_nvfp4_out(offs, sfo, qx[0], qx[1], up[0], up[1], Mt, F3, H3, qh[2], sf_rows,
                                               gsA=qx[2], gsB=up[2], four_over_six=True, out=fq),
            flops=2 * Mt * F3 * H3, peak_kind="fp4")
        del fq
        del up
        dn = experts(moe.W_dn)
        Cdn = torch.empty(Mt, H3, dtype=torch.bfloat16, device=dev)
        row("a9 grouped NVFP4 GEMM down", f"{Mt} routed rows x {H3} x {F3}, 64 experts",
            lambda: api.grouped_gemm(0, offs, sfo, qh[0], qh[1], dn[0], dn[1], Mt, H3, F3, gsA=qh[2], gsB=dn[2],
                                     out=Cdn), flops=2 * Mt * H3 * F3, peak_kind="fp4")
    del flush, flush_r
    return rows


# ---------------------------------------------------------------------- ours
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    ap.add_argument("--rows-only", default=None, metavar="SUBSTR",
                    help="run only the per-row measurements whose name contains SUBSTR, print them, exit")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, rank)
    if args.rows_only is not None:
        import torch
        hbm, bf16, _ = peaks()
        torch.cuda.set_device(0)
        print(json.dumps(measure_rows(hbm, bf16 * NOMINAL_FP4_OVER_BF16, bf16 * NOMINAL_FP8_OVER_BF16,
                                      reps=max(args.steps, 1), only=args.rows_only)), flush=True)
        return

    import torch
    import torch.distributed as dist

    from fp8_math_b200 import api, bsq
    from fp8_math_b200 import workloads as W

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    # ---- inputs (seeded, resident in HBM before timing)
    A_h, W_h, seed = W.nvfp4_linear_rht()
    mask = bsq.bsq_rht_sign_mask(seed)
    A = A_h.cuda()
    Wd = W_h.cuda()
    dev = A.device
    KB = K // 16
    ca = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    sa = torch.zeros(bsq.bsq_sf_bytes(M, KB), dtype=torch.uint8, device=dev)
    ga = torch.empty(1, dtype=torch.float32, device=dev)
    cw = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
    sw = torch.zeros(bsq.bsq_sf_bytes(N, KB), dtype=torch.uint8, device=dev)
    gw = torch.empty(1, dtype=torch.float32, device=dev)
    Cm = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    s_ptr = stream.cuda_stream

    def q_a():
        bsq.bsq_quant_nvfp4(A, M, K, K, 0, 0, 1, mask, None, 0, None, None, None, ga, ca, sa, s_ptr)

    def q_w():
        bsq.bsq_quant_nvfp4(Wd, N, K, K, 1, 0, 1, mask, None, 0, None, None, None, gw, cw, sw, s_ptr)

    def gemm():
        bsq.bsq_gemm_blockscaled(bsq.BSQ_NVFP4, ca, sa, ga, cw, sw, gw, M, N, K, Cm, N, bsq.BSQ_OUT_BF16, s_ptr)

    def step():
        q_a()
        q_w()
        gemm()

    # A: amax pass + 1x16 quantize pass; W: one launch (amax and 16x16 quantize
    # in one cooperative kernel); the GEMM.  (The 8-byte scratch reset before
    # A's amax pass is a cudaMemsetAsync, not a kernel of the library.)
    launches_per_step = 4

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = bsq.bsq_check()
    if st != bsq.BSQ_OK:
        raise RuntimeError("device error in warm-up: " + bsq.status_str(st))

    # ---- per-kernel breakdown (events on the launching stream)
    def time_fn(fn, reps):
        # one event pair around `reps` back-to-back calls (the event clock
        # ticks in ~2 us steps, too coarse for one call)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return [e0.elapsed_time(e1) / reps]

    # ---- the timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    gemm_ms, qa_ms, qw_ms = [], [], []
    with ClockSampler(local) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        # breakdown pass (same calls, one event pair each; not part of ms_per_step)
        reps = max(10, min(args.steps, 50))
        qa_ms = time_fn(q_a, reps)
        qw_ms = time_fn(q_w, reps)
        gemm_ms = time_fn(gemm, reps)
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1) / args.steps
    st = bsq.bsq_check()
    if st != bsq.BSQ_OK:
        raise RuntimeError("device error in timed region: " + bsq.status_str(st))
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)

    flops = 2.0 * M * N * K
    value = job_tflops(world, flops, ms)

    # ---- end to end through the C ABI with host buffers (pinned), copies timed.
    # Every step copies its inputs host->device and its bf16 product back;
    # the copies of neighbouring steps overlap the kernels (host->device and
    # device->host streams, two device buffer sets), as a serving loop would.
    A_pin = A_h.pin_memory()
    W_pin = W_h.pin_memory()
    C_pins = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    A_b = [A, torch.empty_like(A)]
    W_b = [Wd, torch.empty_like(Wd)]
    C_b = [Cm, torch.empty_like(Cm)]
    h2d = torch.cuda.Stream()
    d2h = torch.cuda.Stream()
    e2e_steps = max(3, min(args.steps, 10))

    def e2e_run(n):
        done_in = [None, None]   # compute finished reading the inputs of buffer b
        done_out = [None, None]  # device->host copy of buffer b finished
        start = torch.cuda.Event()
        start.record(stream)
        for i in range(n):
            b = i & 1
            h2d.wait_event(start)
            if done_in[b] is not None:
                h2d.wait_event(done_in[b])
            with torch.cuda.stream(h2d):
                A_b[b].copy_(A_pin, non_blocking=True)
                W_b[b].copy_(W_pin, non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(h2d)
            stream.wait_event(ready)
            if done_out[b] is not None:
                stream.wait_event(done_out[b])
            bsq.bsq_quant_nvfp4(A_b[b], M, K, K, 0, 0, 1, mask, None, 0, None, None, None, ga, ca, sa, s_ptr)
            bsq.bsq_quant_nvfp4(W_b[b], N, K, K, 1, 0, 1, mask, None, 0, None, None, None, gw, cw, sw, s_ptr)
            bsq.bsq_gemm_blockscaled(bsq.BSQ_NVFP4, ca, sa, ga, cw, sw, gw, M, N, K, C_b[b], N, bsq.BSQ_OUT_BF16,
                                     s_ptr)
            done_in[b] = torch.cuda.Event()
            done_in[b].record(stream)
            d2h.wait_event(done_in[b])
            with torch.cuda.stream(d2h):
                C_pins[b].copy_(C_b[b], non_blocking=True)
            done_out[b] = torch.cuda.Event()
            done_out[b].record(d2h)
        for ev in done_out:
            if ev is not None:
                stream.wait_event(ev)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    st = bsq.bsq_check()
    if st != bsq.BSQ_OK:
        raise RuntimeError("device error in the end-to-end run: " + bsq.status_str(st))
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)

    hbm, bf16, src = peaks()
    fp4_peak = bf16 * NOMINAL_FP4_OVER_BF16
    g_ms = statistics.mean(gemm_ms)
    gemm_tflops = flops / (g_ms * 1e-3) / 1e12
    # algorithmic bytes of a quantize call (amax pass + quantize pass): 2 B read
    # for the amax, then 2 B read + 0.5 B codes + 1/16 B scales per element
    qa_bytes = M * K * (2 + 2 + 0.5 + 1 / 16)
    qw_bytes = N * K * (2 + 2 + 0.5 + 1 / 16)
    qa_gbs = qa_bytes / (statistics.mean(qa_ms) * 1e-3) / 1e9
    qw_gbs = qw_bytes / (statistics.mean(qw_ms) * 1e-3) / 1e9

    rows = None
    if rank == 0 and world == 1 and not args.no_rows:
        del A_pin, W_pin, C_pins, A_b, W_b, C_b
        rows = measure_rows(hbm, fp4_peak, bf16 * NOMINAL_FP8_OVER_BF16)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_line()

    clk_sum = clk.summary()
    mhz = clk_sum.get("sm_mhz")
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "out": "bf16",
                       "l2": "inputs larger than L2 (A+W bf16 = 176 MiB > 126 MB); no flush",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": gemm_tflops / fp4_peak,
                         "traffic": ncu_traffic("gemm_pair_nvfp4_8192x14336x4096.md",
                                                ["fp8_math_b200/csrc/gemm.cu", "fp8_math_b200/csrc/sm100.cuh",
                                                 "fp8_math_b200/csrc/common.cuh", "fp8_math_b200/csrc/nvfp4.cuh"]),
                         "algorithmic_bytes": (M * K + N * K) // 2 + (M + N) * (K // 16) + M * N * 2,
                         "kernel": "gemm_bs2_kernel (NVFP4 8192x14336x4096, CTA pairs)",
                         "peak_source": f"{src} bf16 burst {bf16} x {NOMINAL_FP4_OVER_BF16} (nominal FP4/BF16), "
                                        f"of {src}"},
            "breakdown": {
                "gemm_ms": g_ms, "gemm_tflops": gemm_tflops, "gemm_frac_of_9pf": gemm_tflops / 9000.0,
                # the GEMM's time in SM cycles at the median sampled clock, and its
                # rate scaled to the maximum clock (random FP4 data draws the clock
                # down under the power limit; the MMA rate per cycle is unchanged)
                "gemm_mcycles_at_median_clock": (g_ms * 1e-3 * mhz * 1e6 / 1e6) if mhz else None,
                "gemm_tflops_at_max_clock": (gemm_tflops * clk_sum["sm_max_mhz"] / mhz)
                if mhz and clk_sum.get("sm_max_mhz") else None,
                "quant_A_ms": statistics.mean(qa_ms), "quant_A_gbs": qa_gbs,
                "quant_W_ms": statistics.mean(qw_ms), "quant_W_gbs": qw_gbs,
                "quant_frac_of_hbm": {"A": qa_gbs / hbm, "W": qw_gbs / hbm, "hbm_gbs": hbm, "source": src},
            },
            "e2e": {"value": job_tflops(world, flops, e2e_ms), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": (M + N) * K * 2, "d2h_bytes_per_step": M * N * 2,
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk_sum,
            "cpu_baseline": cpu,
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
