#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 INT8 linear-layer hot path on B200.

One step is one pass of the whole hot path over one batch of synthetic input
of the Llama-3-8B attention-projection workload (K = 4096; fused QKV N = 6144
and O-projection N = 4096; bf16 activations with 0.1% outlier channels x60;
calibration batch 128 x 512 tokens; alpha 0.5; token counts 16/128/1024/4096;
bf16 out):

  1. calibration absmax over the 65536-token batch      (sq_calib_absmax)
  2. smoothing factors for each linear                    (sq_smooth_factors)
  3. smoothed per-output-channel int8 weights             (sq_smooth_quant_weight)
  4. for every token count M and linear: the online linear, sq_quant_act
     then sq_w8a8_gemm (the two kernels sq_linear runs, called separately so
     the GEMM kernel can be timed on its own; with SQ_LINEAR_FUSED=1 up to 32
     tokens run sq_linear's fused kernel instead)

value = int8 operations of all GEMMs in the step (2 M N K each) / step time,
in TOPS, inputs resident in HBM.  e2e = the same through the same C-ABI calls
with the step's inputs copied from pinned host memory and the outputs read
back inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sq|reference]

Under torchrun (N > 1) every rank runs an independent replica of the step on
its own GPU (the path has no exchange step); value is the aggregate over ranks
with the time taken as the maximum over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from w8a8_int8_gemm_channel_b200 import workloads as wls  # noqa: E402

METRIC = "sq_linear INT8 TOPS & GB/s on 1 B200; % of INT8 tensor peak / HBM roofline"
UNIT = "TOPS"
DEFAULT_WORKLOAD = "llama3_8b_attn"

# int8 dense tensor peak = measured bf16 peak x the nominal int8:bf16 ratio (4.5 : 2.25)
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the prefill GEMM kernel (dram__bytes_read.sum +
# dram__bytes_write.sum), keyed by (M, N, K), from the ncu capture summarised
# in the profile named below.
GEMM_TRAFFIC_BYTES = {
    (1024, 6144, 4096): 29417216 + 256,
    (1024, 4096, 4096): 21018880 + 0,
    (4096, 6144, 4096): 42038528 + 3244032,
    (4096, 4096, 4096): 33625600 + 16128,
}
GEMM_TRAFFIC_SOURCE = "profiles/gemm_i8_pair_4096x6144x4096.md"


# ---------------------------------------------------------------------------
# environment helpers
# ---------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {
            "hbm_gbs": float(p["hbm_gbs"]),
            "bf16_tflops": float(p["bf16_tflops"]),
            "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
            "source": "measured",
        }
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, period_ms=50):
        self.period_ms = period_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms), "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, gpu_indices=None):
        if self.proc is None:
            return None
        time.sleep(self.period_ms / 1000.0 * 2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        idx = int(parts[0])
                        rows.append((idx, float(parts[1]), float(parts[2]), parts[5:9]))
                    except ValueError:
                        continue
        finally:
            os.unlink(self.path)
        if gpu_indices is not None:
            rows = [r for r in rows if r[0] in gpu_indices] or rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_max_mhz": max(r[2] for r in rows), "reasons": reasons, "samples": len(rows)}


def visible_gpu_index(local_rank):
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    if cvd:
        ids = [s.strip() for s in cvd.split(",") if s.strip()]
        try:
            return [int(ids[local_rank])]
        except (ValueError, IndexError):
            return None
    return [local_rank]


# ---------------------------------------------------------------------------
# the step (CUDA path, through the C ABI)
# ---------------------------------------------------------------------------

class Step:
    """Inputs, outputs and the C-ABI call sequence of one step of a workload."""

    def __init__(self, wl: wls.Workload, device, base_seed=0):
        import w8a8_int8_gemm_channel_b200 as sq

        self.sq = sq
        self.lib = sq.lib()
        self.wl = wl
        self.device = device
        self.in_dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.out_dt = torch.bfloat16 if wl.out_dtype == "bf16" else torch.float32
        self.in_code = sq.SQ_BF16 if wl.dtype == "bf16" else sq.SQ_F32
        self.out_code = sq.SQ_BF16 if wl.out_dtype == "bf16" else sq.SQ_F32
        lin0 = wl.linears[0]
        K = lin0.K
        assert all(l.K == K for l in wl.linears), "one shared calibration batch needs one K"
        self.K = K
        self.xcal = wls.calibration(wl, lin0, device=device, base_seed=base_seed)
        self.ax = torch.zeros(K, dtype=torch.float32, device=device)
        self.lins = []
        for lin in wl.linears:
            d = {"lin": lin, "w": wls.weight(wl, lin, device=device, base_seed=base_seed),
                 "s": torch.empty(K, dtype=torch.float32, device=device),
                 "wq": torch.empty(lin.N, K, dtype=torch.int8, device=device),
                 "sw": torch.empty(lin.N, dtype=torch.float32, device=device),
                 "x": {}, "y": {}}
            for M in wl.Ms:
                d["x"][M] = wls.inputs(wl, lin, M, device=device, base_seed=base_seed)
                d["y"][M] = torch.empty(M, lin.N, dtype=self.out_dt, device=device)
            self.lins.append(d)
        Mmax = max(wl.Ms)
        self.xq = torch.empty(Mmax, K, dtype=torch.int8, device=device)
        self.sx = torch.empty(Mmax, dtype=torch.float32, device=device)
        self.ws_bytes = max(sq.sq_linear_workspace_size(M, l.N, K) for M in wl.Ms for l in wl.linears)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=device)
        torch.cuda.synchronize()

    # -- algorithmic work ------------------------------------------------------
    def gemm_ops(self):
        return sum(2 * M * d["lin"].N * self.K for d in self.lins for M in self.wl.Ms)

    def input_bytes(self):
        b = self.xcal.numel() * self.xcal.element_size()
        for d in self.lins:
            b += d["w"].numel() * d["w"].element_size()
            b += sum(x.numel() * x.element_size() for x in d["x"].values())
        return b

    def output_bytes(self):
        return sum(y.numel() * y.element_size() for d in self.lins for y in d["y"].values())

    def quant_kernels(self):
        """Kernels one quantiser call launches: one single-pass kernel while
        the factor tables fit shared memory and a row fits 16 chunks per lane
        of 8 warps, else a scale kernel and a code kernel."""
        esize = 2 if self.in_code == self.sq.SQ_BF16 else 4
        nch = self.K * esize // 16
        bb = esize == 2 and self.K * 6 <= 64 * 1024
        smem = self.K * 4 + (self.K * 2 if bb else 0)
        if os.environ.get("SQ_QUANT_KIND") == "2":
            return 2
        return 1 if smem <= 232448 - 1024 and nch <= 32 * 16 * 8 else 2

    def launches_per_step(self):
        """Kernels of this library one step launches: the calibration absmax
        (1); per linear the zeroing of the factors' accumulator, the weight's
        input-channel absmax and the factors (3) and the weight quantiser; per
        token count and linear either the fused linear (1) or the activation
        quantiser and the GEMM (1)."""
        q = self.quant_kernels()
        n = 1
        n += (3 + q) * len(self.lins)
        for M in self.wl.Ms:
            n += len(self.lins) * (1 if self.fused(M) else q + 1)
        return n

    def fused(self, M):
        return self.sq.sq_linear_workspace_size(M, self.lins[0]["lin"].N, self.K) == 0

    # -- the call sequence -------------------------------------------------------
    def run(self, stream, gemm_events=None, stage_events=None, capturing=False):
        """Enqueue one step on `stream`.  gemm_events: list receiving
        (M, N, start, end) around each prefill GEMM; stage_events: list
        receiving (name, start, end) around every call.  capturing: the
        stream is being captured into a CUDA graph (events become graph
        nodes that record on every replay)."""
        lib, K = self.lib, self.K
        st = stream.cuda_stream

        def ev():
            e = torch.cuda.Event(enable_timing=True, external=capturing)
            e.record(stream)
            return e

        def call(name, fn, *args):
            s0 = ev() if stage_events is not None else None
            r = fn(*args)
            if r != 0:
                raise RuntimeError(f"{name}: {self.sq.status_string(r)}")
            if stage_events is not None:
                stage_events.append((name, s0, ev()))

        self.ax.zero_()
        call("calib_absmax", lib.sq_calib_absmax, self.xcal.data_ptr(), self.in_code,
             self.xcal.shape[0], K, K, self.ax.data_ptr(), st)
        for d in self.lins:
            lin = d["lin"]
            call(f"smooth_factors[{lin.name}]", lib.sq_smooth_factors, self.ax.data_ptr(),
                 d["w"].data_ptr(), self.in_code, lin.N, K, self.wl.alpha, d["s"].data_ptr(), None, st)
            call(f"smooth_quant_weight[{lin.name}]", lib.sq_smooth_quant_weight, d["w"].data_ptr(),
                 self.in_code, lin.N, K, d["s"].data_ptr(), d["wq"].data_ptr(), d["sw"].data_ptr(), st)
        for M in self.wl.Ms:
            for d in self.lins:
                lin = d["lin"]
                x, y = d["x"][M], d["y"][M]
                if self.fused(M):
                    call(f"linear[{lin.name},M={M}]", lib.sq_linear, x.data_ptr(), self.in_code,
                         d["s"].data_ptr(), d["wq"].data_ptr(), d["sw"].data_ptr(), M, lin.N, K,
                         y.data_ptr(), self.out_code, None, 0, st)
                    continue
                call(f"quant_act[{lin.name},M={M}]", lib.sq_quant_act, x.data_ptr(), self.in_code,
                     M, K, d["s"].data_ptr(), self.xq.data_ptr(), self.sx.data_ptr(), st)
                g0 = ev() if gemm_events is not None and stage_events is None else None
                call(f"gemm[{lin.name},M={M}]", lib.sq_w8a8_gemm, self.xq.data_ptr(),
                     self.sx.data_ptr(), d["wq"].data_ptr(), d["sw"].data_ptr(), M, lin.N, K,
                     y.data_ptr(), self.out_code, st)
                if g0 is not None:
                    gemm_events.append((M, lin.N, g0, ev()))

    # -- per-stage algorithmic bytes / ops ---------------------------------------------
    def stage_work(self, name):
        """(ops, bytes, bound) for a stage name produced by run()."""
        K = self.K
        ein = 2 if self.in_code == self.sq.SQ_BF16 else 4
        eout = 2 if self.out_code == self.sq.SQ_BF16 else 4
        if name == "calib_absmax":
            return 0, self.xcal.numel() * ein + 8 * K, "hbm"
        lname = name[name.index("[") + 1:name.index("]")].split(",")[0]
        N = next(d["lin"].N for d in self.lins if d["lin"].name == lname)
        if name.startswith("smooth_factors"):
            return 0, N * K * ein + 12 * K, "hbm"
        if name.startswith("smooth_quant_weight"):
            return 0, N * K * ein + 4 * K + N * K + 4 * N, "hbm"
        M = int(name.split("M=")[1].rstrip("]"))
        if name.startswith("quant_act"):
            return 0, M * K * ein + 4 * K + M * K + 4 * M, "hbm"
        ops = 2 * M * N * K
        if name.startswith("gemm"):
            b = M * K + N * K + 4 * (M + N) + M * N * eout
        else:  # fused linear
            b = M * K * ein + 4 * K + N * K + 4 * N + M * N * eout
        bound = "tensor" if ops / b > 600 else "hbm"
        return ops, b, bound


# ---------------------------------------------------------------------------
# CPU oracle baseline (a bounded sample of the same step, scaled to the step)
# ---------------------------------------------------------------------------

class CpuSample:
    """Times the CPU oracle on a bounded sample of every stage of the step and
    scales each stage's time by (full work / sampled work)."""

    def __init__(self, wl: wls.Workload, base_seed=0):
        from oracle import oracle

        self.o = oracle
        self.wl = wl
        lin0 = wl.linears[0]
        self.K = lin0.K
        self.calib_rows = 2048
        self.w_rows = 256
        self.lin_rows = 8
        # seeded CPU draws with the workload's distributions (same recipe, fewer rows)
        self.xcal = self._np(wls.activations(wl, lin0, self.calib_rows, "calib", base_seed=base_seed))
        self.w = {l.name: self._np(wls.weight(wl, l, rows=self.w_rows, base_seed=base_seed))
                  for l in wl.linears}
        self.x = {l.name: self._np(wls.inputs(wl, l, self.lin_rows, base_seed=base_seed)) for l in wl.linears}

    @staticmethod
    def _np(t):
        t = t.contiguous()
        if t.dtype == torch.bfloat16:
            import numpy as np

            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()

    def step(self):
        """Returns (sampled seconds, estimated full-step seconds, ops of the full step)."""
        import numpy as np

        o, wl, K = self.o, self.wl, self.K
        T = wl.calib_tokens
        spent = 0.0
        est = 0.0
        t0 = time.perf_counter()
        ax = o.calib_absmax(self.xcal)
        dt = time.perf_counter() - t0
        spent += dt
        est += dt * T / self.calib_rows
        ops = 0
        for lin in wl.linears:
            w = self.w[lin.name]
            t0 = time.perf_counter()
            aw = o.weight_in_absmax(w)
            s = o.smooth_factors(ax, aw, wl.alpha)
            dt = time.perf_counter() - t0
            spent += dt
            est += dt * lin.N / self.w_rows
            t0 = time.perf_counter()
            wq, sw = o.smooth_quant_weight(w, s)
            dt = time.perf_counter() - t0
            spent += dt
            est += dt * lin.N / self.w_rows
            # the online path for lin_rows tokens against w_rows output channels
            for M in wl.Ms:
                rows = min(M, self.lin_rows)
                t0 = time.perf_counter()
                xq, sx = o.quant_act(self.x[lin.name][:rows], s)
                acc = o.gemm_i32(xq, wq)
                o.dequant(acc, sx, sw, wl.out_dtype)
                dt = time.perf_counter() - t0
                spent += dt
                est += dt * (M / rows) * (lin.N / self.w_rows)
                ops += 2 * M * lin.N * K
        return spent, est, ops

    def describe(self):
        return (f"oracle on {self.calib_rows} of {self.wl.calib_tokens} calibration tokens, "
                f"{self.w_rows} weight rows per linear, and up to {self.lin_rows} tokens per token "
                "count against those rows; each stage's time scaled by full/sampled work")


def cpu_baseline(wl, target_s=12.0):
    samp = CpuSample(wl)
    samp.step()  # warm (builds/loads the oracle)
    spent_total, est_total, ops = 0.0, 0.0, 0
    n = 0
    while spent_total < target_s and n < 5000:
        spent, est, ops = samp.step()
        spent_total += spent
        est_total += est
        n += 1
    est_step = est_total / n
    return {"value": ops / est_step / 1e12, "unit": UNIT, "cores": samp.o.num_threads(),
            "kind": "oracle", "sample": samp.describe() + f"; {n} sampled steps, "
                                                           f"{spent_total:.1f} s of CPU time",
            "est_full_step_s": est_step}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = wls.WORKLOADS[args.workload]
    samp = CpuSample(wl)
    for _ in range(args.warmup):
        samp.step()
    spent_total, est_total, ops = 0.0, 0.0, 0
    budget = 150.0
    steps = 0
    for i in range(args.steps):
        spent, est, ops = samp.step()
        spent_total += spent
        est_total += est
        steps += 1
        if spent_total > budget:
            break
    est_step = est_total / steps
    value = ops / est_step / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
        "warmup": args.warmup, "ms_per_step": est_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "impl": "reference",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": samp.o.num_threads(), "kind": "oracle",
                         "sample": samp.describe() + f"; {steps} sampled steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl):
    lin_desc = {l.name: {"N": l.N, "K": l.K} for l in wl.linears}
    return {"workload": wl.name, "description": wl.description, "linears": lin_desc,
            "M": list(wl.Ms), "calib_tokens": wl.calib_tokens, "alpha": wl.alpha,
            "in_dtype": wl.dtype, "out_dtype": wl.out_dtype,
            "l2": "inputs larger than L2: every step streams the calibration batch "
                  f"({wl.calib_tokens} x {wl.linears[0].K} {wl.dtype}) first",
            "parallelism": "replicas"}


# ---------------------------------------------------------------------------
# single-call cases (per-kernel timing and profiler captures)
# ---------------------------------------------------------------------------

def run_case(spec, steps, warmup, flush_l2=True, settle_us=0.0):
    """Time one C-ABI call on synthetic data.  spec is one of
    gemm:M,N,K  linear:M,N,K  quant_act:M,K  quant_w:N,K  calib:T,K
    smooth_factors:N,K  rmsnorm_quant:M,K  silu_mul_quant:M,I  gptq_hessian:T,K  gptq_factor:K
    gptq_rows:N,K.  Prints one JSON line with the median time."""
    import w8a8_int8_gemm_channel_b200 as sq

    lib = sq.lib()
    kind, dims = spec.split(":")
    d = [int(v) for v in dims.split(",")]
    dev = torch.device("cuda", 0)
    st = torch.cuda.current_stream().cuda_stream
    peaks = load_peaks()
    bf, i8, f32 = torch.bfloat16, torch.int8, torch.float32
    r = lambda *shape, dt=bf, sc=1.0: (torch.randn(*shape, device=dev) * sc).to(dt)
    ops, nbytes = 0, 0
    if kind in ("gemm", "linear"):
        M, N, K = d
        wq = torch.randint(-127, 128, (N, K), device=dev, dtype=i8)
        sw = torch.rand(N, device=dev) * 1e-3
        y = torch.empty(M, N, device=dev, dtype=bf)
        ops = 2 * M * N * K
        if kind == "gemm":
            xq = torch.randint(-127, 128, (M, K), device=dev, dtype=i8)
            sx = torch.rand(M, device=dev)
            fn = lambda: lib.sq_w8a8_gemm(xq.data_ptr(), sx.data_ptr(), wq.data_ptr(), sw.data_ptr(),
                                          M, N, K, y.data_ptr(), sq.SQ_BF16, st)
            nbytes = M * K + N * K + 4 * (M + N) + 2 * M * N
        else:
            x = r(M, K)
            s = torch.rand(K, device=dev) + 0.5
            ws_n = sq.sq_linear_workspace_size(M, N, K)
            ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
            fn = lambda: lib.sq_linear(x.data_ptr(), sq.SQ_BF16, s.data_ptr(), wq.data_ptr(),
                                       sw.data_ptr(), M, N, K, y.data_ptr(), sq.SQ_BF16,
                                       ws.data_ptr() if ws_n else None, ws_n, st)
            nbytes = 2 * M * K + 4 * K + N * K + 4 * N + 2 * M * N
    elif kind == "quant_act":
        M, K = d
        x, s = r(M, K), torch.rand(K, device=dev) + 0.5
        xq, sx = torch.empty(M, K, dtype=i8, device=dev), torch.empty(M, device=dev)
        fn = lambda: lib.sq_quant_act(x.data_ptr(), sq.SQ_BF16, M, K, s.data_ptr(), xq.data_ptr(),
                                      sx.data_ptr(), st)
        nbytes = 3 * M * K + 4 * K + 4 * M
    elif kind == "rmsnorm_quant":
        M, K = d
        h, g = r(M, K), torch.rand(K, device=dev) + 0.5
        xq, sx = torch.empty(M, K, dtype=i8, device=dev), torch.empty(M, device=dev)
        fn = lambda: lib.sq_rmsnorm_quant(h.data_ptr(), sq.SQ_BF16, M, K, g.data_ptr(), 1e-5, xq.data_ptr(),
                                          sx.data_ptr(), None, st)
        nbytes = 3 * M * K + 4 * K + 4 * M
    elif kind == "silu_mul_quant":
        M, I = d
        gu, s = r(M, 2 * I), torch.rand(I, device=dev) + 0.5
        xq, sx = torch.empty(M, I, dtype=i8, device=dev), torch.empty(M, device=dev)
        fn = lambda: lib.sq_silu_mul_quant(gu.data_ptr(), sq.SQ_BF16, M, I, s.data_ptr(), xq.data_ptr(),
                                           sx.data_ptr(), None, st)
        nbytes = 4 * M * I + M * I + 4 * I + 4 * M
    elif kind in ("gptq_hessian", "gptq_factor", "gptq_rows"):
        # GPTQ stages (offline): gptq_hessian:T,K  gptq_factor:K  gptq_rows:N,K
        f64 = torch.float64
        if kind == "gptq_hessian":
            T_, K = d
            x, s = r(T_, K), torch.rand(K, device=dev) + 0.5
            H = torch.empty(K, K, dtype=f64, device=dev)
            fn = lambda: lib.sq_gptq_hessian(x.data_ptr(), sq.SQ_BF16, T_, K, s.data_ptr(), H.data_ptr(), st)
            nbytes = 2 * T_ * K + 8 * K * K
        elif kind == "gptq_factor":
            (K,) = d
            xc = torch.randn(2 * K, K, device=dev, dtype=f64)
            H0 = xc.T @ xc
            H = H0.clone()
            U = torch.empty_like(H)
            ws = torch.empty(int(lib.sq_gptq_workspace_size(K)), dtype=torch.uint8, device=dev)

            def fn():
                H.copy_(H0)
                return lib.sq_gptq_factor(H.data_ptr(), K, 0.01, U.data_ptr(), ws.data_ptr(), ws.numel(), st)
            nbytes = 3 * 8 * K * K
        else:
            N, K = d
            w, s = r(N, K, sc=0.02), torch.rand(K, device=dev) + 0.5
            xc = torch.randn(2 * K, K, device=dev, dtype=f64)
            H = xc.T @ xc
            U = torch.empty_like(H)
            ws = torch.empty(int(lib.sq_gptq_workspace_size(K)), dtype=torch.uint8, device=dev)
            assert lib.sq_gptq_factor(H.data_ptr(), K, 0.01, U.data_ptr(), ws.data_ptr(), ws.numel(), st) == 0
            wq, sw = torch.empty(N, K, dtype=i8, device=dev), torch.empty(N, device=dev)
            fn = lambda: lib.sq_gptq_quant_weight(w.data_ptr(), sq.SQ_BF16, N, K, s.data_ptr(), U.data_ptr(),
                                                  wq.data_ptr(), sw.data_ptr(), st)
            nbytes = 2 * N * K + N * K + 4 * N
    elif kind == "quant_w":
        N, K = d
        w, s = r(N, K, sc=0.02), torch.rand(K, device=dev) + 0.5
        wq, sw = torch.empty(N, K, dtype=i8, device=dev), torch.empty(N, device=dev)
        fn = lambda: lib.sq_smooth_quant_weight(w.data_ptr(), sq.SQ_BF16, N, K, s.data_ptr(),
                                                wq.data_ptr(), sw.data_ptr(), st)
        nbytes = 3 * N * K + 4 * K + 4 * N
    elif kind == "calib":
        T, K = d
        x, ax = r(T, K), torch.zeros(K, device=dev)
        fn = lambda: lib.sq_calib_absmax(x.data_ptr(), sq.SQ_BF16, T, K, K, ax.data_ptr(), st)
        nbytes = 2 * T * K
    elif kind == "smooth_factors":
        N, K = d
        w, ax, s = r(N, K, sc=0.02), torch.rand(K, device=dev) * 10, torch.empty(K, device=dev)
        fn = lambda: lib.sq_smooth_factors(ax.data_ptr(), w.data_ptr(), sq.SQ_BF16, N, K, 0.5,
                                           s.data_ptr(), None, st)
        nbytes = 2 * N * K + 8 * K
    else:
        raise SystemExit(f"unknown case {spec}")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush_l2 else None
    for _ in range(warmup):
        assert fn() == 0
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        if settle_us > 0:
            # idle the GPU after the flush so its write-back does not overlap the call
            torch.cuda._sleep(int(settle_us * 1965))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        rc = fn()
        e1.record()
        assert rc == 0, sq.status_string(rc)
        times.append((e0, e1))
    torch.cuda.synchronize()
    us = statistics.median(a.elapsed_time(b) for a, b in times) * 1e3
    out = {"case": spec, "us": round(us, 2), "settle_us": settle_us, "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1),
           "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 3), "l2_flushed": flush_l2}
    if ops:
        out["TOPS"] = round(ops / (us * 1e-6) / 1e12, 1)
        out["tensor_frac_burst"] = round(out["TOPS"] / (INT8_PER_BF16 * peaks["bf16_tflops"]), 3)
    stc, code = sq.sq_device_status()
    assert stc == 0, f"device error {code:#x}"
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------------------
# replicas: one process per GPU, each running the whole step on its own data
# ---------------------------------------------------------------------------

def max_over_ranks(ms, world, device):
    """The slowest rank's device time; every rank calls this at the same point."""
    if world == 1:
        return ms
    import torch.distributed as dist

    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tops(world, ops_per_step, steps, ms):
    """Whole-job throughput: every replica's ops over the slowest rank's time."""
    return world * ops_per_step * steps / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# main arm
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="sq", choices=["sq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wls.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--breakdown-steps", type=int, default=20)
    ap.add_argument("--case", action="append", default=None,
                    help="time single calls instead of the step, e.g. gemm:4096,6144,4096")
    ap.add_argument("--no-flush", action="store_true")
    ap.add_argument("--settle-us", type=float, default=0.0,
                    help="--case: GPU idle time between the L2 flush and the timed call")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=False,
                    help="replay the step as a CUDA graph in the timed region")
    args = ap.parse_args()
    if args.case:
        for c in args.case:
            run_case(c, args.steps, max(args.warmup, 3), flush_l2=not args.no_flush, settle_us=args.settle_us)
        return 0

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch.distributed as dist

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group(backend="nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(device)
    wl = wls.WORKLOADS[args.workload]
    peaks = load_peaks()
    step = Step(wl, device)
    stream = torch.cuda.Stream(device)

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step.run(stream)
    stream.synchronize()
    st, code = step.sq.sq_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device error word {code:#x} after warm-up")

    # The step as a CUDA graph: S steps per graph (S divides the step count),
    # replayed steps / S times.  The GEMM events inside the graph record on
    # every replay, so after the timed region they hold the last replay's S
    # steps.  Without --graph the steps are enqueued eagerly and every GEMM
    # launch of the timed region is bracketed by its own events.
    graph = None
    gemm_events = []
    per_graph = 1
    if args.graph:
        per_graph = max(d for d in range(1, min(args.steps, 10) + 1) if args.steps % d == 0)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(per_graph):
                step.run(stream, gemm_events=gemm_events, capturing=True)
        for _ in range(2):
            graph.replay()
        stream.synchronize()

    # timed region
    sampler = ClockSampler() if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.2)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        if graph is not None:
            for _ in range(args.steps // per_graph):
                graph.replay()
        else:
            for _ in range(args.steps):
                step.run(stream, gemm_events=gemm_events)
        t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop(visible_gpu_index(local_rank)) if sampler else None
    barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world, device)
    st, code = step.sq.sq_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device error word {code:#x} after the timed region")

    ms_per_step = elapsed_ms / args.steps
    ops_step = step.gemm_ops()
    value = aggregate_tops(world, ops_step, args.steps, elapsed_ms)

    # roofline of the dominant kernel: the prefill tcgen05 GEMM (M >= 1024)
    g_ops = 0
    g_ms = 0.0
    g_n = 0
    g_traffic = []
    for (M, N, e0, e1) in gemm_events:
        if M < 1024:
            continue
        g_ops += 2 * M * N * step.K
        g_ms += e0.elapsed_time(e1)
        g_n += 1
        key = (M, N, step.K)
        if key in GEMM_TRAFFIC_BYTES:
            g_traffic.append(GEMM_TRAFFIC_BYTES[key])
    int8_peak = INT8_PER_BF16 * peaks["bf16_tflops_sustained"]
    achieved = g_ops / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
    roofline = {
        "kernel": "gemm_i8_pair_kernel (tcgen05.mma.cta_group::2 kind::i8, 256-row tiles on CTA pairs)",
        "bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s",
        "frac": (achieved / int8_peak) if achieved else None,
        "traffic": (sum(g_traffic) / len(g_traffic)) if len(g_traffic) == g_n and g_n else None,
        "traffic_source": GEMM_TRAFFIC_SOURCE,
        "peak_note": f"int8 dense = 2 x {peaks['source']} sustained bf16 cuBLAS "
                     f"({peaks['bf16_tflops_sustained']:.0f} TFLOP/s); 'TFLOP/s' here counts int8 ops",
        "launches": g_n, "avg_launch_us": g_ms / max(g_n, 1) * 1e3,
        "events": (f"the timed region's last graph replay ({per_graph} steps)" if graph is not None
                   else "every launch of the timed region"),
        "ops_per_launch": g_ops / max(g_n, 1),
    }

    # per-stage breakdown (separate, untimed pass with an event around every call)
    stages = {}
    if rank == 0 and args.breakdown_steps > 0:
        ev = []
        with torch.cuda.stream(stream):
            for _ in range(args.breakdown_steps):
                step.run(stream, stage_events=ev)
        stream.synchronize()
        acc = {}
        for name, e0, e1 in ev:
            acc.setdefault(name, []).append(e0.elapsed_time(e1))
        for name, ts in acc.items():
            us = statistics.median(ts) * 1e3
            ops, b, bound = step.stage_work(name)
            ent = {"us": round(us, 2), "bound": bound, "GB/s": round(b / (us * 1e-6) / 1e9, 1),
                   "hbm_frac": round(b / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 3)}
            if ops:
                ent["TOPS"] = round(ops / (us * 1e-6) / 1e12, 1)
                ent["tensor_frac"] = round(ops / (us * 1e-6) / 1e12 /
                                           (INT8_PER_BF16 * peaks["bf16_tflops"]), 3)
            stages[name] = ent

    # end to end: every step's inputs copied from pinned host memory and its
    # outputs read back.  Two device buffer sets alternate, so the upload of
    # step i+1 (one copy stream) and the download of step i (another) overlap
    # the computation of step i; each buffer set is reused only after the
    # computation and the download that used it have finished.
    e2e = None
    if not args.no_e2e:
        e2e_steps = args.e2e_steps or max(4, min(args.steps, 20))
        sets = [step, Step(wl, device)]
        h_xcal = step.xcal.cpu().pin_memory()
        h_w = [d["w"].cpu().pin_memory() for d in step.lins]
        h_x = [{M: x.cpu().pin_memory() for M, x in d["x"].items()} for d in step.lins]
        h_y = [[{M: torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for M, y in d["y"].items()}
                for d in step.lins] for _ in range(2)]
        h2d = step.input_bytes()
        d2h = step.output_bytes()
        s_in = torch.cuda.Stream(device)
        s_out = torch.cuda.Stream(device)
        ev = lambda: torch.cuda.Event(enable_timing=False)
        done = [ev(), ev()]      # computation on set b finished
        drained = [ev(), ev()]   # download of set b's outputs finished

        def e2e_step(i):
            b = i % 2
            st = sets[b]
            loaded = ev()
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[b])
                st.xcal.copy_(h_xcal, non_blocking=True)
                for j, d in enumerate(st.lins):
                    d["w"].copy_(h_w[j], non_blocking=True)
                    for M in wl.Ms:
                        d["x"][M].copy_(h_x[j][M], non_blocking=True)
                loaded.record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(loaded)
                if i >= 2:
                    stream.wait_event(drained[b])
                st.run(stream)
                done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[b])
                for j, d in enumerate(st.lins):
                    for M in wl.Ms:
                        h_y[b][j][M].copy_(d["y"][M], non_blocking=True)
                drained[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        stream.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i + 2)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        e2e = {"value": aggregate_tops(world, ops_step, e2e_steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / e2e_steps, "steps": e2e_steps,
               "pipelining": "two device buffer sets; uploads, computation and downloads on three streams"}
        del sets

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": dict(workload_config(wl),
                           launch="cuda_graph" if graph is not None else "eager"),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": step.launches_per_step() * args.steps,
            "clocks": clocks,
            "peaks": peaks,
            "stages": stages,
        }
        print(json.dumps(line), flush=True)
    graph = None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
