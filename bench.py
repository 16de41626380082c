#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 INT8 linear layer on B200.

The headline step is the online linear of the Llama-3-70B-shaped workload
(the largest configuration): for M = 2048 and 8192 tokens, each of the four
linears (QKV 8192 -> 10240, O 8192 -> 8192, gate/up 8192 -> 57344, down
28672 -> 8192; bf16 activations with 0.1% outlier channels x80, alpha 0.85,
bf16 out) runs ``sq_linear`` -- dynamic per-token int8 quantisation of
X / s, then the int8 x int8 -> int32 tcgen05 GEMM with its dequantising
epilogue -- on weights that were calibrated, smoothed and quantised
beforehand.

    value = sum over the step's calls of 2 M N K int8 operations / step time,
            in TOPS, every input resident in HBM.

The same run also measures, each as its own block of the JSON line:
  * roofline  the dominant kernel (the tcgen05 pair GEMM): a second pass of
              the same steps issues the two calls sq_linear makes
              (sq_quant_act, sq_w8a8_gemm) with CUDA events around every GEMM
              launch; achieved = ops per launch / average launch time;
  * configs   every workload (small, Llama-3-8B attention, MLP and decode,
              Llama-3-70B): per (linear, M) sq_linear and its two kernels,
              each call timed alone with L2 flushed before it; for the decode
              workload also the calls back to back;
  * offline   the preparation stages of every workload (calibration absmax,
              smoothing factors, smoothed int8 weights), each timed alone
              with L2 flushed;
  * e2e       the headline step through sq_linear with the activations
              uploaded from pinned host memory and the outputs read back
              inside the timed region;
  * cpu_baseline  the CPU oracle on a bounded sample of the headline step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sq|reference]

Under torchrun (N > 1) every rank runs an independent replica of the
headline step on its own GPU (the path has no exchange step); value is the
aggregate over ranks, the time the maximum over ranks.  ``--case`` times
single calls (used for the profiler captures).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from w8a8_int8_gemm_channel_b200 import workloads as wls  # noqa: E402

METRIC = "sq_linear INT8 TOPS & GB/s on 1 B200; % of INT8 tensor peak / HBM roofline"
UNIT = "TOPS"
DEFAULT_WORKLOAD = "llama3_70b"
CONFIG_ORDER = ("small", "llama3_8b_attn", "llama3_8b_mlp", "llama3_8b_decode", "llama3_70b")

# int8 dense tensor peak = measured bf16 peak x the nominal int8:bf16 ratio (4.5 : 2.25)
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2

# DRAM bytes (read + write) per launch of the pair GEMM, keyed by (M, N, K),
# from one ncu capture each (--metrics dram__bytes_read.sum,dram__bytes_write.sum)
# of `bench.py --case gemm:M,N,K`, taken on the kernel sources whose digest is
# GEMM_TRAFFIC_DIGEST; reported only while the sources still have that digest.
GEMM_TRAFFIC = {
    (2048, 10240, 8192): 122725376,
    (2048, 8192, 8192): 97641728,
    (2048, 57344, 8192): 710615808,
    (2048, 8192, 28672): 518321152,
    (8192, 10240, 8192): 555117824,
    (8192, 8192, 8192): 454479872,
    (8192, 57344, 8192): 3574615296,
    (8192, 8192, 28672): 2260607744,
}
GEMM_TRAFFIC_DIGEST = "31600fee3b553dd1"


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


def kernel_digest():
    """Digest of the CUDA sources (kernels and launchers)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "w8a8_int8_gemm_channel_b200", "csrc")
    for name in sorted(os.listdir(d)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(d, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


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


def _esize(name):
    return 2 if name == "bf16" else 4


def linear_bytes(M, N, K, ein, eout):
    """Algorithmic HBM bytes of one sq_linear call: X read, s, Wq, sw read, Y written."""
    return M * K * ein + 4 * K + N * K + 4 * N + M * N * eout


def gemm_bytes(M, N, K, eout):
    return M * K + N * K + 4 * (M + N) + M * N * eout


def quant_bytes(M, K, ein):
    return M * K * ein + 4 * K + M * K + 4 * M


def bound_of(ops, nbytes, peaks):
    """Tensor-bound where the arithmetic intensity is above the ridge of the
    measured peaks, else HBM-bound."""
    ridge = INT8_PER_BF16 * peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    return "tensor" if nbytes and ops / nbytes > ridge else "hbm"


def rates(us, ops, nbytes, peaks):
    """TOPS, GB/s and the fraction of the bounding roofline (burst int8 peak
    for tensor-bound calls, measured copy bandwidth for HBM-bound ones)."""
    s = us * 1e-6
    gbs = nbytes / s / 1e9
    ent = {"us": round(us, 2), "GB/s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 3)}
    if ops:
        tops = ops / s / 1e12
        ent["TOPS"] = round(tops, 1)
        ent["tensor_frac"] = round(tops / (INT8_PER_BF16 * peaks["bf16_tflops"]), 3)
    b = bound_of(ops, nbytes, peaks)
    ent["bound"] = b
    ent["frac"] = ent["tensor_frac"] if b == "tensor" else ent["hbm_frac"]
    return ent


# ---------------------------------------------------------------------------
# one workload, prepared on the device through the C ABI
# ---------------------------------------------------------------------------

class Prepared:
    """Inputs, prepared weights and outputs of one workload.

    Per linear: its calibration batch and bf16/fp32 weight (kept for the
    offline block), the smoothing factors, the int8 weight and its scales
    (computed once here by sq_calib_absmax, sq_smooth_factors and
    sq_smooth_quant_weight), and per token count M the activations X and the
    output Y."""

    def __init__(self, wl: wls.Workload, device, base_seed=0, keep_offline_inputs=True):
        import w8a8_int8_gemm_channel_b200 as sq

        self.sq = sq
        self.lib = sq.lib()
        self.wl = wl
        self.device = device
        self.ein = _esize(wl.dtype)
        self.eout = _esize(wl.out_dtype)
        self.in_code = sq.SQ_BF16 if wl.dtype == "bf16" else sq.SQ_F32
        self.out_code = sq.SQ_BF16 if wl.out_dtype == "bf16" else sq.SQ_F32
        out_dt = torch.bfloat16 if wl.out_dtype == "bf16" else torch.float32
        st = torch.cuda.current_stream(device).cuda_stream
        self.lins = []
        for lin in wl.linears:
            K, N = lin.K, lin.N
            d = {"lin": lin, "xcal": wls.calibration(wl, lin, device=device, base_seed=base_seed),
                 "w": wls.weight(wl, lin, device=device, base_seed=base_seed),
                 "ax": torch.zeros(K, dtype=torch.float32, device=device),
                 "s": torch.empty(K, dtype=torch.float32, device=device),
                 "wq": torch.empty(N, K, dtype=torch.int8, device=device),
                 "sw": torch.empty(N, dtype=torch.float32, device=device),
                 "x": {}, "y": {}}
            self._ok("sq_calib_absmax", self.lib.sq_calib_absmax(
                d["xcal"].data_ptr(), self.in_code, d["xcal"].shape[0], K, K, d["ax"].data_ptr(), st))
            self._ok("sq_smooth_factors", self.lib.sq_smooth_factors(
                d["ax"].data_ptr(), d["w"].data_ptr(), self.in_code, N, K, wl.alpha, d["s"].data_ptr(), None, st))
            self._ok("sq_smooth_quant_weight", self.lib.sq_smooth_quant_weight(
                d["w"].data_ptr(), self.in_code, N, K, d["s"].data_ptr(), d["wq"].data_ptr(), d["sw"].data_ptr(),
                st))
            for M in wl.Ms:
                d["x"][M] = wls.inputs(wl, lin, M, device=device, base_seed=base_seed)
                d["y"][M] = torch.empty(M, N, dtype=out_dt, device=device)
            if not keep_offline_inputs:
                d["xcal"] = None
                d["w"] = None
            self.lins.append(d)
        self.ws_bytes = max(sq.sq_linear_workspace_size(M, d["lin"].N, d["lin"].K)
                            for M in wl.Ms for d in self.lins)
        self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=device)
        self.gws_bytes = max(sq.sq_w8a8_gemm_workspace_size(M, d["lin"].N, d["lin"].K)
                             for M in wl.Ms for d in self.lins)
        self.gws = torch.empty(max(self.gws_bytes, 256), dtype=torch.uint8, device=device)
        Mmax = max(wl.Ms)
        Kmax = max(l.K for l in wl.linears)
        self.xq = torch.empty(Mmax * Kmax, dtype=torch.int8, device=device)
        self.sx = torch.empty(Mmax, dtype=torch.float32, device=device)
        torch.cuda.synchronize(device)

    def _ok(self, name, r):
        if r != 0:
            raise RuntimeError(f"{name}: {self.sq.status_string(r)}")

    # -- the calls ---------------------------------------------------------------
    def calls(self):
        """(linear entry, M) in step order: every linear for each token count."""
        return [(d, M) for M in self.wl.Ms for d in self.lins]

    def linear(self, d, M, st):
        lin = d["lin"]
        self._ok(f"sq_linear[{lin.name},M={M}]", self.lib.sq_linear(
            d["x"][M].data_ptr(), self.in_code, d["s"].data_ptr(), d["wq"].data_ptr(), d["sw"].data_ptr(),
            M, lin.N, lin.K, d["y"][M].data_ptr(), self.out_code,
            self.ws.data_ptr() if self.ws_bytes else None, self.ws_bytes, st))

    def quant(self, d, M, st):
        lin = d["lin"]
        self._ok("sq_quant_act", self.lib.sq_quant_act(
            d["x"][M].data_ptr(), self.in_code, M, lin.K, d["s"].data_ptr(), self.xq.data_ptr(),
            self.sx.data_ptr(), st))

    def gemm(self, d, M, st):
        """The GEMM as sq_linear runs it: with its own workspace (sq_w8a8_gemm_ws)."""
        lin = d["lin"]
        self._ok("sq_w8a8_gemm_ws", self.lib.sq_w8a8_gemm_ws(
            self.xq.data_ptr(), self.sx.data_ptr(), d["wq"].data_ptr(), d["sw"].data_ptr(), M, lin.N, lin.K,
            d["y"][M].data_ptr(), self.out_code, self.gws.data_ptr(), self.gws_bytes, st))

    # offline stages of one linear (the weights are re-derived in place)
    def calib(self, d, st):
        lin = d["lin"]
        d["ax"].zero_()
        self._ok("sq_calib_absmax", self.lib.sq_calib_absmax(
            d["xcal"].data_ptr(), self.in_code, d["xcal"].shape[0], lin.K, lin.K, d["ax"].data_ptr(), st))

    def factors(self, d, st):
        lin = d["lin"]
        self._ok("sq_smooth_factors", self.lib.sq_smooth_factors(
            d["ax"].data_ptr(), d["w"].data_ptr(), self.in_code, lin.N, lin.K, self.wl.alpha, d["s"].data_ptr(),
            None, st))

    def quant_weight(self, d, st):
        lin = d["lin"]
        self._ok("sq_smooth_quant_weight", self.lib.sq_smooth_quant_weight(
            d["w"].data_ptr(), self.in_code, lin.N, lin.K, d["s"].data_ptr(), d["wq"].data_ptr(),
            d["sw"].data_ptr(), st))

    # -- work --------------------------------------------------------------------
    def ops(self, d, M):
        return 2 * M * d["lin"].N * d["lin"].K

    def step_ops(self):
        return sum(self.ops(d, M) for d, M in self.calls())

    def step_linear_bytes(self):
        return sum(linear_bytes(M, d["lin"].N, d["lin"].K, self.ein, self.eout) for d, M in self.calls())

    def quant_kernels(self, K):
        """Kernels one quantiser call launches: one single-pass kernel while
        the factor tables fit shared memory and a row fits 16 chunks a lane
        over 8 warps, else a scale kernel and a code kernel."""
        nch = K * self.ein // 16
        bb = self.ein == 2 and K * 6 <= 64 * 1024
        smem = K * 4 + (K * 2 if bb else 0)
        return 1 if smem <= 232448 - 1024 and nch <= 32 * 16 * 8 else 2

    def linear_kernels(self, d, M):
        if self.sq.sq_linear_workspace_size(M, d["lin"].N, d["lin"].K) == 0:
            return 1  # the fused decode kernel
        return self.quant_kernels(d["lin"].K) + 1

    def step_launches(self):
        return sum(self.linear_kernels(d, M) for d, M in self.calls())

    def input_bytes(self):
        return sum(d["x"][M].numel() * d["x"][M].element_size() for d, M in self.calls())

    def output_bytes(self):
        return sum(d["y"][M].numel() * d["y"][M].element_size() for d, M in self.calls())

    def free_offline_inputs(self):
        for d in self.lins:
            d["xcal"] = None
            d["w"] = None


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------

class Flusher:
    """Evicts L2 by reading a buffer twice its size.  A read leaves only clean
    lines behind; a write (a memset) would leave up to a full L2 of dirty
    lines whose write-back then competes with the timed call for HBM."""

    def __init__(self, device):
        self.buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)
        self.out = torch.empty((), dtype=torch.int64, device=device)

    def __call__(self):
        torch.sum(self.buf, 0, dtype=torch.int64, out=self.out)


def time_alone(fn, stream, flush, reps=7, warm=2):
    """Median CUDA-event time (us) of fn(st) on `stream`, L2 flushed before
    every timed call."""
    st = stream.cuda_stream
    with torch.cuda.stream(stream):
        for _ in range(warm):
            fn(st)
        evs = []
        for _ in range(reps):
            flush()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(st)
            e1.record(stream)
            evs.append((e0, e1))
    stream.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3


def config_block(p: Prepared, stream, flush, peaks, reps=7):
    """Every (linear, M) call of a workload timed alone: sq_linear and its two
    kernels (the fused decode kernel has no separate parts)."""
    wl = p.wl
    out = {"workload": wl.name, "description": wl.description, "calls": {}}
    t_lin = 0.0
    ops_all = 0
    bytes_all = 0
    for d, M in p.calls():
        lin = d["lin"]
        N, K = lin.N, lin.K
        ops = p.ops(d, M)
        lb = linear_bytes(M, N, K, p.ein, p.eout)
        us = time_alone(lambda st: p.linear(d, M, st), stream, flush, reps)
        ent = {"M": M, "N": N, "K": K, "linear": rates(us, ops, lb, peaks)}
        if p.sq.sq_linear_workspace_size(M, N, K) > 0:
            uq = time_alone(lambda st: p.quant(d, M, st), stream, flush, reps)
            p.quant(d, M, stream.cuda_stream)  # the codes the GEMM below reads
            ug = time_alone(lambda st: p.gemm(d, M, st), stream, flush, reps)
            ent["quant_act"] = rates(uq, 0, quant_bytes(M, K, p.ein), peaks)
            ent["gemm"] = rates(ug, ops, gemm_bytes(M, N, K, p.eout), peaks)
            ent["gemm"]["call"] = "sq_w8a8_gemm_ws (its counter-clearing kernel included)"
        else:
            ent["fused"] = True
        out["calls"][f"{lin.name},M={M}"] = ent
        t_lin += us
        ops_all += ops
        bytes_all += lb
    out["sum_alone"] = {"TOPS": round(ops_all / (t_lin * 1e-6) / 1e12, 2),
                        "GB/s": round(bytes_all / (t_lin * 1e-6) / 1e9, 1), "us": round(t_lin, 2)}
    return out


def back_to_back(p: Prepared, stream, steps=20, warm=3, graph=False):
    """The workload's calls back to back (launches overlapped), `steps` times:
    (us per pass, GB/s of algorithmic bytes, TOPS).  graph=True captures one
    pass in a CUDA graph and replays it, so the host's per-call launch work
    (argument marshalling, tensor maps, two launches a call) is not in the
    timed region -- the way a decode loop runs its layers."""
    st = stream.cuda_stream
    g = None
    with torch.cuda.stream(stream):
        for _ in range(warm):
            for d, M in p.calls():
                p.linear(d, M, st)
    stream.synchronize()
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for d, M in p.calls():
                p.linear(d, M, st)
        with torch.cuda.stream(stream):
            for _ in range(warm):
                g.replay()
        stream.synchronize()
    with torch.cuda.stream(stream):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            if g is not None:
                g.replay()
            else:
                for d, M in p.calls():
                    p.linear(d, M, st)
        e1.record(stream)
    stream.synchronize()
    del g
    us = e0.elapsed_time(e1) * 1e3 / steps
    return {"us_per_pass": round(us, 2), "GB/s": round(p.step_linear_bytes() / (us * 1e-6) / 1e9, 1),
            "TOPS": round(p.step_ops() / (us * 1e-6) / 1e12, 2), "passes": steps,
            "launch": "one CUDA graph a pass" if graph else "eager, one sq_linear call at a time"}


def offline_block(p: Prepared, stream, flush, peaks, reps=5):
    """Preparation stages of a workload, each timed alone with L2 flushed."""
    out = {}
    for d in p.lins:
        lin = d["lin"]
        N, K = lin.N, lin.K
        T = d["xcal"].shape[0]
        us = time_alone(lambda st: p.calib(d, st), stream, flush, reps)
        out[f"calib_absmax[{lin.name}]"] = dict(rates(us, 0, T * K * p.ein + 4 * K, peaks), T=T, K=K)
        us = time_alone(lambda st: p.factors(d, st), stream, flush, reps)
        out[f"smooth_factors[{lin.name}]"] = dict(rates(us, 0, N * K * p.ein + 12 * K, peaks), N=N, K=K)
        us = time_alone(lambda st: p.quant_weight(d, st), stream, flush, reps)
        out[f"smooth_quant_weight[{lin.name}]"] = dict(rates(us, 0, N * K * p.ein + 4 * K + N * K + 4 * N, peaks),
                                                       N=N, K=K)
    return out


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample of the headline step
# ---------------------------------------------------------------------------

class CpuSample:
    """The online linear of every (linear, M) of a workload, run by the CPU
    oracle on `rows` tokens (all K channels) against `cols` output channels:
    per-token quantisation, int32 GEMM and dequantisation.  The smoothing
    factors come from the oracle on a small calibration sample (untimed)."""

    def __init__(self, wl: wls.Workload, rows=8, cols=256, base_seed=0):
        from oracle import oracle

        self.o = oracle
        self.wl = wl
        self.rows = rows
        self.cols = cols
        self.data = []
        for lin in wl.linears:
            xcal = self._np(wls.activations(wl, lin, 256, "calib_sample", base_seed=base_seed))
            w = self._np(wls.weight(wl, lin, rows=cols, base_seed=base_seed))
            _, _, s, wq, sw = oracle.prepare(xcal, w, wl.alpha)
            x = {M: self._np(wls.activations(wl, lin, min(M, rows), f"x_sample{M}", base_seed=base_seed))
                 for M in wl.Ms}
            self.data.append((lin, s, wq, sw, x))

    @staticmethod
    def _np(t):
        t = t.contiguous()
        if t.dtype == torch.bfloat16:
            import numpy as np

            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()

    def step(self):
        """Runs one sampled step; returns (seconds, int8 ops computed)."""
        o = self.o
        ops = 0
        t0 = time.perf_counter()
        for M in self.wl.Ms:
            for lin, s, wq, sw, x in self.data:
                xq, sx = o.quant_act(x[M], s)
                acc = o.gemm_i32(xq, wq)
                o.dequant(acc, sx, sw, self.wl.out_dtype)
                ops += 2 * xq.shape[0] * wq.shape[0] * lin.K
        return time.perf_counter() - t0, ops

    def describe(self):
        return (f"the oracle's online linear (per-token quantisation, int32 GEMM, dequantisation) for every "
                f"(linear, M) of {self.wl.name} on {self.rows} tokens (all K channels) against {self.cols} "
                f"output channels; throughput = the sample's int8 ops / its wall time")


def cpu_baseline(wl, target_s=12.0):
    samp = CpuSample(wl)
    samp.step()  # warm (loads the oracle)
    spent, ops, n = 0.0, 0, 0
    while spent < target_s and n < 10000:
        t, o = samp.step()
        spent += t
        ops += o
        n += 1
    return {"value": ops / spent / 1e12, "unit": UNIT, "cores": samp.o.num_threads(), "kind": "oracle",
            "sample": samp.describe() + f"; {n} sampled steps, {spent:.1f} s"}


def workload_config(wl, step_desc=True):
    cfg = {"workload": wl.name, "description": wl.description,
           "linears": {l.name: {"N": l.N, "K": l.K} for l in wl.linears},
           "M": list(wl.Ms), "calib_tokens": wl.calib_tokens, "alpha": wl.alpha,
           "in_dtype": wl.dtype, "out_dtype": wl.out_dtype, "parallelism": "replicas", "launch": "eager"}
    if step_desc:
        cfg["step"] = ("sq_linear for every (linear, M), weights calibrated, smoothed and quantised "
                       "beforehand (their stages are timed in `offline`)")
        cfg["l2"] = ("inputs larger than L2: a step reads "
                     f"{sum(l.N * l.K for l in wl.linears) / 1e6:.0f} MB of int8 weights per token count "
                     "and the calls' activations and outputs, so every call starts with its operands cold")
    return cfg


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
    spent, ops = 0.0, 0
    for _ in range(args.steps):
        t, o = samp.step()
        spent += t
        ops += o
    value = ops / spent / 1e12
    cfg = workload_config(wl)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": spent / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic", "impl": "reference",
        "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": samp.o.num_threads(), "kind": "oracle",
                         "sample": samp.describe()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# single-call cases (per-kernel timing and profiler captures)
# ---------------------------------------------------------------------------

def run_case(spec, steps, warmup, flush_l2=True, settle_us=0.0):
    """Time one C-ABI call on synthetic data.  spec is one of
    gemm:M,N,K  linear:M,N,K  quant_act:M,K  quant_w:N,K  calib:T,K
    smooth_factors:N,K  rmsnorm_quant:M,K  silu_mul_quant:M,I  gptq_hessian:T,K  gptq_factor:K
    gptq_rows:N,K  copy:bytes.  Prints one JSON line with the median time."""
    import w8a8_int8_gemm_channel_b200 as sq

    lib = sq.lib()
    kind, dims = spec.split(":")
    d = [int(v) for v in dims.split(",")]
    dev = torch.device("cuda", 0)
    st = torch.cuda.current_stream().cuda_stream
    peaks = load_peaks()
    bf, i8 = torch.bfloat16, torch.int8
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
            if os.environ.get("SQ_BENCH_GEMM_WS", "1") == "1":  # as sq_linear runs it
                gn = sq.sq_w8a8_gemm_workspace_size(M, N, K)
                gws = torch.empty(gn, dtype=torch.uint8, device=dev)
                fn = lambda: lib.sq_w8a8_gemm_ws(xq.data_ptr(), sx.data_ptr(), wq.data_ptr(), sw.data_ptr(),
                                                 M, N, K, y.data_ptr(), sq.SQ_BF16, gws.data_ptr(), gn, st)
            else:
                fn = lambda: lib.sq_w8a8_gemm(xq.data_ptr(), sx.data_ptr(), wq.data_ptr(), sw.data_ptr(),
                                              M, N, K, y.data_ptr(), sq.SQ_BF16, st)
            nbytes = gemm_bytes(M, N, K, 2)
        else:
            x = r(M, K)
            s = torch.rand(K, device=dev) + 0.5
            ws_n = sq.sq_linear_workspace_size(M, N, K)
            ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
            fn = lambda: lib.sq_linear(x.data_ptr(), sq.SQ_BF16, s.data_ptr(), wq.data_ptr(),
                                       sw.data_ptr(), M, N, K, y.data_ptr(), sq.SQ_BF16,
                                       ws.data_ptr() if ws_n else None, ws_n, st)
            nbytes = linear_bytes(M, N, K, 2, 2)
    elif kind == "quant_act":
        M, K = d
        x, s = r(M, K), torch.rand(K, device=dev) + 0.5
        xq, sx = torch.empty(M, K, dtype=i8, device=dev), torch.empty(M, device=dev)
        fn = lambda: lib.sq_quant_act(x.data_ptr(), sq.SQ_BF16, M, K, s.data_ptr(), xq.data_ptr(),
                                      sx.data_ptr(), st)
        nbytes = quant_bytes(M, K, 2)
    elif kind == "rmsnorm_quant":
        M, K = d
        h, g = r(M, K), torch.rand(K, device=dev) + 0.5
        xq, sx = torch.empty(M, K, dtype=i8, device=dev), torch.empty(M, device=dev)
        fn = lambda: lib.sq_rmsnorm_quant(h.data_ptr(), sq.SQ_BF16, M, K, g.data_ptr(), 1e-5, xq.data_ptr(),
                                          sx.data_ptr(), None, st)
        nbytes = quant_bytes(M, K, 2)
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
    elif kind == "copy":
        # device-to-device copy of `bytes` bytes: the bandwidth a kernel of this size can reach
        (n,) = d
        a = torch.empty(n, dtype=torch.uint8, device=dev)
        b = torch.empty_like(a)
        fn = lambda: (b.copy_(a), 0)[1]
        nbytes = 2 * n
    else:
        raise SystemExit(f"unknown case {spec}")
    flush = Flusher(dev) if flush_l2 else None
    for _ in range(warmup):
        assert fn() == 0
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        if flush is not None:
            flush()
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
    out = {"case": spec, "settle_us": settle_us, "l2_flushed": flush_l2}
    out.update(rates(us, ops, nbytes, peaks))
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sq", choices=["sq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wls.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload and offline blocks")
    ap.add_argument("--case", action="append", default=None,
                    help="time single calls instead of the step, e.g. gemm:4096,6144,4096")
    ap.add_argument("--no-flush", action="store_true")
    ap.add_argument("--settle-us", type=float, default=0.0,
                    help="--case: GPU idle time between the L2 flush and the timed call")
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
    step = Prepared(wl, device)
    step.free_offline_inputs()
    stream = torch.cuda.Stream(device)
    st = stream.cuda_stream

    def barrier():
        if world > 1:
            dist.barrier()

    def run_step(call_events=None):
        for d, M in step.calls():
            if call_events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            step.linear(d, M, st)
            if call_events is not None:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(stream)
                call_events.append((d, M, e0, e1))

    # warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            run_step()
    stream.synchronize()
    stc, code = step.sq.sq_device_status(stream)
    if stc != 0:
        raise RuntimeError(f"device error word {code:#x} after warm-up")

    # timed region: `steps` steps of sq_linear over every (linear, M)
    sampler = ClockSampler() if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.2)
    call_events = []
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for _ in range(args.steps):
            run_step(call_events)
        t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop(visible_gpu_index(local_rank)) if sampler else None
    barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world, device)
    stc, code = step.sq.sq_device_status(stream)
    if stc != 0:
        raise RuntimeError(f"device error word {code:#x} after the timed region")
    ms_per_step = elapsed_ms / args.steps
    ops_step = step.step_ops()
    value = aggregate_tops(world, ops_step, args.steps, elapsed_ms)
    burst = INT8_PER_BF16 * peaks["bf16_tflops"]

    # sq_linear calls of the timed region (each bracketed by its own events)
    lin_ms = sum(e0.elapsed_time(e1) for _, _, e0, e1 in call_events)
    lin_ops = sum(step.ops(d, M) for d, M, _, _ in call_events)
    linear_calls = {"calls": len(call_events), "avg_call_us": lin_ms / len(call_events) * 1e3,
                    "TOPS": lin_ops / (lin_ms * 1e-3) / 1e12,
                    "frac_of_burst_int8": lin_ops / (lin_ms * 1e-3) / 1e12 / burst}

    # the dominant kernel: a second pass of the same steps issuing the two
    # calls sq_linear makes, with events around every GEMM launch
    gemm_events = []
    quant_ms = 0.0
    with torch.cuda.stream(stream):
        qev = []
        for _ in range(args.steps):
            for d, M in step.calls():
                q0 = torch.cuda.Event(enable_timing=True)
                q0.record(stream)
                step.quant(d, M, st)
                g0 = torch.cuda.Event(enable_timing=True)
                g0.record(stream)
                step.gemm(d, M, st)
                g1 = torch.cuda.Event(enable_timing=True)
                g1.record(stream)
                gemm_events.append((d, M, g0, g1))
                qev.append((q0, g0))
    stream.synchronize()
    quant_ms = sum(a.elapsed_time(b) for a, b in qev)
    g_ops = sum(step.ops(d, M) for d, M, _, _ in gemm_events if M >= 1024)
    g_ms = sum(e0.elapsed_time(e1) for d, M, e0, e1 in gemm_events if M >= 1024)
    g_n = sum(1 for _, M, _, _ in gemm_events if M >= 1024)
    achieved = g_ops / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
    digest = kernel_digest()
    traffic = None
    if GEMM_TRAFFIC_DIGEST == digest and g_n:
        t = [GEMM_TRAFFIC.get((M, d["lin"].N, d["lin"].K)) for d, M, _, _ in gemm_events if M >= 1024]
        if all(v is not None for v in t):
            traffic = sum(t) / len(t)
    roofline = {
        "kernel": "gemm_i8_pair_kernel (tcgen05.mma.cta_group::2 kind::i8, 256-row tiles on CTA pairs)",
        "bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
        "frac": (achieved / burst) if achieved else None,
        "traffic": traffic,
        "traffic_note": ("ncu dram bytes per launch of this kernel version" if traffic is not None else
                         "null: no ncu capture recorded for the current kernel sources"),
        "kernel_digest": digest,
        "peak_note": (f"int8 dense = 2 x {peaks['source']} burst bf16 cuBLAS ({peaks['bf16_tflops']:.1f} "
                      "TFLOP/s); the timed region is well under a second; 'TFLOP/s' counts int8 ops"),
        "launches": g_n, "avg_launch_us": g_ms / max(g_n, 1) * 1e3, "ops_per_launch": g_ops / max(g_n, 1),
        "events": ("a second pass of the timed steps issuing sq_quant_act and sq_w8a8_gemm_ws (the quantiser "
                   "and the GEMM that sq_linear runs) with CUDA events on the launching stream around every GEMM "
                   "call (which includes its counter-clearing kernel)"),
        "share_of_split_pass": g_ms / (g_ms + quant_ms) if g_ms + quant_ms > 0 else None,
    }

    # per-workload and offline blocks (one GPU only)
    configs = None
    offline = None
    if rank == 0 and world == 1 and not args.no_configs:
        flush = Flusher(device)
        configs = {}
        offline = {}
        for name in CONFIG_ORDER:
            if name == wl.name:
                p = Prepared(wl, device)
            else:
                p = Prepared(wls.WORKLOADS[name], device)
            blk = config_block(p, stream, flush, peaks)
            if name == "llama3_8b_decode":
                note = (f"{sum(l.N * l.K for l in p.wl.linears) / 1e6:.0f} MB of int8 weights rotate through "
                        "every token count, more than L2 holds")
                for key, gr in (("back_to_back", False), ("back_to_back_graph", True)):
                    b2b = back_to_back(p, stream, graph=gr)
                    blk[key] = dict(b2b, hbm_frac=round(b2b["GB/s"] / peaks["hbm_gbs"], 3), l2=note)
            configs[name] = blk
            offline[name] = offline_block(p, stream, flush, peaks)
            del p
            torch.cuda.empty_cache()
        del flush
        torch.cuda.empty_cache()

    # end to end through sq_linear: every step uploads its activations from
    # pinned host memory and reads every output back.  Two device buffer sets
    # alternate so the upload of step i+1 and the download of step i overlap
    # the computation of step i; a set is reused only after the computation
    # and the download that last used it have finished.
    e2e = None
    if not args.no_e2e:
        e2e_steps = args.e2e_steps or max(3, min(args.steps, 6))
        sets = [step, Prepared(wl, device, keep_offline_inputs=False)]
        h_x = [d["x"][M].cpu().pin_memory() for d, M in step.calls()]
        h_y = [[torch.empty(d["y"][M].shape, dtype=d["y"][M].dtype, pin_memory=True) for d, M in step.calls()]
               for _ in range(2)]
        h2d = step.input_bytes()
        d2h = step.output_bytes()
        s_in = torch.cuda.Stream(device)
        s_out = torch.cuda.Stream(device)
        ev = lambda: torch.cuda.Event(enable_timing=False)
        done = [ev(), ev()]
        drained = [ev(), ev()]

        def e2e_step(i):
            b = i % 2
            p = sets[b]
            calls = p.calls()
            loaded = ev()
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[b])
                for j, (d, M) in enumerate(calls):
                    d["x"][M].copy_(h_x[j], non_blocking=True)
                loaded.record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(loaded)
                if i >= 2:
                    stream.wait_event(drained[b])
                for d, M in calls:
                    p.linear(d, M, st)
                done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[b])
                for j, (d, M) in enumerate(calls):
                    h_y[b][j].copy_(d["y"][M], non_blocking=True)
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
               "copies": "activations X of every call uploaded, outputs Y of every call downloaded, each step",
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
            "config": workload_config(wl),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": step.step_launches() * args.steps,
            "clocks": clocks,
            "peaks": peaks,
            "step_linear": {"GB/s": step.step_linear_bytes() * args.steps / (elapsed_ms * 1e-3) / 1e9,
                            "frac_of_burst_int8": value / world / burst},
            "linear_calls": linear_calls,
            "configs": configs,
            "offline": offline,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
