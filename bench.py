"""Benchmark of the NVFP4 W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--configs default|none|NAME,NAME,...] [--impl reference]

A step is one pass of the hot path over one batch of seeded synthetic input,
with weights quantized beforehand (a W4A4 checkpoint holds them in NVFP4).
The headline workload (default) is the gated MLP at 32K prefill tokens, the
largest single-GPU configuration:

  mlp32k     X 32768x5120 (5 outlier channels x30) -> quantize X (dynamic
             global) -> gate_up GEMM 34816x5120 whose epilogue applies
             silu(gate)*up and writes bf16 h with its per-CTA max|h| ->
             quantize h (dynamic global) -> down GEMM 5120x17408

Other workloads (--workload, or entries of the `configs` object):
  tiny            X 64x256 @ W 256x256
  outlier         X 8192x5120 (8 channels x50) @ W 5120x5120
  outlier_static  the same with a calibrated static activation global
  gdn_fused       X 8192x5120 @ fused qkv|z|a|b 12384x5120 (fold offline)
  mlp32k_static   the 32K MLP with h quantized in the gate_up epilogue with a
                  calibrated static global (no bf16 h at all)
  mlp32k_unfused  the 32K MLP as separate kernels: GEMM -> silu*mul ->
                  amax + quantize -> GEMM
  decode:M:K:N    few-token layer, e.g. decode:1:5120:17408 (HBM-bound)
Linear workloads run one nvfp4_linear call per step.

Metric: TFLOP/s of the whole step (2*M*N*K summed over its GEMMs, over the
step's device time), with the dominant GEMM's fraction of the dense FP4
tensor peak and the quantizer's GB/s alongside. Inputs stay resident in HBM.
Prefill steps: L2 (126 MB) is flushed before every timed step, outside the
timed events (256 MiB written, then 256 MiB read). Decode steps run back to
back as a CUDA graph over rotating copies of the weights whose total is more
than 3x L2 (as consecutive layers of a model stream their own weights), so
no step finds its weights in L2; the graph is replayed and timed as a whole.
The end-to-end figure moves X from and Y to pinned host memory every step.

Multi-GPU (torchrun): every rank runs the headline step on its own batch
(weak scaling, no collective on the data path); the per-rank device time is
reduced with MAX and the value counts all ranks' FLOPs. The `configs` object
is measured at N=1 only.

--impl reference times the CPU oracle (the plain reference this library is
checked against) on the host cores, on a bounded row sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 W4A4 GEMM TFLOPS incl. act quant, % dense FP4 peak; quant GB/s"
FP4_SPEC_TFLOPS = 9000.0          # B200 dense FP4, public spec
QUANT_BYTES_PER_ELEM = 2.5625     # read bf16 + write 0.5 code + 1/16 scale
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 * 1000 * 1000
HEADLINE = "mlp32k"
DECODE_SHAPES = [f"decode:{m}:{k}:{n}" for (k, n) in ((5120, 17408), (17408, 5120))
                 for m in (1, 8, 32, 128, 256)]
DEFAULT_CONFIGS = ["tiny", "outlier", "gdn_fused", "mlp32k_static", "mlp32k_unfused"] + \
    DECODE_SHAPES


class L2Flush:
    """Evicts L2 (126 MB) between timed steps: writes a 256 MiB buffer, then
    reads a second one, so the flush's own dirty lines are written back here
    and not by the next timed kernel's first reads."""

    def __init__(self):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def __call__(self, value: int = 1):
        self.w.fill_(value & 0xFF)
        self.r.max()


def peaks():
    """Roofline denominators: the measured peaks if present."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        mp = json.load(open(path))
        return {"hbm_gbs": float(mp["hbm_gbs"]), "bf16_tflops": float(mp["bf16_tflops"]),
                "bf16_tflops_sustained": float(mp.get("bf16_tflops_sustained", mp["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None
        self.stamped = True

    def _spawn(self, query: str):
        return subprocess.Popen(
            ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={query}",
             "--format=csv,noheader,nounits", "-lms", "100"],
            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)

    def start(self):
        try:
            self.proc = self._spawn(self.Q)
            time.sleep(0.3)
            if self.proc.poll() is not None:  # query refused: sample without the stamp
                self.stamped = False
                self.proc = self._spawn(self.Q.partition(",")[2])
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            now = time.time()
            self.samples.append(self.parse(line, now) if self.stamped else (now, line.strip()))
        # the stamped query was refused after the start-up check: sample
        # again without the stamp (arrival times) for the rest of the run
        if self.stamped and not self.samples and self.proc.poll() not in (None, 0):
            self.stamped = False
            try:
                self.proc = self._spawn(self.Q.partition(",")[2])
            except Exception:
                return
            for line in self.proc.stdout:
                self.samples.append((time.time(), line.strip()))

    @staticmethod
    def parse(line: str, arrival: float):
        """(sample time, fields after the timestamp). The time is nvidia-smi's
        own stamp (local time, "YYYY/MM/DD HH:MM:SS.mmm"), so output that a
        pipe delivers in bursts still lands in the right window; the arrival
        time if the stamp does not parse (the field is dropped either way)."""
        stamp, _, rest = line.strip().partition(",")
        try:
            whole, _, ms = stamp.strip().partition(".")
            t = time.mktime(time.strptime(whole, "%Y/%m/%d %H:%M:%S")) + float("0." + (ms or "0"))
        except ValueError:
            t = arrival
        return t, rest.strip()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float, extended: bool = False):
        """Median SM clock, max clock and the throttle reasons seen between t0
        and t1: the timed region, or (`extended`) the timed region followed by
        a second of the same step when the timed region alone is shorter than
        a few sample periods. Fewer than 3 samples there: the whole run."""
        rows = [s for (t, s) in self.samples if t0 <= t <= t1]
        window = ("timed region + 1 s of the same step (timed region shorter than the "
                  "sample period)" if extended else "timed region")
        if len(rows) < 3:
            rows = [s for (_, s) in self.samples]
            window = "whole run (fewer than 3 samples in the timed window)"
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            # say why there is no clock record instead of a bare null
            rc = None if self.proc is None else self.proc.poll()
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "window": window,
                    "error": ("nvidia-smi could not be started" if self.proc is None else
                              f"nvidia-smi gave no parseable samples (exit code {rc}, "
                              f"{'stamped' if self.stamped else 'unstamped'} query)")}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "window": window}


# ------------------------------------------------------------- multi-rank --

def rank_x_seed(rank: int) -> int:
    """Each replica quantizes its own batch: per-rank activation seed."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    return wl.SEED_X + 1000 * rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """Device time of the job = the slowest rank (MAX all-reduce)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank's FLOPs over the slowest rank's time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def linear_launches(m: int, k: int, static_global: bool) -> int:
    """Kernels one nvfp4_linear call launches (the library's dispatch): at
    most LINEAR_IN_KERNEL_MAX_TOKENS tokens are quantized inside the GEMM;
    a dynamic global over X above ONE_PASS_MAX_BYTES adds the amax pass."""
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4 as nv
    amax_pass = (not static_global) and m * k * 2 > nv.ONE_PASS_MAX_BYTES
    quantizer = m > nv.LINEAR_IN_KERNEL_MAX_TOKENS
    return 1 + int(quantizer) + int(amax_pass)


def decode_rotation(weight_bytes: int) -> int:
    """Weight copies a decode run rotates over: their total is at least 3x
    L2, so a step's weights were evicted by the others' since its last use."""
    return max(3, math.ceil(3 * L2_BYTES / weight_bytes))


def decode_step_bytes(m: int, n: int, k: int) -> int:
    """Algorithmic bytes of one decode step: weight codes and scales once,
    X in bf16, Y out in bf16 (the quantized X stays in L2 between the
    quantizer and the GEMM and is not counted)."""
    return n * k // 2 + n * k // 16 + m * k * 2 + m * n * 2


# ------------------------------------------------------------------ inputs --

def make_inputs(name: str, rank: int = 0) -> dict:
    """Host (CPU) bf16 tensors of one workload, drawn once and shared by the
    GPU arm and the oracle leg. The activation seed is per rank."""
    from nvfp4_w4a4_quantized_elem_b200 import workloads as wl
    if name in ("tiny", "outlier", "outlier_static"):
        cfg = wl.tiny() if name == "tiny" else wl.outlier()
        cfg.x_seed = rank_x_seed(rank)
        inp = dict(kind="linear", x=cfg.x(), w=cfg.w(), m=cfg.m, n=cfg.n, k=cfg.k,
                   gemms=[(cfg.m, cfg.n, cfg.k)])
        if name == "tiny":
            inp["desc"] = "tiny: X 64x256 ~N(0,1) @ W 256x256 ~N(0,0.02); quantize X + W4A4 GEMM"
        else:
            inp["desc"] = (f"outlier: X {cfg.m}x{cfg.k} bf16 ~N(0,1) with 8 channels x50, "
                           f"W {cfg.n}x{cfg.k} ~N(0,0.02) NVFP4; quantize X + W4A4 GEMM -> bf16")
        if name == "outlier_static":
            # the served recipe's static activation global: calibrated on four
            # other seeded batches of the same distribution (running amax)
            cal = []
            for seed in (101, 102, 103, 104):
                cfg.x_seed = seed
                cal.append(cfg.x())
            inp["calib"] = cal
            inp["desc"] = inp["desc"].replace("quantize X", "quantize X with a calibrated static "
                                              "global")
        return inp
    if name == "gdn_fused":
        cfg = wl.gdn_fused()
        return dict(kind="linear", x=wl.gaussian_bf16(cfg.m, cfg.k, 1.0, rank_x_seed(rank)),
                    w_modules=cfg.weights(), m=cfg.m, n=cfg.n, k=cfg.k,
                    gemms=[(cfg.m, cfg.n, cfg.k)],
                    desc=(f"gdn_fused: X {cfg.m}x{cfg.k} @ fused qkv|z|a|b {cfg.n}x{cfg.k} "
                          "(per-module globals folded offline); quantize X + one fused GEMM"))
    if name in ("mlp32k", "mlp32k_static", "mlp32k_unfused"):
        cfg = wl.mlp32k()
        ch = wl.outlier_channels(cfg.d, cfg.n_outliers)
        x = wl.gaussian_bf16(cfg.m, cfg.d, 1.0, rank_x_seed(rank), ch, cfg.outlier_factor)
        kind = {"mlp32k": "mlp", "mlp32k_static": "mlp_static",
                "mlp32k_unfused": "mlp_unfused"}[name]
        how = {"mlp": ("gate_up GEMM with silu*mul in its epilogue (bf16 h + per-CTA max|h|) -> "
                       "quantize h (dynamic global)"),
               "mlp_static": ("gate_up GEMM with silu*mul + NVFP4 quantization of h (calibrated "
                              "static global) in its epilogue"),
               "mlp_unfused": ("gate_up GEMM (bf16 out) -> silu*mul -> amax + quantize h "
                               "(dynamic global)")}[kind]
        return dict(kind=kind, x=x, w_gate_up=cfg.w_gate_up(), w_down=cfg.w_down(), m=cfg.m,
                    n=cfg.d, k=cfg.d, ffn=cfg.ffn,
                    gemms=[(cfg.m, 2 * cfg.ffn, cfg.d), (cfg.m, cfg.d, cfg.ffn)],
                    desc=(f"{name}: X {cfg.m}x{cfg.d} bf16 ~N(0,1) with {cfg.n_outliers} channels "
                          f"x{cfg.outlier_factor:g} -> quantize X (dynamic global) -> {how} -> "
                          f"down GEMM {cfg.d}x{cfg.ffn}; weights ~N(0,0.02) / ~N(0,0.015) NVFP4"))
    if name.startswith("decode:"):
        m, k, n = (int(v) for v in name.split(":")[1:])
        cfg = wl.decode(m, k, n)
        cfg.x_seed = rank_x_seed(rank)
        return dict(kind="decode", x=cfg.x(), w=cfg.w(), m=m, n=n, k=k, gemms=[(m, n, k)],
                    desc=(f"decode: X {m}x{k} bf16 ~N(0,1) -> nvfp4_linear ("
                          + ("tokens quantized inside the few-token W4A4 GEMM"
                             if m <= 8 else
                             "quantize, then the W4A4 GEMM launched to overlap it")
                          + f") vs W {n}x{k} ~N(0,0.02) NVFP4"))
    raise SystemExit(f"unknown workload {name}")


def make_workload(name: str, inp: dict) -> dict:
    """Device-resident inputs and pre-quantized weights of one workload."""
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4
    wk = dict(inp)
    wk["name"] = name
    wk["x"] = inp["x"].cuda()
    if "w" in inp:
        wk["W"] = nvfp4.quantize(inp["w"].cuda())
    if "w_modules" in inp:
        wk["W"] = nvfp4.fuse_group([nvfp4.quantize(w.cuda()) for w in inp["w_modules"]])
    if "calib" in inp:
        cal = nvfp4.Calibrator()
        for c in inp["calib"]:
            cal.observe(c.cuda())
        wk["x_global"] = cal.global_scale
    if wk["kind"] in ("mlp", "mlp_static", "mlp_unfused"):
        wgu = inp["w_gate_up"].cuda()
        if wk["kind"] == "mlp_unfused":
            wk["Wgu"] = nvfp4.quantize(wgu)
        else:
            wk["Wgi"] = nvfp4.quantize(nvfp4.interleave_gate_up(wgu))
        del wgu
        wk["Wd"] = nvfp4.quantize(inp["w_down"].cuda())
        if wk["kind"] == "mlp_static":
            # offline calibration of h's static global on this batch
            A = nvfp4.quantize(wk["x"])
            ws = nvfp4.swiglu_quant_dynamic_workspace(wk["m"], wk["ffn"])
            nvfp4.gemm_swiglu_quant_dynamic(A, wk["Wgi"], workspace=ws)
            h = ws[:wk["m"] * wk["ffn"] * 2].view(torch.bfloat16).view(wk["m"], wk["ffn"])
            wk["gh"] = nvfp4.Calibrator().observe(h).clone()
            del A, ws, h
    torch.cuda.synchronize()
    return wk


# ----------------------------------------------------------------- the step --

class Step:
    """One pass of the hot path over device-resident inputs.
    linear:       one nvfp4_linear call (its GEMM launch overlaps the
                  quantizer, so no event can sit between them);
    mlp:          quantize X | nvfp4_gemm_swiglu_quant_dynamic | down GEMM;
    mlp_static:   quantize X | nvfp4_gemm_swiglu_quant | down GEMM;
    mlp_unfused:  quantize X | gate_up GEMM | silu*mul + quantize h | down GEMM.
    Events, when given, are recorded at the phase boundaries shown by |."""

    LAUNCHES = {"mlp": 5, "mlp_static": 4, "mlp_unfused": 7}

    def __init__(self, wk, stream):
        from nvfp4_w4a4_quantized_elem_b200 import nvfp4
        self.nv = nvfp4
        self.wk = wk
        self.s = stream
        dev = wk["x"].device
        m, k = wk["x"].shape
        self.kind = wk["kind"]
        self.A = nvfp4.NVFP4Tensor.empty(m, k, dev)
        self.ws = torch.empty(nvfp4.quantize_workspace_bytes(m, k), dtype=torch.uint8, device=dev)
        self.gws = None
        one_pass = m * k * 2 <= nvfp4.ONE_PASS_MAX_BYTES  # quantizer takes the max itself
        if self.kind == "linear":
            n = wk["W"].rows
            self.y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
            nb = nvfp4.gemm_workspace_bytes(m, n, k)
            if nb:
                self.gws = torch.zeros(nb, dtype=torch.uint8, device=dev)
            self.lws = nvfp4.linear_workspace(m, n, k, dev)
            self.launches = linear_launches(m, k, wk.get("x_global") is not None)
            self.nphases = 2
        else:
            ffn = wk["ffn"]
            self.H = nvfp4.NVFP4Tensor.empty(m, ffn, dev)
            self.y = torch.empty((m, wk["n"]), dtype=torch.bfloat16, device=dev)
            if self.kind == "mlp":
                self.hws = nvfp4.swiglu_quant_dynamic_workspace(m, ffn, dev)
            if self.kind == "mlp_unfused":
                self.ygu = torch.empty((m, 2 * ffn), dtype=torch.bfloat16, device=dev)
                self.h = torch.empty((m, ffn), dtype=torch.bfloat16, device=dev)
            self.launches = self.LAUNCHES[self.kind] - (1 if one_pass else 0)
            self.nphases = 5 if self.kind == "mlp_unfused" else 4

    def h_bf16(self):
        """bf16 h of the last step (mlp: in the fused call's workspace)."""
        if self.kind == "mlp":
            m, ffn = self.wk["m"], self.wk["ffn"]
            return self.hws[:m * ffn * 2].view(torch.bfloat16).view(m, ffn)
        return self.h if self.kind == "mlp_unfused" else None

    def run(self, ev=None, x=None, y=None):
        """One step; `x`/`y` replace the resident input/output buffers."""
        nv, wk, s = self.nv, self.wk, self.s
        x = wk["x"] if x is None else x
        y = self.y if y is None else y
        rec = (lambda i: ev[i].record(s)) if ev is not None else (lambda i: None)
        rec(0)
        if self.kind == "linear":
            nv.linear(x, wk["W"], out=y, global_scale=wk.get("x_global"), workspace=self.lws,
                      stream=s)
            rec(1)
            return y
        nv.quantize(x, out=self.A, workspace=self.ws, stream=s)
        rec(1)
        if self.kind == "mlp":
            nv.gemm_swiglu_quant_dynamic(self.A, wk["Wgi"], out=self.H, workspace=self.hws,
                                         stream=s)
            rec(2)
        elif self.kind == "mlp_static":
            nv.gemm_swiglu_quant(self.A, wk["Wgi"], wk["gh"], out=self.H, stream=s)
            rec(2)
        else:
            nv.gemm(self.A, wk["Wgu"], out=self.ygu, stream=s)
            rec(2)
            nv.silu_mul(self.ygu, out=self.h, stream=s)
            nv.quantize(self.h, out=self.H, workspace=self.ws, stream=s)
            rec(3)
        nv.gemm(self.H, wk["Wd"], out=y, stream=s)
        rec(self.nphases - 1)
        return y


def timed(stream, fn, reps, flush=None, tag=1):
    """Mean device time (ms) of fn() over `reps` calls, CUDA events on
    `stream` around each call, L2 flushed before each (outside the events)."""
    evs = []
    with torch.cuda.stream(stream):
        for _ in range(reps):
            if flush is not None:
                flush(tag)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
    stream.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def quantizer_alone(nv, x, stream, flush=None, reps=10):
    """The quantizer kernel alone (static global: no amax pass) over x into
    a scratch output: GB/s of its 2.5625 B per element. Calls run back to
    back in one CUDA graph, each on its own copy of x (R copies totalling
    at least 2x L2, so every call streams its x from HBM), the graph
    replayed and timed as a whole: the kernel's throughput without the
    launch and event cost of a lone call."""
    g = torch.full((1,), 7.0, dtype=torch.float32, device=x.device)
    nbytes = x.shape[0] * x.shape[1] * 2
    R = max(1, math.ceil(2 * L2_BYTES / nbytes))
    xs = [x] + [x.clone() for _ in range(R - 1)]
    outs = [nv.NVFP4Tensor.empty(x.shape[0], x.shape[1], x.device) for _ in range(R)]

    def calls():
        for xi, oi in zip(xs, outs):
            nv.quantize(xi, global_scale=g, out=oi, stream=stream)

    with torch.cuda.stream(stream):
        calls()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        calls()
    n = max(2, math.ceil(reps / R))
    with torch.cuda.stream(stream):
        graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            graph.replay()
        e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1) / (n * R)
    del graph, xs, outs
    elems = x.shape[0] * x.shape[1]
    return {"shape": list(x.shape), "ms": round(ms, 5),
            "gbs": round(elems * QUANT_BYTES_PER_ELEM / (ms * 1e-3) / 1e9, 1),
            "timing": f"{n} replays of a graph of {R} calls on {R} copies of x"}


def gemm_alone(nv, A, B, y, ws, stream, reps=12):
    """The GEMM kernel alone on the step's operands: back-to-back calls in one
    CUDA graph, each on its own copy of A and of Y (R copies, so that each
    call's A and Y total at least 2x L2 over the rotation), the graph
    replayed and timed as a whole: the kernel's duration without the launch
    and event cost of a lone call. Returns (ms per call, description)."""
    per_call = A.codes.numel() + A.sf.numel() + y.numel() * y.element_size()
    R = max(1, math.ceil(2 * L2_BYTES / per_call))
    As = [A] + [nv.NVFP4Tensor(A.codes.clone(), A.sf.clone(), A.global_scale.clone(), A.rows, A.k)
                for _ in range(R - 1)]
    ys = [y] + [torch.empty_like(y) for _ in range(R - 1)]

    def calls():
        for a, yy in zip(As, ys):
            nv.gemm(a, B, out=yy, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        calls()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        calls()
    n = max(2, math.ceil(reps / R))
    with torch.cuda.stream(stream):
        graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            graph.replay()
        e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1) / (n * R)
    del graph, As, ys
    return ms, (f"{n} replays of a CUDA graph of {R} GEMM calls, each on its own copy of A and "
                "Y, one event pair around all")


def cublaslt_reference(A, B, stream, flush, reps=10):
    """The same GEMM through cuBLASLt's NVFP4 path (torch._scaled_mm on the
    step's own codes and swizzled block scales; no global scales, which do
    not change its time), L2 flushed before each call: the library ceiling
    on this machine, reported as context. None where this torch has none."""
    try:
        a = A.codes.view(torch.float4_e2m1fn_x2)
        b = B.codes.view(torch.float4_e2m1fn_x2)
        sa = A.sf.view(torch.float8_e4m3fn)
        sb = B.sf.view(torch.float8_e4m3fn)
        f = lambda: torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
        with torch.cuda.stream(stream):
            f()
        ms = timed(stream, f, reps, flush, 7)
        return round(2 * A.rows * B.rows * A.k / (ms * 1e-3) / 1e12, 1)
    except Exception:
        return None


# A kernel of at least this duration, run back to back inside a multi-kernel
# step, runs under the board's power cap: its roofline takes the sustained
# peak (a seconds-long GEMM loop under the cap); shorter kernels the burst one.
SUSTAINED_MIN_MS = 1.0


def tensor_roofline(name, flops, ms, pk, kernel, lib=None):
    burst = 4.0 * pk["bf16_tflops"]
    sustained = 4.0 * pk["bf16_tflops_sustained"]
    use_sustained = ms >= SUSTAINED_MIN_MS
    fp4_peak = sustained if use_sustained else burst
    tf = flops / (ms * 1e-3) / 1e12
    out = {"bound": "tensor", "achieved": round(tf, 1), "peak": round(fp4_peak, 1),
           "unit": "TFLOP/s", "frac": round(tf / fp4_peak, 4), "traffic": dram_traffic(name),
           "kernel": kernel, "kernel_ms": round(ms, 5),
           "peak_source": (f"4 x bf16 {'sustained' if use_sustained else 'burst'} of "
                           f"{pk['source']} ({pk['bf16_tflops_sustained' if use_sustained else 'bf16_tflops']}"
                           " TF/s; 4 = nominal FP4/BF16 dense ratio); "
                           + ("sustained: a kernel of >= 1 ms inside a long step runs under the "
                              "power cap" if use_sustained else "burst: a kernel timed alone")),
           "frac_of_burst_peak": round(tf / burst, 4),
           "frac_of_sustained_peak": round(tf / sustained, 4),
           "frac_of_fp4_spec_9000": round(tf / FP4_SPEC_TFLOPS, 4),
           "algorithmic_flops_per_launch": flops}
    if lib:
        out["cublaslt_nvfp4_tflops"] = lib
        out["vs_cublaslt"] = round(tf / lib, 4)
    return out


def measure_prefill(wk, stream, flush, steps, warmup, pk, dist=None):
    """Timed steps of a prefill workload + its per-kernel figures."""
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4 as nv
    step = Step(wk, stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush(1)
            step.run()
    stream.synchronize()
    assert nv.read_fault(stream) == 0
    nph = step.nphases
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nph)] for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush(i & 0xFF)  # evict L2 outside the timed events
            step.run(events[i])
    stream.synchronize()
    torch.cuda.synchronize()
    t1 = time.time()
    if dist is not None:
        dist.barrier()
    step_ms = [events[i][0].elapsed_time(events[i][nph - 1]) for i in range(steps)]
    phase_ms = [statistics.mean(events[i][j].elapsed_time(events[i][j + 1]) for i in range(steps))
                for j in range(nph - 1)]
    res = {"step": step, "step_ms_sum": sum(step_ms), "t0": t0, "t1": t1, "phase_ms": phase_ms}
    res["figures"] = prefill_components(wk, step, stream, flush, phase_ms, pk)
    assert nv.read_fault(stream) == 0
    return res


def prefill_components(wk, step, stream, flush, phase_ms, pk):
    """Per-kernel figures of a prefill workload, each kernel (or call) timed
    alone with L2 flushed before each call: the roofline of the dominant
    GEMM, the quantizer's GB/s, the cuBLASLt NVFP4 time of the same GEMM.
    Outputs land in the step's own buffers with the step's own values."""
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4 as nv
    s = stream
    name = wk["name"]
    comp = {}
    if step.kind == "linear":
        qd = timed(s, lambda: nv.quantize(wk["x"], global_scale=wk.get("x_global"), out=step.A,
                                          workspace=step.ws, stream=s), 10, flush, 5)
        g_ms, g_how = gemm_alone(nv, step.A, wk["W"], step.y, step.gws, s)
        (mm, nn, kk) = wk["gemms"][0]
        lib = cublaslt_reference(step.A, wk["W"], s, flush) if mm > 64 else None
        comp["phase_timing"] = ("quantizer (as in the step) launched alone 10 times, CUDA "
                                "events on its stream, L2 flushed before each; GEMM: " + g_how)
        comp["quantize_ms"] = round(qd, 5)
        comp["gemm_ms"] = round(g_ms, 5)
        comp["quant"] = quantizer_alone(nv, wk["x"], s)
        roof = tensor_roofline(name, 2 * mm * nn * kk, g_ms, pk,
                               "nvfp4::gemm::gemm_kernel" if mm > 64 else
                               "nvfp4::skinny::skinny_kernel", lib)
        return comp, roof
    (m1, n1, k1), (m2, n2, k2) = wk["gemms"]
    f1, f2 = 2 * m1 * n1 * k1, 2 * m2 * n2 * k2
    comp["phase_ms"] = [round(v, 5) for v in phase_ms]
    comp["quant_x"] = quantizer_alone(nv, wk["x"], s)
    down_ms = timed(s, lambda: nv.gemm(step.H, wk["Wd"], out=step.y, stream=s), 5, flush, 5)
    comp["down_gemm"] = {"ms": round(down_ms, 5), "tflops": round(f2 / (down_ms * 1e-3) / 1e12, 1)}
    if step.kind == "mlp":
        call_ms = timed(s, lambda: nv.gemm_swiglu_quant_dynamic(step.A, wk["Wgi"], out=step.H,
                                                                workspace=step.hws, stream=s),
                        5, flush, 5)
        comp["quant_h"] = quantizer_alone(nv, step.h_bf16(), s, reps=5)
        g_ms = call_ms - comp["quant_h"]["ms"]
        comp["gate_up_call_ms"] = round(call_ms, 5)
        comp["phase_timing"] = (
            "each call alone, 5 times, L2 flushed before each; the fused gate_up GEMM's time = "
            "the nvfp4_gemm_swiglu_quant_dynamic call (GEMM + quantizer over h) minus the "
            "quantizer alone over the same h (inside the call it finds part of h in L2, so the "
            "GEMM time is, if anything, overstated)")
        kernel = "nvfp4::gemm::gemm_kernel (SwiGLU epilogue: bf16 h + per-CTA max|h|)"
        lib = cublaslt_reference(step.A, wk["Wgi"], s, flush, reps=5)
    elif step.kind == "mlp_static":
        g_ms = timed(s, lambda: nv.gemm_swiglu_quant(step.A, wk["Wgi"], wk["gh"], out=step.H,
                                                     stream=s), 5, flush, 5)
        comp["phase_timing"] = "each call alone, 5 times, L2 flushed before each"
        kernel = "nvfp4::gemm::gemm_kernel (SwiGLU + static NVFP4 quantization of h in the epilogue)"
        lib = cublaslt_reference(step.A, wk["Wgi"], s, flush, reps=5)
    else:
        g_ms = timed(s, lambda: nv.gemm(step.A, wk["Wgu"], out=step.ygu, stream=s), 5, flush, 5)
        comp["quant_h"] = quantizer_alone(nv, step.h, s, reps=5)
        comp["phase_timing"] = "each call alone, 5 times, L2 flushed before each"
        kernel = "nvfp4::gemm::gemm_kernel (gate_up, bf16 out)"
        lib = cublaslt_reference(step.A, wk["Wgu"], s, flush, reps=5)
    comp["gate_up_gemm"] = {"ms": round(g_ms, 5), "tflops": round(f1 / (g_ms * 1e-3) / 1e12, 1)}
    roof = tensor_roofline(name, f1, g_ms, pk, kernel, lib)
    roof["other_gemm"] = {"kernel": "nvfp4::gemm::gemm_kernel (down projection)",
                          "achieved": comp["down_gemm"]["tflops"],
                          "frac_of_burst_peak":
                              round(comp["down_gemm"]["tflops"] / (4.0 * pk["bf16_tflops"]), 4),
                          "frac_of_sustained_peak":
                              round(comp["down_gemm"]["tflops"] /
                                    (4.0 * pk["bf16_tflops_sustained"]), 4),
                          "algorithmic_flops_per_launch": f2}
    return comp, roof


class DecodeRun:
    """Decode steps back to back: R copies of the weights (total >= 3x L2)
    and of X, one CUDA graph of R nvfp4_linear steps (each on its own copy;
    the GEMM of each step and the quantizer of the next are launched to
    overlap their predecessors, as in a model's layer sequence), replayed
    as a whole. Also graphs of R GEMMs alone (pre-quantized X) and of R
    quantizer calls alone for the component figures, and R one-step graphs
    for the end-to-end loop."""

    def __init__(self, wk, stream):
        from nvfp4_w4a4_quantized_elem_b200 import nvfp4 as nv
        self.nv, self.wk, self.s = nv, wk, stream
        m, n, k = wk["m"], wk["n"], wk["k"]
        W = wk["W"]
        self.R = decode_rotation(W.codes.numel() + W.sf.numel())
        self.Ws = [W] + [nv.NVFP4Tensor(W.codes.clone(), W.sf.clone(), W.global_scale.clone(),
                                        W.rows, W.k) for _ in range(self.R - 1)]
        self.xs = [wk["x"]] + [wk["x"].clone() for _ in range(self.R - 1)]
        self.ys = [torch.empty((m, n), dtype=torch.bfloat16, device="cuda") for _ in range(self.R)]
        self.lws = nv.linear_workspace(m, n, k)
        self.As = [nv.quantize(x) for x in self.xs]
        nb = nv.gemm_workspace_bytes(m, n, k)
        self.gws = torch.zeros(nb, dtype=torch.uint8, device="cuda") if nb else None
        self.gstatic = torch.full((1,), 7.0, dtype=torch.float32, device="cuda")
        self.Aq = nv.NVFP4Tensor.empty(m, k)
        self.A, self.y = self.As[0], self.ys[0]   # what the oracle leg samples
        self.launches_per_step = linear_launches(m, k, static_global=False)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):      # eager run of every call before capture
            self._linear_all()
            self._gemm_all()
            self._quant_all()
        stream.synchronize()
        self.g_step = self._capture(self._linear_all)
        self.g_gemm = self._capture(self._gemm_all)
        self.g_quant = self._capture(self._quant_all)
        self.g_one = [self._capture(lambda i=i: self._linear(i)) for i in range(self.R)]

    def _linear(self, i):
        self.nv.linear(self.xs[i], self.Ws[i], out=self.ys[i], workspace=self.lws, stream=self.s)

    def _linear_all(self):
        for i in range(self.R):
            self._linear(i)

    def _gemm_all(self):
        for i in range(self.R):
            self.nv.gemm(self.As[i], self.Ws[i], out=self.ys[i], workspace=self.gws,
                         stream=self.s)

    def _quant_all(self):
        for i in range(self.R):
            self.nv.quantize(self.xs[i], global_scale=self.gstatic, out=self.Aq, stream=self.s)

    def _capture(self, fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.s):
            fn()
        self.s.synchronize()
        return g

    def replays(self, g, n):
        """Device ms of n back-to-back replays of graph g (one event pair)."""
        s = self.s
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(n):
                g.replay()
            e1.record(s)
        s.synchronize()
        return e0.elapsed_time(e1)


def measure_decode(wk, stream, steps, warmup, pk, dist=None):
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4 as nv
    run = DecodeRun(wk, stream)
    R = run.R
    n_rep = max(1, math.ceil(steps / R))
    for _ in range(warmup):
        run.replays(run.g_step, 1)
    assert nv.read_fault(stream) == 0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    total_ms = run.replays(run.g_step, n_rep)
    t1 = time.time()
    if dist is not None:
        dist.barrier()
    n_steps = n_rep * R
    # the GEMMs of the linear graph above wrote ys; the components below
    # rewrite them with the same values
    gemm_ms = run.replays(run.g_gemm, n_rep) / n_steps
    quant_ms = run.replays(run.g_quant, n_rep) / n_steps
    run.replays(run.g_step, 1)
    m, n, k = wk["m"], wk["n"], wk["k"]
    step_bytes = decode_step_bytes(m, n, k)
    ms = total_ms / n_steps
    gbs = step_bytes / (ms * 1e-3) / 1e9
    gemm_bytes = n * k // 2 + n * k // 16 + m * k // 2 + m * k // 16 + m * n * 2
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / pk["hbm_gbs"], 4), "traffic": dram_traffic(wk["name"]),
            "kernel": (("nvfp4_linear step: " + ("" if run.launches_per_step == 1 else
                                                  "amax_kernel + ") +
                        "skinny_kernel with in-kernel token quantization")
                       if m <= nv.LINEAR_IN_KERNEL_MAX_TOKENS else
                       ("nvfp4_linear step: quantize_kernel (" +
                        ("takes the max itself" if run.launches_per_step == 2 else
                         "after amax_kernel") + ") + " +
                        ("skinny_kernel" if m <= 64 else "gemm_kernel")))
                      + ", back to back over rotating weight copies",
            "peak_source": f"measured copy bandwidth ({pk['source']})",
            "algorithmic_bytes_per_launch": step_bytes,
            "gemm_alone_us": round(gemm_ms * 1e3, 2),
            "gemm_alone_gbs": round(gemm_bytes / (gemm_ms * 1e-3) / 1e9, 1),
            "gemm_alone_frac": round(gemm_bytes / (gemm_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
    comp = {"weight_copies_rotated": R,
            "weight_bytes_per_copy": run.Ws[0].codes.numel() + run.Ws[0].sf.numel(),
            "quant": {"shape": [m, k], "us_per_call": round(quant_ms * 1e3, 2),
                      "gbs": round(m * k * QUANT_BYTES_PER_ELEM / (quant_ms * 1e-3) / 1e9, 2),
                      "timing": "quantizer alone, static global, R calls in one graph"},
            "timing": (f"{n_rep} replays of one CUDA graph of {R} nvfp4_linear steps "
                       f"(one per weight copy), one event pair around all {n_steps} steps")}
    assert nv.read_fault(stream) == 0
    return {"run": run, "step_ms_sum": total_ms, "n_steps": n_steps, "t0": t0, "t1": t1,
            "figures": (comp, roof)}


def measure_e2e_prefill(step, wk, stream, flops, n):
    """Through the public API with host buffers: every step copies X from
    pinned host memory, runs the hot path and copies Y back to pinned memory.
    Pipelined the way a server streams batches: uploads, compute and
    downloads on three streams with double-buffered device tensors, so step
    i+1's upload and step i-1's download (PCIe is full duplex) overlap step
    i's compute; the timed region spans all n steps' transfers and compute,
    fill and drain included."""
    x_host = wk["x"].cpu().pin_memory()
    y = step.y
    h2d = x_host.numel() * x_host.element_size()
    d2h = y.numel() * y.element_size()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    x_dev = [torch.empty_like(wk["x"]) for _ in range(2)]
    y_dev = [y, torch.empty_like(y)]
    y_host = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(2)]

    def pipeline(k):
        ev = lambda: torch.cuda.Event()
        e_in, e_c, e_out = [ev() for _ in range(k)], [ev() for _ in range(k)], [ev() for _ in range(k)]
        for i in range(k):
            b = i & 1
            if i >= 2:
                s_in.wait_event(e_c[i - 2])          # x_dev[b] read by step i-2
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
            e_in[i].record(s_in)
            stream.wait_event(e_in[i])
            if i >= 2:
                stream.wait_event(e_out[i - 2])      # y_dev[b] downloaded
            with torch.cuda.stream(stream):
                step.run(x=x_dev[b], y=y_dev[b])
            e_c[i].record(stream)
            s_out.wait_event(e_c[i])
            with torch.cuda.stream(s_out):
                y_host[b].copy_(y_dev[b], non_blocking=True)
            e_out[i].record(s_out)
        return e_out[k - 1]

    torch.cuda.synchronize()
    pipeline(2)                                   # warm
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    stream.wait_event(t0)
    s_out.wait_event(t0)
    last = pipeline(n)
    s_out.wait_event(last)
    t1.record(s_out)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    return {"value": flops / (ms * 1e-3) / 1e12, "ms_per_step": ms, "h2d": h2d, "d2h": d2h,
            "schedule": "pipelined: upload / compute / download on three streams, "
                        "double-buffered"}


def measure_e2e_decode(run, wk, stream, flops, n):
    """Serial on one stream, per step: X from pinned host memory to the
    step's device copy, one replay of that copy's one-step graph (the
    nvfp4_linear call), Y back to pinned host memory."""
    x_host = wk["x"].cpu().pin_memory()
    y_host = torch.empty(run.ys[0].shape, dtype=torch.bfloat16, pin_memory=True)
    h2d = x_host.numel() * x_host.element_size()
    d2h = y_host.numel() * y_host.element_size()
    R = run.R

    def one(i):
        run.xs[i % R].copy_(x_host, non_blocking=True)
        run.g_one[i % R].replay()
        y_host.copy_(run.ys[i % R], non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(R):
            one(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            one(i)
        e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1) / n
    return {"value": flops / (ms * 1e-3) / 1e12, "ms_per_step": ms, "h2d": h2d, "d2h": d2h,
            "schedule": "serial on one stream: H2D X, one-step graph replay, D2H Y"}


def code_tokens(src: str) -> str:
    """C/CUDA source without its comments, whitespace runs collapsed: what
    the compiler sees of it (string and character literals kept whole)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(csrc: str | None = None) -> str:
    """Hash of the code of every kernel source (comments and layout
    excluded): a DRAM-traffic figure is only reported while the kernels are
    the ones it was measured on."""
    d = csrc or os.path.join(ROOT, "nvfp4_w4a4_quantized_elem_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")):
            h.update(f.encode())
            h.update(code_tokens(open(os.path.join(d, f), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def dram_traffic(workload: str):
    """DRAM bytes per launch of the roofline's kernel (per step for decode)
    from the committed ncu summary, if it was taken on the current kernel
    sources; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        d = json.load(open(p))
        e = d.get(workload)
        if e and e.get("csrc_sha256_16") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ GPU arm --

def l2_note(kind):
    if kind == "decode":
        return ("inputs larger than L2: steps rotate over weight copies totalling >= 3x L2 "
                "(no flush)")
    return ("flushed before every timed step, outside the events: 256 MiB written, then 256 MiB "
            "read so the flush's dirty lines are written back first")


def run_config(name, args, stream, flush, pk, sampler, rank=0, world=1, dist=None,
               steps=None, cpu_seconds=2.0, headline=False):
    """Build, time and report one workload."""
    steps = steps or args.steps
    inp = make_inputs(name, rank)
    wk = make_workload(name, inp)
    flops = sum(2 * m * n * k for (m, n, k) in wk["gemms"])
    if wk["kind"] == "decode":
        res = measure_decode(wk, stream, steps, args.warmup, pk, dist)
        n_steps = res["n_steps"]
        launches = res["run"].launches_per_step * n_steps
        obj = res["run"]
    else:
        res = measure_prefill(wk, stream, flush, steps, args.warmup, pk, dist)
        n_steps = steps
        launches = res["step"].launches * n_steps
        obj = res["step"]
    comp, roof = res["figures"]
    t0, t1 = res["t0"], res["t1"]
    t2 = t1
    if headline and t1 - t0 < 1.0:
        # one extra second of the same step for the clock record when the
        # timed region is shorter than a few sample periods (no number)
        with torch.cuda.stream(stream):
            end = time.time() + 1.0
            while time.time() < end:
                for _ in range(5):
                    if wk["kind"] == "decode":
                        obj.g_step.replay()
                    else:
                        obj.run()
                stream.synchronize()
        t2 = time.time()
    total_ms = max_over_ranks(res["step_ms_sum"], dist, "cuda")
    ms_per_step = total_ms / n_steps
    value = job_throughput(flops, world, ms_per_step)
    e2e_n = max(3, min(n_steps, 20))
    if wk["kind"] == "decode":
        e2e = measure_e2e_decode(obj, wk, stream, flops, e2e_n)
    else:
        e2e = measure_e2e_prefill(obj, wk, stream, flops, e2e_n)
    e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dist, "cuda")
    e2e["value"] = job_throughput(flops, world, e2e["ms_per_step"])
    rec = {"value": round(value, 2), "unit": "TFLOP/s", "ms_per_step": round(ms_per_step, 5),
           "steps": n_steps, "workload": wk["desc"], "gemms_mnk": wk["gemms"],
           "l2": l2_note(wk["kind"]), "roofline": roof, "components": comp,
           "e2e": {"value": round(e2e["value"], 3), "unit": "TFLOP/s",
                   "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                   "ms_per_step": round(e2e["ms_per_step"], 5), "schedule": e2e["schedule"]},
           "gpu_launches": launches,
           "clocks": sampler.summary(t0, t2, extended=t2 > t1) if sampler else None}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gpu_sample = sample_outputs(obj)
        rec["cpu_baseline"] = cpu_baseline(name, budget_s=cpu_seconds, gpu_sample=gpu_sample,
                                           workload=name, inputs=inp)
    # free this workload's device memory before the next one
    del res, wk, obj
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def run_gpu(args):
    from nvfp4_w4a4_quantized_elem_b200 import build as nb, nvfp4
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        nb.build()
    if dist is not None:
        dist.barrier()
    nvfp4.lib()
    stream = torch.cuda.Stream()
    flush = L2Flush()
    pk = peaks()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)

    head = run_config(args.workload, args, stream, flush, pk, sampler, rank, world, dist,
                      cpu_seconds=args.cpu_seconds, headline=True)
    configs = None
    if world == 1 and args.configs != "none":
        names = DEFAULT_CONFIGS if args.configs == "default" else args.configs.split(",")
        configs = {}
        for name in names:
            if name == args.workload:
                continue
            configs[name] = run_config(name, args, stream, flush, pk, sampler,
                                       steps=min(args.steps, 20),
                                       cpu_seconds=args.config_cpu_seconds)
    sampler.stop()

    out = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": head["steps"],
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1*e2m1 (e4m3 block scales) -> f32 acc -> bf16",
        "data": "synthetic (seeded Gaussian, shapes of a 27B hybrid model's projections)",
        "config": {"workload": head["workload"], "gemms_mnk": head["gemms_mnk"], "l2": head["l2"],
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "roofline": head["roofline"],
        "components": head["components"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if "cpu_baseline" in head:
        out["cpu_baseline"] = head["cpu_baseline"]
    if configs is not None:
        out["configs"] = configs
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------ CPU oracle arm --

def _bits(t):
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_workload(name, inputs=None):
    """The oracle's view of a workload: host X bits (first 1024 rows) and
    the weights quantized by the oracle itself, from the same seeded tensors
    the GPU arm uploads; `x_amax` is max|X| over all of X (over the
    calibration batches for a static global), from which the oracle takes
    the activation global."""
    import oracle as orc
    inp = inputs if inputs is not None else make_inputs(name)
    if inp["kind"] in ("linear", "decode"):
        if "w_modules" in inp:
            qw = orc.fuse_group([orc.quantize(_bits(w)) for w in inp["w_modules"]])
        else:
            qw = orc.quantize(_bits(inp["w"]))
        xa = inp["calib"] if "calib" in inp else [inp["x"]]
        return orc, dict(kind="linear", x_bits=_bits(inp["x"][:1024]), qw=qw,
                         x_amax=max(orc.tensor_amax(_bits(x)) for x in xa),
                         flops_per_row=2 * inp["n"] * inp["k"])
    ffn, d = inp["ffn"], inp["k"]
    return orc, dict(kind="mlp", x_bits=_bits(inp["x"][:1024]),
                     x_amax=orc.tensor_amax(_bits(inp["x"])),
                     qgu=orc.quantize(_bits(inp["w_gate_up"])), qd=orc.quantize(_bits(inp["w_down"])),
                     ffn=ffn, flops_per_row=2 * (2 * ffn) * d + 2 * d * ffn)


def oracle_sample_step(orc, w, rows, times=None):
    """One bounded sample of the step on the CPU oracle: quantize `rows`
    rows of X (dynamic global over the sample) and their FP64 GEMM rows
    (MLP: gate_up, silu*mul on bf16-rounded outputs, requantize h, down).
    `times` (a dict) accumulates the seconds spent quantizing X and in the
    GEMMs."""
    import numpy as np
    rows = min(rows, len(w["x_bits"]))
    xs = w["x_bits"][:rows]
    t0 = time.perf_counter()
    qa = orc.quantize(np.ascontiguousarray(xs))
    t1 = time.perf_counter()
    if w["kind"] == "linear":
        y = orc.gemm(qa, w["qw"])
        if times is not None:
            times["quant"] = times.get("quant", 0.0) + t1 - t0
            times["gemm"] = times.get("gemm", 0.0) + time.perf_counter() - t1
        return y
    y = orc.gemm(qa, w["qgu"])
    yb = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    h = orc.silu_mul(yb)
    return orc.gemm(orc.quantize(h), w["qd"])


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(name, budget_s=15.0, rows=128, gpu_sample=None, workload=None, inputs=None):
    """The oracle as it stands, timed on the host cores on a bounded row
    sample of the workload (scaled per FLOP), with the measured step's
    outputs checked against it on their first rows (`parity`)."""
    orc, w = oracle_workload(name, inputs)
    rows = min(rows, len(w["x_bits"]))
    oracle_sample_step(orc, w, 8)  # warm (builds/loads the oracle)
    t0 = time.perf_counter()
    reps = 0
    times = {}
    while True:
        oracle_sample_step(orc, w, rows, times)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 50:
            break
    tflops = w["flops_per_row"] * rows * reps / el / 1e12
    out = {"value": tflops, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
           "cpu_model": cpu_model(),
           "sample": f"{reps} x ({rows} rows of X: oracle quantize + FP64 GEMM(s) vs the full "
                     f"pre-quantized weights), {el:.1f} s of host time, scaled per FLOP"}
    if times.get("quant"):
        k = w["x_bits"].shape[1]
        out["quant_gbs"] = round(reps * rows * k * QUANT_BYTES_PER_ELEM / times["quant"] / 1e9, 4)
        out["gemm_gflops"] = round(w["flops_per_row"] * rows * reps / times["gemm"] / 1e9, 2)
    if gpu_sample is not None:
        try:
            fn = oracle_parity if w["kind"] == "linear" else oracle_parity_mlp
            out["parity"] = fn(orc, w, workload or name, gpu_sample)
        except Exception as e:  # a report field: never lose the measured line over it
            out["parity"] = {"pass": False, "error": f"{type(e).__name__}: {e}"}
    return out


def sample_outputs(step, rows=128):
    """The first rows of the measured step's output and of its quantized X
    (codes, the first 128-row block of swizzled scales, global), copied to
    the host for the oracle leg. MLP steps add h's NVFP4 rows (codes, first
    scale block, global) and, where the step has a bf16 h, its first rows
    and the whole bf16 h (for max|h|). Taken after the timed steps, whose
    launches all compute these same values."""
    r = min(rows, step.y.shape[0])
    A = step.A
    block = 128 * (-(-A.k // 64) * 4)  # one row block of swizzled scales
    if step.y.is_cuda:
        torch.cuda.synchronize()
    out = dict(rows=r, y=step.y[:r].float().cpu().numpy(), codes=A.codes[:r].cpu().numpy(),
               sf=A.sf[:block].cpu().numpy(), g=A.global_scale.cpu().numpy()[0])
    H = getattr(step, "H", None)
    if H is not None:
        hblock = 128 * (-(-H.k // 64) * 4)
        out.update(h_codes=H.codes[:r].cpu().numpy(), h_sf=H.sf[:hblock].cpu().numpy(),
                   h_g=H.global_scale.cpu().numpy()[0], h_k=H.k)
        h = step.h_bf16()
        if h is not None:
            h_host = h.cpu()
            out.update(h_rows=_bits(h_host[:r]), h_full=_bits(h_host))
    return out


def _x_checks(orc, w, gpu):
    """The sampled X rows quantized by the oracle with the global it derives
    from the seeded inputs (2688 / max|X| over the whole X, or the running
    max over the calibration batches): codes, first scale block and global
    must be the GPU's, bit for bit."""
    import numpy as np
    g = orc.global_from_amax(w["x_amax"])
    r = gpu["rows"]
    qa = orc.quantize(np.ascontiguousarray(w["x_bits"][:r]), global_in=g)
    blk = gpu["sf"].size
    exact = (np.array_equal(gpu["codes"], qa.codes) and
             np.array_equal(gpu["sf"], qa.sf_swizzled[:blk]) and
             np.float32(gpu["g"]).view(np.uint32) == np.float32(g).view(np.uint32))
    return qa, bool(exact)


def _y_checks(orc, qa, qw, y_gpu):
    """Y rows against the FP64 oracle GEMM: relative Frobenius error vs the
    result rounded to bf16 (limit 1e-3), and the worst excess over the
    per-element bound 2e-2 ||x_m|| ||w_n|| (must be <= 0)."""
    import numpy as np
    ref = torch.from_numpy(orc.gemm(qa, qw)).to(torch.bfloat16).double().numpy()
    err = y_gpu.astype(np.float64) - ref
    fro = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    col = np.concatenate([np.linalg.norm(orc.dequantize_rows(qw, np.arange(i, min(i + 1024, qw.rows))),
                                         axis=1) for i in range(0, qw.rows, 1024)])
    row = np.linalg.norm(orc.dequantize(qa), axis=1)
    excess = float(np.max(np.abs(err) - 2e-2 * row[:, None] * col[None, :]))
    return fro, excess


def oracle_parity(orc, w, workload, gpu):
    """The measured step against the oracle on its first rows: quantized X
    bit-exact (see _x_checks), Y within the GEMM tolerance."""
    import numpy as np
    qa, x_exact = _x_checks(orc, w, gpu)
    fro, excess = _y_checks(orc, qa, w["qw"], gpu["y"])
    ok = bool(x_exact and fro <= 1e-3 and excess <= 0.0 and np.all(np.isfinite(gpu["y"])))
    return {"rows": gpu["rows"], "x_codes_scales_global_bit_exact": bool(x_exact),
            "y_rel_fro": fro, "y_rel_fro_limit": 1e-3,
            "y_worst_excess_over_elem_bound": excess, "pass": ok}


def oracle_parity_mlp(orc, w, workload, gpu):
    """The measured MLP step against the oracle on its first rows:
    quantized X bit-exact. Where the step has a bf16 h: h rows within 1e-3
    relative Frobenius of the oracle's silu*mul of its own (bf16-rounded)
    gate_up rows; h's global bit-equal to 2688 / max|h| (the oracle's max
    over the GPU's whole bf16 h); h's codes and first scale block bit-equal
    to the oracle's quantization of the GPU's h rows with that global. Y
    rows within the GEMM tolerance of the oracle's down GEMM on the GPU's
    quantized h rows."""
    import numpy as np
    qa, x_exact = _x_checks(orc, w, gpu)
    r = gpu["rows"]
    rep = {"rows": r, "x_codes_scales_global_bit_exact": bool(x_exact)}
    ok = x_exact
    if "h_rows" in gpu:
        ygu = orc.gemm(qa, w["qgu"])
        yb = torch.from_numpy(ygu).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        h_ref = torch.from_numpy(orc.silu_mul(yb).view(np.int16)).view(torch.bfloat16).double()
        h_gpu = torch.from_numpy(gpu["h_rows"].view(np.int16)).view(torch.bfloat16).double()
        h_fro = float(torch.linalg.norm(h_gpu - h_ref) / max(float(torch.linalg.norm(h_ref)),
                                                             1e-300))
        gh = orc.global_from_amax(orc.tensor_amax(gpu["h_full"]))
        qh = orc.quantize(np.ascontiguousarray(gpu["h_rows"]), global_in=gh)
        hblk = gpu["h_sf"].size
        h_exact = (np.array_equal(gpu["h_codes"], qh.codes) and
                   np.array_equal(gpu["h_sf"], qh.sf_swizzled[:hblk]) and
                   np.float32(gpu["h_g"]).view(np.uint32) == np.float32(gh).view(np.uint32))
        rep.update(h_rel_fro_vs_oracle_gate_up=h_fro, h_codes_scales_global_bit_exact=bool(h_exact))
        ok = ok and h_exact and h_fro <= 1e-3
    else:
        # no bf16 h in this step: the down GEMM is checked on the GPU's own
        # quantized h rows (codes, the first scale block unswizzled, global)
        k = gpu["h_k"]
        sf_rm = orc.sf_unswizzle(gpu["h_sf"], 128, k)[:r]
        qh = orc.Quantized(np.ascontiguousarray(gpu["h_codes"]), np.ascontiguousarray(sf_rm),
                           np.float32(gpu["h_g"]), r, k)
    fro, excess = _y_checks(orc, qh, w["qd"], gpu["y"])
    ok = bool(ok and fro <= 1e-3 and excess <= 0.0 and np.all(np.isfinite(gpu["y"])))
    rep.update(y_rel_fro=fro, y_rel_fro_limit=1e-3, y_worst_excess_over_elem_bound=excess, pass_=ok)
    rep["pass"] = rep.pop("pass_")
    return rep


def run_reference(args):
    """The CPU oracle on the headline workload (or --workload), on the host
    cores: each step is one bounded row sample of the workload; the line
    carries the same metric, unit and config as the GPU arm's."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = make_inputs(args.workload)
    orc, w = oracle_workload(args.workload, inp)
    rows = min(args.ref_rows, len(w["x_bits"]))
    for _ in range(args.warmup):
        oracle_sample_step(orc, w, 4)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_sample_step(orc, w, rows)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = w["flops_per_row"] * rows / (ms * 1e-3) / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64 (oracle)",
           "data": "synthetic (seeded Gaussian, shapes of a 27B hybrid model's projections)",
           "config": {"workload": inp["desc"], "gemms_mnk": inp["gemms"],
                      "l2": l2_note(inp["kind"]),
                      "parallelism": f"replicas x{world} (independent batches, no collective)"},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(),
                            "kind": "oracle",
                            "sample": f"{rows} rows of X per step: oracle quantize + FP64 "
                                      "GEMM(s), scaled per FLOP"},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE,
                    help="mlp32k | mlp32k_static | mlp32k_unfused | tiny | outlier | "
                         "outlier_static | gdn_fused | decode:M:K:N")
    ap.add_argument("--configs", default="default",
                    help="default | none | comma-separated workload names")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=16)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--config-cpu-seconds", type=float, default=1.5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
