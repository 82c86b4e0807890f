#!/usr/bin/env python
"""Throughput benchmark of the quantized linear layers on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qlin|reference]
                    [--no-suite]

Headline workload (the JSON line's value): BitLinear ternary decode GEMV,
K = N = 4096, M in {1, 8}, multiply and divide scale modes.  One step = the
four layer calls.  Weights rotate over device copies whose total exceeds the
L2 cache, so every launch streams its weights from HBM.  The K timed steps run
as CUDA-graph replays between CUDA events on the launching stream, bracketed
by a barrier and a device synchronise; multi-GPU runs take the maximum time
over ranks (weak scaling: every rank runs its own copy of the workload, no
collective on the data path).

The "suite" key times every other hot-path operation (MLX-affine decode and
prefill, W8A8 / W4A8 at M in {1, 256, 4096}, the raw int8 GEMM, quantize /
dequantize and the per-token activation quantiser) with its own roofline.

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "qlinear weight-GB/s at M≤16 & TFLOP/s (TOPS) at M≥256, % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense int8 : bf16 tensor-core ratio on B200 (4.5 : 2.25 POPS)


# ---------------------------------------------------------------- environment

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# The source files each recorded kernel is compiled from (its own .cu and the
# shared header of device helpers): its ncu counters stay valid while these hash
# the same.
KERNEL_SOURCES = {
    "bitlinear_kernel": ("k_bitlinear.cu", "qlin_common.cuh"),
}


def kernel_source_hash(kernel_key: str = "bitlinear_kernel") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_linear_qmm_b200", "csrc")
    for name in KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the
    kernel's current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path) or kernel_key not in KERNEL_SOURCES:
        return None
    want = kernel_source_hash(kernel_key)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 3 and not line.startswith("#") and parts[0] == kernel_key and parts[1] == want:
                return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [s.strip() for s in line.split(",")]
                if len(p) >= 10:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r[4].isdigit() and int(r[4]) >= 50] or rows

        def num(s):
            try:
                return float(s)
            except ValueError:
                return float("nan")
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in load:
            for name, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([num(r[1]) for r in load])),
                "sm_max_mhz": float(np.max([num(r[2]) for r in rows])),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ---------------------------------------------------------------- timing

def time_windows(step_fn, steps: int, warmup: int, windows: int = 5, soak_s: float = 0.0, barrier=None) -> dict:
    """Times exactly `steps` steps as `windows` back-to-back CUDA-graph replays (each a window of
    steps // windows steps; the last also takes the remainder), with a CUDA event between windows on
    the launching stream.  Returns ms per step over all the steps ("ms") and the median, min and
    max of the windows' ms per step."""
    windows = max(1, min(windows, steps))
    per = steps // windows
    sizes = [per] * windows
    sizes[-1] += steps - per * windows
    for i in range(warmup):
        step_fn(i)
    torch.cuda.synchronize()
    graphs = {}
    for n in set(sizes):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                step_fn(i)
        graphs[n] = g
    for g in graphs.values():
        g.replay()  # untimed: the first replay uploads the graph
    torch.cuda.synchronize()
    if soak_s > 0:
        t0 = time.time()
        while time.time() - t0 < soak_s:
            graphs[sizes[0]].replay()
            torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(windows + 1)]
    ev[0].record()
    for w, n in enumerate(sizes):
        graphs[n].replay()
        ev[w + 1].record()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    per_step = [ev[w].elapsed_time(ev[w + 1]) / n for w, n in enumerate(sizes)]
    total = ev[0].elapsed_time(ev[-1])
    del graphs
    return {"ms": total / steps, "median": float(np.median(per_step)), "min": float(np.min(per_step)),
            "max": float(np.max(per_step)), "windows": windows}


def time_steps(step_fn, steps: int, warmup: int, **kw) -> float:
    """Median over 5 windows of ms per step (see time_windows)."""
    return time_windows(step_fn, steps, warmup, **kw)["median"]


def _copies(bytes_per_copy: int, l2_bytes: int, minimum: int = 2) -> int:
    """Copies whose total is at least twice the L2 size."""
    return max(minimum, int(math.ceil(2 * l2_bytes / max(1, bytes_per_copy))))


# ---------------------------------------------------------------- headline workload

class BitlinearDecode:
    """BitLinear ternary decode GEMV: x bf16 [M, 4096], packed uint8 [1024, 4096],
    M in {1, 8}, weight_scale 0.5, multiply and divide modes; no bias."""
    key = "bitlinear_kernel"
    unit = "GB/s"
    bound = "hbm"

    def __init__(self, l2_bytes: int):
        from bit_quantized_linear_qmm_b200 import qlin
        self.ql = qlin
        self.cases = synth.BITLINEAR_DECODE
        c0 = self.cases[0]
        self.K, self.N = c0.K, c0.N
        self.wbytes = self.N // 4 * self.K
        packed = torch.from_numpy(c0.packed()).cuda()
        self.copies = _copies(self.wbytes, l2_bytes, 8)
        self.pool = [packed.clone() for _ in range(self.copies)]
        self.xs = [c.x().torch("cuda") for c in self.cases]
        self.ys = [torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda") for c in self.cases]
        self.ws = torch.tensor([c0.weight_scale], dtype=torch.float32, device="cuda")
        self.launches_per_step = len(self.cases)
        self.units_per_step = self.wbytes * len(self.cases)
        self.alg_bytes_per_launch = self.wbytes
        self.config = {
            "workload": "bitlinear ternary decode GEMV: x bf16 [M,4096] ~N(0,1), M in {1,8}; packed uint8 "
                        "[1024,4096] (codes uniform {0,1,2}, 4 per byte along N); weight_scale 0.5, multiply and "
                        "divide modes; no bias; y bf16 [M,4096]",
            "layers_per_step": len(self.cases), "K": self.K, "N": self.N, "M": [c.M for c in self.cases],
            "weight_bytes_per_layer": self.wbytes,
            "x_plus_y_bytes_per_step": int(sum(c.M * (c.K + c.N) * 2 for c in self.cases)),
            "l2": f"inputs larger than L2: weights rotate over {self.copies} device copies "
                  f"({self.copies * self.wbytes / 1e6:.0f} MB > {l2_bytes / 1e6:.0f} MB L2)",
        }

    def step(self, i: int):
        for c, case in enumerate(self.cases):
            w = self.pool[(i * len(self.cases) + c) % self.copies]
            self.ql.bitlinear_matmul(self.xs[c], w, case.N, self.ws, case.invert, out=self.ys[c])

    def e2e_prepare(self):
        """The step's inputs (x of the 4 layers) in one pinned host buffer and its results (y) in
        another, so each step moves them with one copy each way.  Two device copies of the input
        buffer: while a step runs its 4 layers on one, the next step's input is copied into the
        other on a side stream; the step then reads its own result back.  Every step still moves
        exactly its input in and its result out."""
        nx = [x.numel() for x in self.xs]
        ny = [y.numel() for y in self.ys]
        self.hx = torch.cat([x.reshape(-1).cpu() for x in self.xs]).pin_memory()
        self.dx2 = [torch.empty_like(self.hx, device="cuda") for _ in range(2)]
        self.hy = torch.empty(sum(ny), dtype=self.ys[0].dtype).pin_memory()
        self.dy = torch.empty_like(self.hy, device="cuda")
        self.xs2 = [[v.view(c.M, c.K) for v, c in zip(torch.split(d, nx), self.cases)] for d in self.dx2]
        self.ys = [v.view(c.M, c.N) for v, c in zip(torch.split(self.dy, ny), self.cases)]
        for d in self.dx2:
            d.copy_(self.hx)
        self.side = torch.cuda.Stream()
        self.h2d = self.hx.numel() * self.hx.element_size()
        self.d2h = self.hy.numel() * self.hy.element_size()

    def e2e_step(self, i: int):
        cur = torch.cuda.current_stream()
        b = i % 2
        self.side.wait_stream(cur)  # the other input buffer was last read by the previous step
        with torch.cuda.stream(self.side):
            self.dx2[1 - b].copy_(self.hx, non_blocking=True)  # the next step's input
        self.xs = self.xs2[b]
        self.step(i)
        self.hy.copy_(self.dy, non_blocking=True)  # this step's result
        cur.wait_stream(self.side)


def cpu_bitlinear_step():
    """One step of the headline workload on the host cores with the oracle; returns weight bytes."""
    import oracle
    cases = synth.BITLINEAR_DECODE
    P = cases[0].packed()
    done = 0
    for case in cases:
        oracle.bitlinear(case.x().vals, P, case.N, case.weight_scale, case.invert)
        done += case.N // 4 * case.K
    return done


def cpu_baseline(budget_s: float = 12.0):
    import oracle
    oracle.build()
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    t0 = time.perf_counter()
    units = cpu_bitlinear_step()
    steps = 1
    while time.perf_counter() - t0 < budget_s * 0.5:
        units += cpu_bitlinear_step()
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": round(units / dt / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{steps} full step(s) of the workload (4 BitLinear layers) on the host cores, {dt:.1f} s"}


# ---------------------------------------------------------------- CPU oracle, every config

def _cpu_rate(fn, units: float, min_s: float = 1.0):
    """Calls fn until min_s has passed (at least twice); returns (units per second, calls, seconds)."""
    fn()  # untimed: warms caches and the OpenMP pool
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_s and n >= 2:
            return units * n / dt, n, dt


def _cpu_affine(case, rows: int, toks: int):
    import oracle
    w = case.weight()[:rows]
    codes, s, b = oracle.affine_quantize(w, case.bits, case.group_size, case.param_dtype)
    x = case.x().vals[:toks]
    lb = case.layer_bias()
    bias = None if lb is None else lb.vals[:rows]
    return (lambda: oracle.affine_matmul(x, codes, s, b, case.bits, case.group_size, bias)), codes, s


def cpu_config_rate(name: str) -> dict:
    """The oracle on a bounded sample of one config, in the config's metric unit."""
    import oracle
    oracle.build()
    kind, arg = CPU_CONFIGS[name]
    if kind == "affine":  # GB/s of weight bytes (codes + scales + biases) in the sample
        case, rows, toks = arg
        fn, codes, s = _cpu_affine(case, rows, toks)
        pbytes = 2 if case.param_dtype == "bf16" else 4
        units, unit = codes.nbytes + 2 * s.size * pbytes, "GB/s"
        sample = f"{rows} of {case.N} output rows, {toks} of {case.M} tokens, K = {case.K}"
    elif kind == "prefill":  # TFLOP/s
        case, rows, toks = arg
        fn, _, _ = _cpu_affine(case, rows, toks)
        units, unit = 2.0 * rows * toks * case.K, "TFLOP/s"
        sample = f"{toks} of {case.M} tokens x {rows} of {case.N} output rows, K = {case.K}"
    elif kind == "bitlinear":
        rows = arg
        cases = synth.BITLINEAR_DECODE
        P = cases[0].packed()[:rows]
        xs = [c.x().vals for c in cases]

        def fn():
            for c, x in zip(cases, xs):
                oracle.bitlinear(x, P, 4 * rows, c.weight_scale, c.invert)
        units, unit = 4.0 * P.nbytes, "GB/s"
        sample = f"packed rows 0..{rows - 1} of 1024 ({4 * rows} of 4096 outputs) of each of the 4 layers"
    else:  # "w8a8" / "w4a8": (case, rows, toks)
        case, rows, toks = arg
        w = case.weight()
        x = case.x().vals[:toks]
        if kind == "w8a8":
            qw, sw = oracle.quantize_int8_rows(w[:rows])
            fn = lambda: oracle.w8a8_linear(x, qw, sw)  # noqa: E731
            wbytes = qw.nbytes + sw.nbytes
        else:
            P, sw = oracle.pack_int4_cols(np.ascontiguousarray(w[:rows].T))
            fn = lambda: oracle.w4a8_linear(x, P, sw)  # noqa: E731
            wbytes = P.nbytes + sw.nbytes
        if case.M <= 16:
            units, unit = float(wbytes), "GB/s"
        else:
            units, unit = 2.0 * rows * toks * case.K, "TFLOP/s"
        sample = f"{toks} of {case.M} tokens x {rows} of {case.N} outputs, K = {case.K}"
    rate, n, dt = _cpu_rate(fn, units)
    scale = 1e9 if unit == "GB/s" else 1e12
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"config": name, "value": rate / scale, "unit": unit, "cores": threads,
            "sample": f"{sample}; {n} calls in {dt:.2f} s"}


def _cpu_configs():
    d = synth.AFFINE_DECODE
    il = synth.INT_LINEAR
    return {
        "cfg1_affine_b4_g64_M4_K512_N512_f32": ("affine", (synth.AFFINE_SMALL, 512, 4)),
        "cfg2_bitlinear_decode_K4096_N4096": ("bitlinear", 64),
        **{f"cfg3_{c.name}": ("affine", (c, 128, c.M)) for c in d},
        "cfg4_affine_prefill_M2048_K4096_N14336": ("prefill", (synth.AFFINE_PREFILL, 64, 64)),
        **{f"cfg5_w8a8_{c.name}": ("w8a8", (c, 256 if c.M == 1 else 64, min(c.M, 32))) for c in il},
        **{f"cfg5_w4a8_{c.name}": ("w4a8", (c, 256 if c.M == 1 else 64, min(c.M, 32))) for c in il},
    }


CPU_CONFIGS = _cpu_configs()


def cpu_table() -> dict:
    """Every config's oracle sample on 1 thread and on all host cores (child processes, so each
    OpenMP runtime starts with its own thread count)."""
    allc = os.cpu_count() or 1
    rows = []
    for name in CPU_CONFIGS:
        row = {"config": name}
        for tag, threads in (("one", 1), ("all", allc)):
            env = dict(os.environ, OMP_NUM_THREADS=str(threads))
            r = subprocess.run([sys.executable, os.path.abspath(__file__), "--cpu-config", name], env=env,
                               capture_output=True, text=True, timeout=600)
            d = json.loads(r.stdout.strip().splitlines()[-1])
            row[tag] = round(d["value"], 4)
            row["unit"] = d["unit"]
            row["sample"] = d["sample"]
        row["cores_all"] = allc
        rows.append(row)
    return {"cpu_table": rows, "cores": allc}


# ---------------------------------------------------------------- suite

def _entry(name, t, units, unit, bound, peak, note=None):
    """Suite line from time_windows() stats `t` (ms per call): value and frac from the median window,
    the spread as the windows' fastest and slowest."""
    scale = 1e9 if unit == "GB/s" else 1e12
    us = t["median"] * 1e3
    val = units / (us * 1e-6) / scale
    e = {"case": name, "us": round(us, 3), "us_min": round(t["min"] * 1e3, 3), "us_max": round(t["max"] * 1e3, 3),
         "windows": t["windows"], "value": round(val, 1), "unit": unit, "bound": bound,
         "frac": round(val / peak, 4), "peak": peak}
    if note:
        e["note"] = note
    return e


def suite(l2: int, peaks: dict, int8_peak: float):
    from bit_quantized_linear_qmm_b200 import qlin as ql
    hbm = float(peaks["hbm_gbs"])
    bf16 = float(peaks["bf16_tflops"])
    out = []
    dev = "cuda"
    tw = time_windows

    # --- MLX-affine layer, small (fp32)
    c = synth.AFFINE_SMALL
    w = torch.from_numpy(c.weight()).to(dev)
    codes, s, b = ql.quantize(w, 4, 64, torch.float32)
    x = c.x().torch(dev)
    bias = c.layer_bias().torch(dev)
    y = torch.empty((c.M, c.N), dtype=torch.float32, device=dev)
    wb = codes.numel() * 4 + s.numel() * 8
    t = tw(lambda i: ql.matmul(x, codes, s, b, 4, 64, bias, out=y), 200, 5)
    out.append(_entry(c.name, t, wb, "GB/s", "hbm", hbm, "launch-bound (0.16 MB)"))

    # --- BitLinear decode, each case alone
    P = torch.from_numpy(synth.BITLINEAR_DECODE[0].packed()).to(dev)
    pool = [P.clone() for _ in range(_copies(P.numel(), l2, 8))]
    ws = torch.tensor([0.5], device=dev)
    for c in synth.BITLINEAR_DECODE:
        x = c.x().torch(dev)
        y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        t = tw(lambda i: ql.bitlinear_matmul(x, pool[i % len(pool)], c.N, ws, c.invert, out=y), 400, 5)
        out.append(_entry(c.name, t, P.numel(), "GB/s", "hbm", hbm))
    del pool

    # --- BitLinear prefill (tcgen05 bf16, exact ternary operands), M = 2048, K = N = 4096
    x = synth.activations(11, (2048, 4096), "bf16").torch(dev)
    y = torch.empty((2048, 4096), dtype=torch.bfloat16, device=dev)
    t = tw(lambda i: ql.bitlinear_matmul(x, P, 4096, ws, False, out=y), 20, 3)
    out.append(_entry("bitlinear_prefill_M2048_K4096_N4096", t, 2.0 * 2048 * 4096 * 4096, "TFLOP/s", "tensor",
                      bf16, "bf16 tcgen05 with exact {-1, 0, 1} operands; inputs L2-resident (x 16.8 MB, W 4.2 MB)"))
    del x, y, P

    # --- MLX-affine decode
    for c in synth.AFFINE_DECODE:
        wd = torch.from_numpy(c.weight()).to(dev)
        codes, s, b = ql.quantize(wd, c.bits, c.group_size, torch.bfloat16)
        del wd
        wb = codes.numel() * 4 + s.numel() * 2 + b.numel() * 2
        pool = [(codes.clone(), s.clone(), b.clone()) for _ in range(_copies(wb, l2, 8))]
        x = c.x().torch(dev)
        bias = c.layer_bias().torch(dev)
        y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)

        def st(i, pool=pool, x=x, bias=bias, y=y, c=c):
            cc, ss, bb = pool[i % len(pool)]
            ql.matmul(x, cc, ss, bb, c.bits, c.group_size, bias, out=y)
        t = tw(st, 200, 5)
        out.append(_entry(c.name, t, wb, "GB/s", "hbm", hbm))
        del pool
        torch.cuda.empty_cache()

    # --- MLX-affine decode, general kernel (3-bit codes straddling words; fp16 x)
    for bits, xd in ((3, "bf16"), (5, "f16")):
        c = synth.AffineCase(f"affine_b{bits}_g64_M1_K4096_N4096_{xd}_general", 1, 4096, 4096, bits, 64, xd, "bf16",
                             True, seed=5)
        wd = torch.from_numpy(c.weight()).to(dev)
        codes, s, b = ql.quantize(wd, bits, 64, torch.bfloat16)
        del wd
        wb = codes.numel() * 4 + s.numel() * 2 + b.numel() * 2
        pool = [(codes.clone(), s.clone(), b.clone()) for _ in range(_copies(wb, l2, 8))]
        x = c.x().torch(dev)
        bias = c.layer_bias().torch(dev)
        y = torch.empty((1, 4096), dtype=x.dtype, device=dev)

        def sg(i, pool=pool, x=x, bias=bias, y=y, bits=bits):
            cc, ss, bb = pool[i % len(pool)]
            ql.matmul(x, cc, ss, bb, bits, 64, bias, out=y)
        t = tw(sg, 200, 5)
        out.append(_entry(c.name, t, wb, "GB/s", "hbm", hbm, "general decode kernel (any width / dtype)"))
        del pool
        torch.cuda.empty_cache()

    # --- MLX-affine prefill (tcgen05, fp16 operands)
    c = synth.AFFINE_PREFILL
    wd = torch.from_numpy(c.weight()).to(dev)
    codes, s, b = ql.quantize(wd, 4, 64, torch.bfloat16)
    t = tw(lambda i: ql.quantize(wd, 4, 64, torch.bfloat16), 10, 2)
    qbytes = wd.numel() * 4 + codes.numel() * 4 + s.numel() * 4
    out.append(_entry("quantize_f32_b4_g64_N14336_K4096", t, qbytes, "GB/s", "hbm", hbm,
                      "reads fp32 W, writes codes + bf16 params"))
    wdq = torch.empty((c.N, c.K), dtype=torch.bfloat16, device=dev)
    t = tw(lambda i: ql.dequantize(codes, s, b, c.K, 4, 64, torch.bfloat16), 10, 2)
    dbytes = codes.numel() * 4 + s.numel() * 4 + wdq.numel() * 2
    out.append(_entry("dequantize_b4_g64_N14336_K4096_bf16", t, dbytes, "GB/s", "hbm", hbm))
    del wd, wdq
    x = c.x().torch(dev)
    bias = c.layer_bias().torch(dev)
    y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
    pool = [(codes.clone(), s.clone(), b.clone()) for _ in range(3)]
    wsp = torch.empty(ql.workspace_size(ql.QLIN_OP_MATMUL, c.M, c.N, c.K, 4, 64), dtype=torch.uint8, device=dev)

    def stp(i):
        cc, ss, bb = pool[i % 3]
        ql.matmul(x, cc, ss, bb, 4, 64, bias, out=y, workspace=wsp)
    t = tw(stp, 20, 3)
    flops = 2.0 * c.M * c.N * c.K
    out.append(_entry(c.name, t, flops, "TFLOP/s", "tensor", bf16,
                      "fp16 operands (x 2^-E, fp16(s q + b)), fp32 accumulate in TMEM; includes the prep kernel"))
    del pool, x, y, wsp
    torch.cuda.empty_cache()

    # --- per-group INT8 (K = N = 4096, group 128): M = 1 FP-activation branch, M = 2048 act-quant branch
    wf = torch.from_numpy(synth.normal(61, (4096, 4096), 0.02)).to(dev)
    qg, sg_ = ql.quantize_int8_groups(wf, 128)
    t = tw(lambda i: ql.quantize_int8_groups(wf, 128), 10, 2)
    out.append(_entry("quantize_int8_groups_N4096_K4096_g128", t, wf.numel() * 5 + sg_.numel() * 4, "GB/s", "hbm",
                      hbm, "reads fp32 W, writes int8 + scales"))
    t = tw(lambda i: ql.quantize_weight_int8(wf, 99.9), 5, 2)
    out.append(_entry("quantize_weight_int8_clip99.9_4096x4096", t, wf.numel() * 5 + 4096 * 4, "GB/s", "hbm", hbm,
                      "per-row percentile: an 11-bit histogram and a counted bin (radix select for dense bins) per row in shared memory"))
    del wf
    pgb = qg.numel() + sg_.numel() * 4
    pool = [(qg.clone(), sg_.clone()) for _ in range(_copies(pgb, l2, 4))]
    for M in (1, 2048):
        x = synth.activations(62, (M, 4096), "bf16").torch(dev)
        y = torch.empty((M, 4096), dtype=torch.bfloat16, device=dev)
        wsz = torch.empty(ql.workspace_size(ql.QLIN_OP_PERGROUP, M, 4096, 4096, 8, 128), dtype=torch.uint8, device=dev)

        def spg(i, x=x, y=y, wsz=wsz):
            qq, ss = pool[i % len(pool)]
            ql.pergroup_linear(x, qq, ss, 128, out=y, workspace=wsz)
        t = tw(spg, 100 if M == 1 else 20, 3)
        if M == 1:
            out.append(_entry("pergroup_M1_K4096_N4096_g128", t, pgb, "GB/s", "hbm", hbm,
                              "fp activation; the resident-weight decode kernel (int8 c as the code c ^ 0x80)"))
        else:
            out.append(_entry("pergroup_M2048_K4096_N4096_g128", t, 2.0 * M * 4096 * 4096, "TFLOP/s", "tensor", bf16,
                              "fp16 operands (int8 x, fp16(s w)); includes act quant + prep"))
        del x, y, wsz
    del pool
    torch.cuda.empty_cache()

    # --- W8A8 / W4A8, K = N = 8192, M in {1, 256, 4096}; weights rotate over copies > 2 x L2
    base = synth.INT_LINEAR[0]
    wf = torch.from_numpy(base.weight()).to(dev)
    qw, sw = ql.quantize_int8_rows(wf)
    P4, s4 = ql.pack_int4_cols(wf.t().contiguous())
    del wf
    n8, n4 = _copies(qw.numel(), l2), _copies(P4.numel(), l2)
    p8 = [qw.clone() for _ in range(n8)]
    p4 = [P4.clone() for _ in range(n4)]
    for c in synth.INT_LINEAR:
        x = c.x().torch(dev)
        y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        wsz = ql.workspace_size(ql.QLIN_OP_W8A8, c.M, c.N, c.K)
        ws_ = torch.empty(wsz, dtype=torch.uint8, device=dev)
        for name, fn, wbytes, ncp in (
                ("w8a8", lambda i: ql.w8a8_linear(x, p8[i % n8], sw, out=y, workspace=ws_), qw.numel() + 4 * c.N, n8),
                ("w4a8", lambda i: ql.w4a8_linear(x, p4[i % n4], s4, out=y, workspace=ws_), P4.numel() + 4 * c.N, n4)):
            t = tw(fn, 50 if c.M < 4096 else 10, 3)
            rot = f"weights rotate over {ncp} copies ({ncp * wbytes / 1e6:.0f} MB)"
            if c.M <= 16:
                out.append(_entry(f"{name}_{c.name}", t, wbytes, "GB/s", "hbm", hbm,
                                  f"includes the activation-quant kernel; {rot}"))
            else:
                ops = 2.0 * c.M * c.N * c.K
                roof = min(int8_peak, hbm * 1e9 * ops / (wbytes + c.M * c.K * 3 + c.M * c.N * 2) / 1e12)
                out.append(_entry(f"{name}_{c.name}", t, ops, "TFLOP/s", "tensor", round(roof, 1),
                                  f"TOPS; includes the activation-quant kernel; peak = min(int8 peak, BW x AI); {rot}"))
        # activation quantiser alone at this M
        if c.M == 4096:
            t = tw(lambda i: ql.quantize_int8_rows(x), 10, 3)
            out.append(_entry("act_quant_M4096_K8192", t, c.M * c.K * 3 + c.M * 4, "GB/s", "hbm", hbm))
        del ws_, x, y
        torch.cuda.empty_cache()
    del p8, p4

    # --- raw int8 GEMM 4096 x 8192 x 8192
    a8 = torch.randint(-128, 128, (4096, 8192), dtype=torch.int8, device=dev)
    b8 = torch.randint(-128, 128, (8192, 8192), dtype=torch.int8, device=dev)
    c32 = torch.empty((4096, 8192), dtype=torch.int32, device=dev)
    t = tw(lambda i: ql.int8_matmul_int32(a8, b8, out=c32), 10, 3)
    out.append(_entry("int8_matmul_int32_M4096_N8192_K8192", t, 2.0 * 4096 * 8192 * 8192, "TFLOP/s", "tensor",
                      int8_peak, "TOPS"))
    return out


def measure_int8_peak():
    """torch._int_mm (cuBLASLt) int8 8192^3, best of 10: context for the int8 denominators."""
    try:
        a = torch.randint(-128, 128, (8192, 8192), dtype=torch.int8, device="cuda")
        b = torch.randint(-128, 128, (8192, 8192), dtype=torch.int8, device="cuda").t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = 1e9
        for _ in range(10):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return 2.0 * 8192 ** 3 / (best * 1e-3) / 1e12
    except Exception:  # noqa: BLE001 - context only
        return None


# ---------------------------------------------------------------- profiling entry (for ncu)

def _prof_bitlinear(M):
    from bit_quantized_linear_qmm_b200 import qlin as ql
    c = synth.BitLinearCase("p", M, 4096, 4096)
    P = torch.from_numpy(c.packed()).cuda()
    x = c.x().torch("cuda")
    ws = torch.tensor([0.5], device="cuda")
    return lambda: ql.bitlinear_matmul(x, P, 4096, ws, False)


def _prof_affine(M, K, N):
    from bit_quantized_linear_qmm_b200 import qlin as ql
    c = synth.AffineCase("p", M, K, N, 4, 128 if M <= 16 else 64, "bf16", "bf16", True,
                         outliers=M > 16)
    codes, s, b = ql.quantize(torch.from_numpy(c.weight()).cuda(), 4, c.group_size, torch.bfloat16)
    x = c.x().torch("cuda")
    bias = c.layer_bias().torch("cuda")
    return lambda: ql.matmul(x, codes, s, b, 4, c.group_size, bias)


def _prof_int(kind, M):
    from bit_quantized_linear_qmm_b200 import qlin as ql
    c = synth.IntCase("p", M, 8192, 8192)
    wf = torch.from_numpy(c.weight()).cuda()
    x = c.x().torch("cuda")
    if kind == "w8a8":
        qw, sw = ql.quantize_int8_rows(wf)
        return lambda: ql.w8a8_linear(x, qw, sw)
    P, s4 = ql.pack_int4_cols(wf.t().contiguous())
    return lambda: ql.w4a8_linear(x, P, s4)


def _prof_affine_b8():
    from bit_quantized_linear_qmm_b200 import qlin as ql
    c = synth.AffineCase("p", 1, 4096, 4096, 8, 64, "bf16", "bf16", True)
    codes, s, b = ql.quantize(torch.from_numpy(c.weight()).cuda(), 8, 64, torch.bfloat16)
    x = c.x().torch("cuda")
    bias = c.layer_bias().torch("cuda")
    return lambda: ql.matmul(x, codes, s, b, 8, 64, bias)


def _prof_quantize():
    from bit_quantized_linear_qmm_b200 import qlin as ql
    w = torch.from_numpy(synth.AFFINE_PREFILL.weight()).cuda()
    return lambda: ql.quantize(w, 4, 64, torch.bfloat16)


def _prof_quantize_bf16():
    from bit_quantized_linear_qmm_b200 import qlin as ql
    w = torch.from_numpy(synth.AFFINE_PREFILL.weight()).cuda().to(torch.bfloat16)
    return lambda: ql.quantize(w, 4, 64, torch.bfloat16)


def _prof_dequantize():
    from bit_quantized_linear_qmm_b200 import qlin as ql
    c = synth.AFFINE_PREFILL
    codes, s, b = ql.quantize(torch.from_numpy(c.weight()).cuda(), 4, 64, torch.bfloat16)
    return lambda: ql.dequantize(codes, s, b, c.K, 4, 64, torch.bfloat16)


def _prof_clip():
    from bit_quantized_linear_qmm_b200 import qlin as ql
    w = torch.from_numpy(synth.normal(61, (4096, 4096), 0.02)).cuda()
    return lambda: ql.quantize_weight_int8(w, 99.9)


def _prof_int8_groups():
    from bit_quantized_linear_qmm_b200 import qlin as ql
    w = torch.from_numpy(synth.normal(61, (4096, 4096), 0.02)).cuda()
    return lambda: ql.quantize_int8_groups(w, 128)


def _prof_act_quant(M=None):
    from bit_quantized_linear_qmm_b200 import qlin as ql
    x = synth.INT_LINEAR[2].x().torch("cuda") if M is None else synth.activations(5, (M, 8192), "bf16").torch("cuda")
    return lambda: ql.quantize_int8_rows(x)


def _prof_bitlinear_prefill():
    from bit_quantized_linear_qmm_b200 import qlin as ql
    P = torch.from_numpy(synth.BITLINEAR_DECODE[0].packed()).cuda()
    x = synth.activations(11, (2048, 4096), "bf16").torch("cuda")
    ws = torch.tensor([0.5], device="cuda")
    return lambda: ql.bitlinear_matmul(x, P, 4096, ws, False)


def _prof_pergroup(M):
    from bit_quantized_linear_qmm_b200 import qlin as ql
    q, s = ql.quantize_int8_groups(torch.from_numpy(synth.normal(61, (4096, 4096), 0.02)).cuda(), 128)
    x = synth.activations(62, (M, 4096), "bf16").torch("cuda")
    return lambda: ql.pergroup_linear(x, q, s, 128)


PROFILE_CASES = {
    "affine_decode_m1_b8": _prof_affine_b8,
    "affine_quantize_n14336": _prof_quantize,
    "act_quant_m4096": _prof_act_quant,
    "act_quant_m256": lambda: _prof_act_quant(256),
    "affine_quantize_bf16_n14336": _prof_quantize_bf16,
    "dequantize_n14336": _prof_dequantize,
    "clip_4096": _prof_clip,
    "int8_groups_4096": _prof_int8_groups,
    "bitlinear_prefill_m2048": _prof_bitlinear_prefill,
    "pergroup_m2048": lambda: _prof_pergroup(2048),
    "pergroup_m1": lambda: _prof_pergroup(1),
    "bitlinear_m1": lambda: _prof_bitlinear(1),
    "bitlinear_m8": lambda: _prof_bitlinear(8),
    "affine_decode_m1": lambda: _prof_affine(1, 4096, 4096),
    "affine_decode_m1_k11008": lambda: _prof_affine(1, 11008, 4096),
    "affine_prefill_m512": lambda: _prof_affine(512, 4096, 14336),
    "affine_prefill_m2048": lambda: _prof_affine(2048, 4096, 14336),
    "w8a8_m4096": lambda: _prof_int("w8a8", 4096),
    "w4a8_m4096": lambda: _prof_int("w4a8", 4096),
    "w8a8_m1": lambda: _prof_int("w8a8", 1),
    "w4a8_m1": lambda: _prof_int("w4a8", 1),
    "w8a8_m256": lambda: _prof_int("w8a8", 256),
    "w4a8_m256": lambda: _prof_int("w4a8", 256),
    "w8a8_m384": lambda: _prof_int("w8a8", 384),  # 256 x 112 tiles of two token sub-tiles
    "w4a8_m384": lambda: _prof_int("w4a8", 384),
}


def profile_case(name):
    fn = PROFILE_CASES[name]()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for i in range(4):
        flush.fill_(i)  # cold L2 for each launch
        fn()
    torch.cuda.synchronize()


# ---------------------------------------------------------------- main

def max_over_ranks(x: float, dist=None, device: str = "cuda") -> float:
    """The largest of every rank's x (the job's time is its slowest rank's); x itself on one rank."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_step: float, ms_per_step: float, scale: float = 1e9) -> float:
    """Units all ranks processed per second (each rank runs its own copy of the step)."""
    return world * units_per_step / (ms_per_step * 1e-3) / scale


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="qlin", choices=["qlin", "reference"])
    ap.add_argument("--no-suite", action="store_true")
    ap.add_argument("--profile", default=None, choices=sorted(PROFILE_CASES),
                    help="run a few launches of one case (for ncu), print nothing else")
    ap.add_argument("--cpu-table", action="store_true",
                    help="time the CPU oracle on a sample of every config, 1 thread and all cores (no GPU)")
    ap.add_argument("--cpu-config", default=None, choices=sorted(CPU_CONFIGS), help=argparse.SUPPRESS)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.profile:
        return profile_case(args.profile)
    if args.cpu_config:
        return print(json.dumps(cpu_config_rate(args.cpu_config)), flush=True)
    if args.cpu_table:
        return print(json.dumps(cpu_table()), flush=True)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return main_reference(args, world, rank)

    from bit_quantized_linear_qmm_b200 import build
    if not os.path.exists(os.path.join(ROOT, "bit_quantized_linear_qmm_b200", "libqlin.so")):
        if rank == 0:
            build.build()
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if dist is not None:
            dist.barrier()

    peaks = load_peaks()
    l2 = torch.cuda.get_device_properties(local_rank).L2_cache_size
    wl = BitlinearDecode(l2)

    sampler = ClockSampler(local_rank)
    sampler.start()
    tm = time_windows(wl.step, args.steps, args.warmup, soak_s=1.0, barrier=barrier)
    ms = tm["ms"]
    clocks = sampler.stop()

    ms_max = max_over_ranks(ms, dist)
    value = whole_job_rate(world, wl.units_per_step, ms_max)

    # roofline of the dominant kernel: algorithmic bytes per launch / average launch duration
    launch_s = ms_max * 1e-3 / wl.launches_per_step
    achieved = wl.alg_bytes_per_launch / launch_s / 1e9
    peak = float(peaks["hbm_gbs"])
    roofline = {"bound": wl.bound, "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": recorded_traffic(wl.key),
                "kernel": wl.key, "peak_source": f"{peaks['source']} hbm_gbs (of {peaks['source']})"}

    wl.e2e_prepare()
    ms_e2e = time_windows(wl.e2e_step, max(1, min(args.steps, 1000)), args.warmup, barrier=barrier)["ms"]
    e2e_value = whole_job_rate(world, wl.units_per_step, max_over_ranks(ms_e2e, dist))

    suite_out = None
    int8_meas = None
    if not args.no_suite:
        int8_meas = measure_int8_peak()
        int8_peak = round(float(peaks["bf16_tflops"]) * INT8_OVER_BF16, 1)
        suite_out = suite(l2, peaks, int8_peak)

    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline()

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": wl.unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": wl.config,
        "roofline": roofline, "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 1), "unit": wl.unit, "h2d_bytes_per_step": wl.h2d,
                "d2h_bytes_per_step": wl.d2h},
        "clocks": clocks, "gpu_launches": wl.launches_per_step * args.steps,
        "ms_per_step_windows": {"median": round(tm["median"], 6), "min": round(tm["min"], 6),
                                "max": round(tm["max"], 6), "windows": tm["windows"],
                                "note": "rank 0's K steps split into back-to-back graph replays"},
    }
    if suite_out is not None:
        line["suite"] = suite_out
        line["int8_peak_tops"] = {"used": round(float(peaks["bf16_tflops"]) * INT8_OVER_BF16, 1),
                                  "rule": "measured bf16 burst x nominal int8/bf16 ratio 2",
                                  "torch_int_mm_8192_measured": None if int8_meas is None else round(int8_meas, 1)}
    print(json.dumps(line), flush=True)


REFERENCE_BUDGET_S = 60.0  # the reference arm's warm-up + timed steps together


def main_reference(args, world, rank):
    """The oracle (CPU) on the headline workload and metric, on the host cores: exactly W untimed
    and K timed steps, each step the first `rows` packed rows of each of the workload's 4 layers,
    with `rows` sized so that the W + K steps take about REFERENCE_BUDGET_S."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    cases = synth.BITLINEAR_DECODE
    P = cases[0].packed()
    xs = [c.x().vals for c in cases]

    def step(rows: int) -> int:
        done = 0
        for c, x in zip(cases, xs):
            oracle.bitlinear(x, P[:rows], 4 * rows, c.weight_scale, c.invert)
            done += rows * c.K
        return done

    t0 = time.perf_counter()
    step(P.shape[0])  # calibration (untimed): one full step; also warms the OpenMP pool
    t_full = time.perf_counter() - t0
    budget = REFERENCE_BUDGET_S / (args.steps + args.warmup)
    rows = P.shape[0] if t_full <= budget else max(8, int(P.shape[0] * budget / t_full) // 8 * 8)
    for _ in range(args.warmup):
        step(rows)
    t0 = time.perf_counter()
    units = 0
    for _ in range(args.steps):
        units += step(rows)
    dt = time.perf_counter() - t0
    value = units / dt / 1e9
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = (f"each step: packed rows 0..{rows - 1} ({rows} of {P.shape[0]}, {4 * rows} of {cases[0].N} outputs) "
              f"of each of the workload's 4 BitLinear layers; {args.warmup} + {args.steps} steps in "
              f"{dt * (1 + args.warmup / args.steps):.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "bitlinear ternary decode GEMV (the CUDA arm's workload), CPU oracle",
                   "rows_per_layer_per_step": rows},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
