#!/usr/bin/env python
"""Throughput benchmark of the quantized linear layers on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qlin|reference]
                    [--workload NAME] [--no-suite]

One step = one pass of the workload's hot path over one batch of synthetic
input (for the default workload, the four BitLinear ternary decode layers
K = N = 4096, M in {1, 8}, multiply and divide scale modes).  Weights rotate
over device copies whose total exceeds the L2 cache, so every launch streams
its weights from HBM.  The K timed steps run as CUDA-graph replays between
CUDA events on the launching stream, bracketed by a barrier and a device
synchronise; multi-GPU runs take the maximum time over ranks (weak scaling:
every rank runs its own copy of the workload, no collective on the data path).

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


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_linear_qmm_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
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


# ---------------------------------------------------------------- workloads

def _rotation_copies(bytes_per_copy: int, l2_bytes: int, minimum: int = 8) -> int:
    """Copies whose total is at least twice the L2 size."""
    return max(minimum, int(math.ceil(2 * l2_bytes / bytes_per_copy)))


class BitlinearDecode:
    """BitLinear ternary decode GEMV: x bf16 [M, 4096], packed uint8 [1024, 4096],
    M in {1, 8}, weight_scale 0.5, multiply and divide modes; no bias."""
    key = "bitlinear_gemv_kernel"
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
        self.copies = _rotation_copies(self.wbytes, l2_bytes)
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

    # end-to-end: host x in, host y out, every step
    def e2e_prepare(self):
        self.hx = [x.cpu().pin_memory() for x in self.xs]
        self.hy = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in self.ys]
        self.h2d = sum(t.numel() * t.element_size() for t in self.hx)
        self.d2h = sum(t.numel() * t.element_size() for t in self.hy)

    def e2e_step(self, i: int):
        for c in range(len(self.cases)):
            self.xs[c].copy_(self.hx[c], non_blocking=True)
        self.step(i)
        for c in range(len(self.cases)):
            self.hy[c].copy_(self.ys[c], non_blocking=True)

    # the oracle on the host cores
    def cpu_step(self):
        import oracle
        P = self.cases[0].packed()
        done = 0
        for case in self.cases:
            x = case.x().vals
            oracle.bitlinear(x, P, case.N, case.weight_scale, case.invert)
            done += self.wbytes
        return done


class AffineDecodeSuite:
    """Each MLX-affine decode layer of the Llama-7B-shaped set, timed alone."""

    def __init__(self, l2_bytes: int):
        from bit_quantized_linear_qmm_b200 import qlin
        self.ql = qlin
        self.l2 = l2_bytes

    def run(self, steps: int):
        out = []
        for case in synth.AFFINE_DECODE:
            w = case.weight()
            wd = torch.from_numpy(w).cuda()
            codes, s, b = self.ql.quantize(wd, case.bits, case.group_size, torch.bfloat16)
            del wd
            wbytes = codes.numel() * 4 + s.numel() * 2 + b.numel() * 2
            copies = _rotation_copies(wbytes, self.l2)
            pool = [(codes.clone(), s.clone(), b.clone()) for _ in range(copies)]
            x = case.x().torch("cuda")
            bias = case.layer_bias().torch("cuda")
            y = torch.empty((case.M, case.N), dtype=torch.bfloat16, device="cuda")

            def step(i, pool=pool, x=x, bias=bias, y=y, case=case, copies=copies):
                c, sc, bi = pool[i % copies]
                self.ql.matmul(x, c, sc, bi, case.bits, case.group_size, bias, out=y)
            ms = time_steps(step, steps, 5)
            gbs = wbytes / (ms * 1e-3) / 1e9
            out.append({"case": case.name, "weight_bytes": int(wbytes), "us": round(ms * 1e3, 3),
                        "GB/s": round(gbs, 1)})
            del pool
            torch.cuda.empty_cache()
        return out


WORKLOADS = {"bitlinear_decode": BitlinearDecode}


# ---------------------------------------------------------------- timing

def _graphs(step_fn, steps: int, per_graph: int):
    """CUDA graphs holding `steps` steps: (graph of per_graph steps, count, remainder graph)."""
    per_graph = max(1, min(per_graph, steps))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(per_graph):
            step_fn(i)
    rem = steps % per_graph
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem):
            for i in range(rem):
                step_fn(i)
    return g, steps // per_graph, g_rem


def time_steps(step_fn, steps: int, warmup: int, per_graph: int = 200, soak_s: float = 0.0, barrier=None):
    """Milliseconds per step over exactly `steps` steps (graph replays between CUDA events)."""
    for i in range(warmup):
        step_fn(i)
    torch.cuda.synchronize()
    g, reps, g_rem = _graphs(step_fn, steps, per_graph)
    g.replay()  # untimed: first replay uploads the graph
    torch.cuda.synchronize()
    if soak_s > 0:
        t0 = time.time()
        while time.time() - t0 < soak_s:
            g.replay()
            torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(reps):
        g.replay()
    if g_rem is not None:
        g_rem.replay()
    ev1.record()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    ms = ev0.elapsed_time(ev1)
    del g, g_rem
    return ms / steps


# ---------------------------------------------------------------- main

def cpu_baseline(workload, budget_s: float = 12.0):
    import oracle
    oracle.build()
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    t0 = time.perf_counter()
    units = workload.cpu_step()  # one full step at least
    steps = 1
    while time.perf_counter() - t0 < budget_s * 0.5:
        units += workload.cpu_step()
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": round(units / dt / 1e9, 3), "unit": workload.unit, "cores": threads, "kind": "oracle",
            "sample": f"{steps} full step(s) of the workload on the host cores ({dt:.1f} s)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="qlin", choices=["qlin", "reference"])
    ap.add_argument("--workload", default="bitlinear_decode", choices=sorted(WORKLOADS))
    ap.add_argument("--no-suite", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return main_reference(args, world, rank)

    from bit_quantized_linear_qmm_b200 import build
    if rank == 0 and not os.path.exists(os.path.join(ROOT, "bit_quantized_linear_qmm_b200", "libqlin.so")):
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
    wl = WORKLOADS[args.workload](l2)

    sampler = ClockSampler(local_rank)
    sampler.start()
    ms = time_steps(wl.step, args.steps, args.warmup, soak_s=1.0, barrier=barrier)
    clocks = sampler.stop()

    t = torch.tensor([ms], dtype=torch.float64, device="cuda")
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    value = world * wl.units_per_step / (ms_max * 1e-3) / 1e9

    # roofline of the dominant kernel: algorithmic bytes per launch / average launch duration
    launch_s = ms_max * 1e-3 / wl.launches_per_step
    achieved = wl.alg_bytes_per_launch / launch_s / 1e9
    peak = float(peaks["hbm_gbs"])
    roofline = {"bound": wl.bound, "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": recorded_traffic(wl.key),
                "kernel": wl.key, "peak_source": f"{peaks['source']} hbm_gbs"}

    # end to end through the public API: host x in, host y out, every step
    wl.e2e_prepare()
    ms_e2e = time_steps(wl.e2e_step, max(1, min(args.steps, 1000)), args.warmup, barrier=barrier)
    t = torch.tensor([ms_e2e], dtype=torch.float64, device="cuda")
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_value = world * wl.units_per_step / (float(t.item()) * 1e-3) / 1e9

    suite = None
    if not args.no_suite:
        suite = {"affine_decode": AffineDecodeSuite(l2).run(200)}

    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline(wl)

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
    }
    if suite is not None:
        line["suite"] = suite
    print(json.dumps(line), flush=True)


def main_reference(args, world, rank):
    """The oracle (CPU) on the same workload and metric, on the host cores."""
    if rank != 0:
        return
    wl_cls = WORKLOADS[args.workload]
    import oracle
    oracle.build()

    class Host:  # CPU-only view of the workload (no device memory)
        pass
    h = Host()
    cases = synth.BITLINEAR_DECODE
    h.unit = "GB/s"
    h.wbytes = cases[0].N // 4 * cases[0].K
    h.cases = cases
    h.cpu_step = lambda: wl_cls.cpu_step(h)
    for _ in range(args.warmup):
        pass
    t0 = time.perf_counter()
    units = 0
    for _ in range(args.steps if args.steps <= 5 else 5):
        units += h.cpu_step()
    dt = time.perf_counter() - t0
    steps_done = args.steps if args.steps <= 5 else 5
    value = units / dt / 1e9
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": h.unit, "n_gpus": world,
        "steps": steps_done, "warmup": args.warmup, "ms_per_step": round(dt / steps_done * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "bitlinear ternary decode GEMV (same as the CUDA arm), CPU oracle"},
        "cpu_baseline": {"value": round(value, 3), "unit": h.unit, "cores": threads, "kind": "oracle",
                         "sample": f"{steps_done} full steps"},
        "e2e": {"value": round(value, 3), "unit": h.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
