"""Time breakdown of a decode kernel inside a chain of dependent layers.

    python -m bit_quantized_linear_qmm_b200.trace_decode [--kind bitlinear|affine] [--layers L]
                                                         [--copies C] [--M M] [--K K] [--N N]

Builds the trace variant of the library (libqlin_trace.so: the same sources
compiled with QLIN_TRACE, whose decode kernels record %globaltimer stamps per
CTA), runs L layers back to back in one CUDA graph with the weights rotating
over C device copies (so each layer streams its weights from HBM) and prints,
averaged over the layers:
  bitlinear: BitLinear layers, K = N = 4096, M = 1, 1, 8, 8 repeating, the
             multiply and divide modes alternating;
  affine:    MLX-affine 4-bit group-128 layers (bf16 x and parameters, layer
             bias), M x K -> N (default 1 x 4096 -> 4096), on the resident-weight
             decode kernel; "x+chunk0" is then wait return -> x and weights landed.

  period        graph time / L (the time per layer)
  release       first CTA's griddepcontrol.wait return minus the previous
                layer's last CTA end
  x+chunk0      wait return -> first 64-k chunk done (x arrival + one chunk)
  loop          rest of the main loop
  reduce        CTA reduction, scaling, bias and y stores
  start->wait   CTA start -> its griddepcontrol.wait return (mean over CTAs)
  start->chunk0 CTA start -> first chunk done (affine: codes and x landed)
  critical      last CTA end minus first wait return
  end spread    last CTA end minus first CTA end
  doubled       SMs that ran two CTAs of the same layer (summed over layers)
"""
from __future__ import annotations

import argparse
import ctypes as C
import os
import sys

import numpy as np
import torch

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from bit_quantized_linear_qmm_b200 import build, qlin  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kind", default="bitlinear", choices=["bitlinear", "affine"])
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--copies", type=int, default=64)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=4096)
    args = ap.parse_args()
    path = build.build(trace=True)
    qlin.LIB_PATH = path  # the binding loads the trace build instead of libqlin.so
    L = qlin.lib()
    read = L.qlin_trace_read if args.kind == "bitlinear" else L.qlin_trace_read_dec
    read.argtypes = [C.c_void_p, C.c_size_t]
    read.restype = C.c_int
    ctas_max = int(L.qlin_trace_ctas())

    torch.cuda.set_device(0)
    if args.kind == "bitlinear":
        cases = synth.BITLINEAR_DECODE  # M = 1, 1, 8, 8; multiply / divide
        N = cases[0].N
        packed = torch.from_numpy(cases[0].packed()).cuda()
        pool = [packed.clone() for _ in range(args.copies)]
        xs = [c.x().torch("cuda") for c in cases]
        ys = [torch.empty((c.M, N), dtype=torch.bfloat16, device="cuda") for c in cases]
        ws = torch.tensor([cases[0].weight_scale], dtype=torch.float32, device="cuda")

        def chain():
            for i in range(args.layers):
                c = i % len(cases)
                qlin.bitlinear_matmul(xs[c], pool[i % len(pool)], N, ws, cases[c].invert, out=ys[c])
    else:
        case = synth.AffineCase("trace", args.M, args.K, args.N, 4, 128, "bf16", "bf16", True, seed=3)
        codes, s, b = qlin.quantize(torch.from_numpy(case.weight()).cuda(), 4, 128, torch.bfloat16)
        pool = [(codes.clone(), s.clone(), b.clone()) for _ in range(args.copies)]
        x = case.x().torch("cuda")
        bias = case.layer_bias().torch("cuda")
        y = torch.empty((args.M, args.N), dtype=torch.bfloat16, device="cuda")

        def chain():
            for i in range(args.layers):
                cc, ss, bb = pool[i % len(pool)]
                qlin.matmul(x, cc, ss, bb, 4, 128, bias, out=y)

    chain()  # first calls outside capture
    torch.cuda.synchronize()
    read(None, 0)  # reset the slot counter; the graph's launches take slots 0 .. L-1
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    period_us = e0.elapsed_time(e1) * 1e3 / args.layers

    buf = np.zeros((args.layers, ctas_max, 8), np.uint64)
    used = read(buf.ctypes.data, buf.nbytes)
    assert used == args.layers, (used, args.layers)
    grid = int(np.count_nonzero(buf[0, :, 0]))
    t = buf[:, :grid, :].astype(np.int64)
    rel, x0, loop, red, crit, spread, dbl = [], [], [], [], [], [], 0
    s2w, s2c = [], []
    for i in range(1, args.layers):
        rel.append(t[i, :, 2].min() - t[i - 1, :, 5].max())
        x0.append((t[i, :, 3] - t[i, :, 2]).mean())
        s2w.append((t[i, :, 2] - t[i, :, 0]).mean())
        s2c.append((t[i, :, 3] - t[i, :, 0]).mean())
        loop.append((t[i, :, 4] - t[i, :, 3]).mean())
        red.append((t[i, :, 5] - t[i, :, 4]).mean())
        crit.append(t[i, :, 5].max() - t[i, :, 2].min())
        spread.append(t[i, :, 5].max() - t[i, :, 5].min())
        sm = t[i, :, 7]
        dbl += int(np.sum(np.bincount(sm) > 1))
    out = {"kind": args.kind, "layers": args.layers, "ctas": grid, "period_us": round(period_us, 3),
           "release_ns": round(float(np.mean(rel))), "x_chunk0_ns": round(float(np.mean(x0))),
           "start_to_wait_ns": round(float(np.mean(s2w))), "start_to_chunk0_ns": round(float(np.mean(s2c))),
           "loop_ns": round(float(np.mean(loop))), "reduce_ns": round(float(np.mean(red))),
           "critical_ns": round(float(np.mean(crit))), "end_spread_ns": round(float(np.mean(spread))),
           "doubled_sms": dbl}
    print(out, flush=True)


if __name__ == "__main__":
    main()
