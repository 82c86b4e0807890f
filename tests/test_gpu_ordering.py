"""The stream-ordering rule of the C ABI (include/qlin.h, "Ordering on a stream"): a call
fetches its packed weights before waiting for its predecessors, so weights written by an
earlier call of the same run of GEMV / GEMM calls need an ordinary operation in between.

Three chained BitLinear calls: call 1 writes y1, whose bytes call 3 then reads directly as its
packed weights; call 2 is an unrelated layer; an ordinary stream operation (an unrelated
torch kernel, or a device copy) sits between call 1 and call 2 and ends the run.  Call 3 must
see call 1's bytes: checked against the oracle on exactly those bytes.  (The same chain without
the ordinary operation is a race the rule forbids; it is not run.)"""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("between", ["kernel", "copy"])
def test_three_chained_calls_with_ordering_point(orc, between):
    ql = build_lib()
    # call 1: y1 bf16 [8, 2048] = 32 KB, read by call 3 as packed weights uint8 [64, 512]
    c1 = synth.BitLinearCase("call1", 8, 1024, 2048, 0.5, False, seed=31)
    x1, P1 = c1.x().torch("cuda"), to_dev(c1.packed())
    ws = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    y1 = torch.empty((8, 2048), dtype=torch.bfloat16, device="cuda")
    # call 2: an unrelated layer
    c2 = synth.BitLinearCase("call2", 1, 4096, 4096, 0.5, True, seed=32)
    x2, P2 = c2.x().torch("cuda"), to_dev(c2.packed())
    y2 = torch.empty((1, 4096), dtype=torch.bfloat16, device="cuda")
    # call 3: K = 512, N = 256, weights = y1's bytes
    c3 = synth.BitLinearCase("call3", 4, 512, 256, 0.25, False, seed=33)
    x3 = c3.x().torch("cuda")
    y3 = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    ws3 = torch.tensor([0.25], dtype=torch.float32, device="cuda")
    scratch_a = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    scratch_b = torch.empty_like(scratch_a)
    P3 = y1.view(torch.uint8).view(64, 512)
    for rep in range(3):
        y1.view(torch.uint8).fill_(0x55)  # stale bytes: all code 1 (weight 0) -> y3 = 0 if read early
        torch.cuda.synchronize()
        ql.bitlinear_matmul(x1, P1, 2048, ws, False, out=y1)                  # call 1 (starts a run)
        if between == "kernel":
            scratch_a.add_(1)                                                 # ordinary kernel: ends the run
        else:
            scratch_b.copy_(scratch_a)                                        # device copy: ends the run
        ql.bitlinear_matmul(x2, P2, 4096, ws, True, out=y2)                   # call 2
        ql.bitlinear_matmul(x3, P3, 256, ws3, False, out=y3)                  # call 3 reads call 1's bytes
        torch.cuda.synchronize()
        P3_host = P3.cpu().numpy()
        assert not np.all(P3_host == 0x55), rep
        yr, mag = orc.bitlinear(c3.x().vals, P3_host, 256, 0.25, False)
        assert_fp_close(y3, yr, mag, None, f"call3 rep {rep}")
    assert ql.device_status() == ql.QLIN_OK


@pytest.mark.parametrize("M", [16, 256])
@pytest.mark.parametrize("op", ["w8a8", "w4a8"])
def test_int8_linear_chain_shares_workspace(op, M):
    """Three chained int8 linears on one stream, each layer's output the next one's input and one
    workspace for all three: the activation quantiser of a call rewrites the workspace that the
    previous call's GEMM reads, so it must wait for that GEMM (above 16 tokens it is placed early,
    as a programmatic dependent).  The chain run back to back gives the bits of the same calls
    separated by synchronisations."""
    ql = build_lib()
    K = N = 2048
    layers = []
    for l in range(3):
        w = torch.from_numpy(synth.normal(40 + l, (N, K), 1.0 / np.sqrt(K))).cuda()
        layers.append(ql.quantize_int8_rows(w) if op == "w8a8" else ql.pack_int4_cols(w.t().contiguous()))
    f = ql.w8a8_linear if op == "w8a8" else ql.w4a8_linear
    x0 = synth.activations(44, (M, K), "bf16").torch("cuda")
    ws = torch.empty(ql.workspace_size(ql.QLIN_OP_W8A8, M, N, K), dtype=torch.uint8, device="cuda")

    def chain(sync):
        x = x0
        for wq, sw in layers:
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            f(x, wq, sw, out=y, workspace=ws)
            if sync:
                torch.cuda.synchronize()
            x = y
        torch.cuda.synchronize()
        return x

    ref = chain(True)
    assert torch.isfinite(ref.float()).all() and ref.float().abs().max() > 0
    for _ in range(5):
        assert torch.equal(chain(False), ref)
