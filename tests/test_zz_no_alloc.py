"""w8a8_linear_noalloc: the W8A8 layer for callers that cannot give the
library device memory (its scratch is a buffer inside libqlin.so).  Checked
through the C ABI against w8a8_linear (bit-equal) and the oracle (fp bar) on
three calls in a row that cover both kernel paths.  This file is collected
last on purpose."""
import ctypes as C

import numpy as np
import pytest
import torch

import synth
from helpers import REL, ABS, build_lib, half_ulp, to_dev

pytestmark = pytest.mark.gpu


def _call_noalloc(ql, x, w, s, bias, y):
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = ql.lib().w8a8_linear_noalloc(C.c_void_p(x.data_ptr()), ql.QLIN_BF16, x.shape[0], x.shape[1],
                                      C.c_void_p(w.data_ptr()), C.c_void_p(s.data_ptr()), w.shape[0],
                                      None if bias is None else C.c_void_p(bias.data_ptr()),
                                      C.c_void_p(y.data_ptr()), st)
    return rc


def test_noalloc_matches_w8a8_linear_twice(orc):
    """Three calls in a row on the built-in scratch: the tcgen05 GEMM (M = 300), the
    weight-streaming GEMV (M = 8) and the GEMM again with a ragged M.  Each is bit-equal
    to w8a8_linear with a caller workspace (the same deterministic kernels) and within
    the fp bar of the oracle."""
    ql = build_lib()
    N, K = 384, 2048
    w = synth.normal(61, (N, K), 0.02)
    qw, sw = orc.quantize_int8_rows(w)
    wd, sd = to_dev(qw), to_dev(sw)
    lb = synth.activations(62, (N,), "bf16", 0.01)
    bias = lb.torch("cuda")
    for call, (M, seed) in enumerate([(300, 63), (8, 65), (17, 64)]):
        xa = synth.activations(seed, (M, K), "bf16")
        x = xa.torch("cuda")
        ws = torch.empty(ql.workspace_size(ql.QLIN_OP_W8A8, M, N, K), dtype=torch.uint8, device="cuda")
        y_ref = ql.w8a8_linear(x, wd, sd, bias, workspace=ws)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(ql, x, wd, sd, bias, y) == ql.QLIN_OK, f"call {call}"
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), f"call {call} (M = {M}): differs from w8a8_linear"
        yr, mag, _, _ = orc.w8a8_linear(xa.vals, qw, sw, lb.vals)
        yd = y.double().cpu().numpy()
        tol = REL * (mag + np.abs(lb.vals)[None, :]) + ABS + half_ulp(np.maximum(np.abs(yd), np.abs(yr)), y.dtype)
        err = np.abs(yd - yr)
        assert (err <= tol).all(), (call, float((err / tol).max()))
    assert ql.device_status() == ql.QLIN_OK


def test_noalloc_rejects_too_large():
    ql = build_lib()
    M, K, N = 2048, 8192, 16  # qx alone is 16 MiB > the 8 MiB built-in scratch
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    s = torch.ones(N, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(ql, x, w, s, None, y) == ql.QLIN_ERR_WORKSPACE
