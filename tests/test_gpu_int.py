"""GPU parity of the int8 paths: raw int8 GEMM (bit-exact), W8A8 and W4A8 layers."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    return build_lib()


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (130, 200, 272), (256, 384, 512), (5, 1000, 4096),
                                   (1280, 4096, 256),  # 160 tiles of 128 x 256: the wide tile path
                                   (128, 128, 16), (333, 129, 1040),
                                   # tiles of two 128-token sub-tiles: the second sub-tile partly past M;
                                   # a last M-tile of one sub-tile, ragged N and a part stage of K
                                   (400, 8192, 256), (300, 8000, 160)])
def test_int8_matmul_int32_bit_exact(ql, orc, M, N, K):
    rng = np.random.default_rng(M * 7 + N)
    a = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    b = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    c = ql.int8_matmul_int32(to_dev(a), to_dev(b))
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy(), orc.int8_matmul(a, b))


@pytest.mark.parametrize("op,M,N", [("W8A8", 400, 8192), ("W8A8", 300, 8000)])
def test_two_subtile_cases_take_that_tile(ql, op, M, N):
    """The parity cases above and below that stand for tiles of two 128-token sub-tiles get that
    tile on this device."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert ql.int8_gemm_tile(getattr(ql, "QLIN_OP_" + op), M, N, sms) == (256, 112)


def test_int8_matmul_extremes(ql, orc):
    """All -128 times all -128 over K = 4096 -> 2^26 per element (exact int32)."""
    a = np.full((130, 4096), -128, np.int8)
    b = np.full((140, 4096), -128, np.int8)
    c = ql.int8_matmul_int32(to_dev(a), to_dev(b))
    torch.cuda.synchronize()
    assert np.all(c.cpu().numpy() == 128 * 128 * 4096)


def _w8a8(ql, orc, case, rows=None, bias=False):
    w = case.weight()
    qw, sw = orc.quantize_int8_rows(w)
    x = case.x()
    lb = synth.activations(case.seed + 2, (case.N,), "bf16", 0.01) if bias else None
    y = ql.w8a8_linear(x.torch("cuda"), to_dev(qw), to_dev(sw), None if lb is None else lb.torch("cuda"))
    torch.cuda.synchronize()
    if rows is not None:
        qw, sw = qw[rows], sw[rows]
        y = y[:, torch.as_tensor(rows, device=y.device)]
    bias_v = None if lb is None else (lb.vals if rows is None else lb.vals[rows])
    yr, mag, _, _ = orc.w8a8_linear(x.vals, qw, sw, bias_v)
    return assert_fp_close(y, yr, mag, bias_v, case.name)


def _w4a8(ql, orc, case, cols=None):
    w = case.weight()                       # [N, K]; W4 quantizes its transpose [K, N]
    P, sw = orc.pack_int4_cols(np.ascontiguousarray(w.T))
    x = case.x()
    y = ql.w4a8_linear(x.torch("cuda"), to_dev(P), to_dev(sw))
    torch.cuda.synchronize()
    if cols is not None:
        P, sw = P[:, cols], sw[cols]
        y = y[:, torch.as_tensor(cols, device=y.device)]
    yr, mag, _, _ = orc.w4a8_linear(x.vals, P, sw)
    return assert_fp_close(y, yr, mag, None, case.name)


SMALL = [synth.IntCase(f"M{M}_K{K}_N{N}", M, K, N, seed=M + K) for (M, K, N) in
         [(1, 256, 128), (3, 512, 272), (17, 1024, 384), (200, 768, 144), (256, 4096, 256)]]
# W8A8 decode GEMV edges (W4A8 needs K % 32 == 0 and N % 16 == 0): two token tiles,
# a k32 step half past K, rows past N
SMALL_W8 = SMALL + [synth.IntCase(f"M{M}_K{K}_N{N}", M, K, N, seed=M + K) for (M, K, N) in
                    [(16, 272, 100), (9, 1040, 64), (8, 4096, 520),
                     (1280, 256, 4096),  # the wide (128 x 256) tile path
                     # two 128-token sub-tiles per tile (one weight stage, two accumulators)
                     (400, 256, 8192), (300, 160, 8000)]]


@pytest.mark.parametrize("case", SMALL_W8, ids=[c.name for c in SMALL_W8])
@pytest.mark.parametrize("bias", [False, True])
def test_w8a8_small(ql, orc, case, bias):
    _w8a8(ql, orc, case, bias=bias)


# W4A8 decode GEMV edges: two token tiles with a partial 64-column strip, a partial last stage
SMALL_W4 = SMALL + [synth.IntCase(f"M{M}_K{K}_N{N}", M, K, N, seed=M + K) for (M, K, N) in
                    [(16, 1024, 112), (9, 544, 48), (1, 8192, 80),
                     (1280, 256, 4096)]]  # the wide (128 x 256) tile path


@pytest.mark.parametrize("case", SMALL_W4, ids=[c.name for c in SMALL_W4])
def test_w4a8_small(ql, orc, case):
    _w4a8(ql, orc, case)


@pytest.mark.parametrize("case", synth.INT_LINEAR, ids=[c.name for c in synth.INT_LINEAR])
def test_w8a8_config_sampled(ql, orc, case):
    rng = np.random.default_rng(2)
    rows = np.sort(rng.choice(case.N, size=96, replace=False))
    sub = synth.IntCase(case.name, min(case.M, 256), case.K, case.N, seed=case.seed)
    _w8a8(ql, orc, sub if case.M > 256 else case, rows)


@pytest.mark.parametrize("case", synth.INT_LINEAR, ids=[c.name for c in synth.INT_LINEAR])
def test_w4a8_config_sampled(ql, orc, case):
    rng = np.random.default_rng(3)
    cols = np.sort(rng.choice(case.N, size=96, replace=False))
    sub = synth.IntCase(case.name, min(case.M, 256), case.K, case.N, seed=case.seed)
    _w4a8(ql, orc, sub if case.M > 256 else case, cols)


def test_w8a8_full_m4096_sampled_rows_and_tokens(ql, orc):
    """The M=4096 layer through one call; checked on sampled tokens x sampled features."""
    case = synth.INT_LINEAR[2]
    w = case.weight()
    qw, sw = orc.quantize_int8_rows(w)
    x = case.x()
    y = ql.w8a8_linear(x.torch("cuda"), to_dev(qw), to_dev(sw))
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    toks = np.sort(rng.choice(case.M, size=64, replace=False))
    feats = np.sort(rng.choice(case.N, size=64, replace=False))
    yr, mag, _, _ = orc.w8a8_linear(x.vals[toks], qw[feats], sw[feats])
    ys = y[torch.as_tensor(toks, device="cuda")][:, torch.as_tensor(feats, device="cuda")]
    assert_fp_close(ys, yr, mag, None, "w8a8 M4096 sampled")


def test_w4a8_full_m4096_sampled_cols_and_tokens(ql, orc):
    """The W4A8 M=4096 layer (K = N = 8192) through one call -- the tcgen05 GEMM with the nibble
    transform -- checked on sampled tokens x sampled output columns (the last included)."""
    case = synth.INT_LINEAR[2]
    w = case.weight()
    P, sw = orc.pack_int4_cols(np.ascontiguousarray(w.T))
    x = case.x()
    y = ql.w4a8_linear(x.torch("cuda"), to_dev(P), to_dev(sw))
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    toks = np.sort(rng.choice(case.M, size=64, replace=False))
    cols = np.sort(rng.choice(case.N, size=64, replace=False))
    cols[-1] = case.N - 1
    yr, mag, _, _ = orc.w4a8_linear(x.vals[toks], np.ascontiguousarray(P[:, cols]), sw[cols])
    ys = y[torch.as_tensor(toks, device="cuda")][:, torch.as_tensor(cols, device="cuda")]
    assert_fp_close(ys, yr, mag, None, "w4a8 M4096 sampled")


def test_int_linear_rejects(ql):
    x = torch.zeros((2, 100), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 100), dtype=torch.int8, device="cuda")
    s = torch.ones(16, device="cuda")
    with pytest.raises(ql.QlinError) as e:
        ql.w8a8_linear(x, w, s)   # K % 16 != 0
    assert e.value.status == ql.QLIN_ERR_INVALID_ARG
    with pytest.raises(ql.QlinError) as e:
        ql.w8a8_linear(x[:, :96].contiguous(), w[:, :96].contiguous(), s, workspace=torch.empty(8, dtype=torch.uint8,
                                                                                                device="cuda"))
    assert e.value.status == ql.QLIN_ERR_WORKSPACE
