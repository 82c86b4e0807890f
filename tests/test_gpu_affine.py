"""GPU parity of qlin_matmul (MLX affine format) against the oracle."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, params_dev, u32_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    return build_lib()


def _run_case(ql, orc, case: synth.AffineCase, rows=None):
    """Runs the layer on the GPU; compares all outputs, or the sampled rows `rows`."""
    w = case.weight()
    codes, s, b = orc.affine_quantize(w, case.bits, case.group_size, case.param_dtype == "bf16")
    x = case.x()
    lb = case.layer_bias()
    y = ql.matmul(x.torch("cuda"), u32_dev(codes), params_dev(s, case.param_dtype),
                  params_dev(b, case.param_dtype), case.bits, case.group_size,
                  None if lb is None else lb.torch("cuda"))
    torch.cuda.synchronize()
    assert y.dtype == (torch.bfloat16 if case.x_dtype == "bf16" else torch.float32)
    if rows is not None:
        codes, s, b = codes[rows], s[rows], b[rows]
        y = y[:, torch.as_tensor(rows, device=y.device)]
    bias_v = None if lb is None else lb.vals if rows is None else lb.vals[rows]
    yr, mag = orc.affine_matmul(x.vals, codes, s, b, case.bits, case.group_size, bias_v)
    return assert_fp_close(y, yr, mag, bias_v, case.name)


SMALL = [
    synth.AffineCase(f"b{b}_g{g}_M{M}_{xd}_{pd}{'_bias' if bias else ''}", M, K, 197, b, g, xd, pd, bias, seed=7)
    for (b, g, K) in [(4, 32, 640), (4, 64, 640), (4, 128, 1280), (2, 64, 768), (2, 128, 1280),
                      (8, 32, 544), (8, 64, 640), (8, 128, 1280)]
    for M in (1, 3, 8, 9, 16)
    for (xd, pd, bias) in [("bf16", "bf16", True), ("f32", "f32", False)]
]


@pytest.mark.parametrize("case", SMALL, ids=[c.name for c in SMALL])
def test_affine_small_shapes(ql, orc, case):
    _run_case(ql, orc, case)


def test_affine_small_layer_full(ql, orc):
    """The 4-bit g64 fp32 layer x[4,512] . W[512,512]^T + bias, every output."""
    _run_case(ql, orc, synth.AFFINE_SMALL)


@pytest.mark.parametrize("case", synth.AFFINE_DECODE, ids=[c.name for c in synth.AFFINE_DECODE])
def test_affine_decode_configs_sampled(ql, orc, case):
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(case.N, size=256, replace=False))
    rows[-1] = case.N - 1
    _run_case(ql, orc, case, rows)


def test_affine_m_above_16(ql, orc):
    case = synth.AffineCase("b4_g64_M40", 40, 512, 130, 4, 64, "bf16", "bf16", True, seed=3)
    _run_case(ql, orc, case)


# M > 16 outside the tensor-core prefill (2- and 8-bit codes, fp32 group parameters): the decode
# kernel over 16-token slices
SLICED = [synth.AffineCase(f"sliced_b{b}_g{g}_M{M}_{xd}_{pd}", M, K, N, b, g, xd, pd, True, seed=23)
          for (M, K, N, b, g, xd, pd) in [(17, 512, 200, 2, 64, "bf16", "bf16"), (40, 1024, 130, 8, 64, "bf16", "bf16"),
                                          (33, 640, 96, 4, 32, "bf16", "f32"), (20, 512, 64, 4, 128, "f32", "f32"),
                                          (48, 768, 72, 8, 128, "f32", "bf16")]]


@pytest.mark.parametrize("case", SLICED, ids=[c.name for c in SLICED])
def test_affine_m_above_16_sliced(ql, orc, case):
    _run_case(ql, orc, case)


# the resident-weight decode kernel (bf16 x, M <= 8, every code block in shared memory, one CTA
# per SM, at most two 16-row tiles per CTA): N = 1000 -> 63 CTAs of 15-16 rows, 2400 -> 148 of
# 16-17, 4096 -> 27-28, 4736 -> exactly 32 (no spare row); K / g even; M = 1 (token-0 epilogue)
# and M = 5, 8 (the general one)
RESIDENT = [synth.AffineCase(f"resident_b{b}_g{g}_M{M}_K{K}_N{N}_{pd}", M, K, N, b, g, "bf16", pd, bias, seed=b + M + N)
            for (b, g, K, N) in [(4, 128, 1024, 4096), (4, 64, 512, 4736), (4, 32, 256, 2400), (2, 64, 768, 4096),
                                 (2, 128, 512, 1000), (8, 64, 512, 4096), (8, 128, 256, 4736), (8, 32, 384, 2400)]
            for M in (1, 5, 8)
            for (pd, bias) in [("bf16", True), ("f32", False)]]


@pytest.mark.parametrize("case", RESIDENT, ids=[c.name for c in RESIDENT])
def test_affine_resident_decode(ql, orc, case):
    rng = np.random.default_rng(case.N)
    rows = None if case.N * case.K <= 4096 * 1024 else np.sort(rng.choice(case.N, size=600, replace=False))
    if rows is not None:
        rows[-1] = case.N - 1
    _run_case(ql, orc, case, rows)


# the same kernel with 16 warps, for code blocks that fill more than half of an SM's shared memory
# (one CTA per SM), and with up to 8 row tiles per CTA: N = 11008 -> 74-75 rows (5 tiles, 3 row
# groups of 5 warps, the 16th warp idle), 9472 -> 64, 13000 -> 87-88 (6 tiles), 8000 -> 54, 7400 -> 50
BIG_RESIDENT = [synth.AffineCase(f"resident16_b{b}_g{g}_M{M}_K{K}_N{N}_{pd}", M, K, N, b, g, "bf16", pd, bias,
                                 seed=b + M + N)
                for (b, g, K, N, M, pd, bias) in [(4, 128, 4096, 11008, 1, "bf16", True),
                                                  (4, 64, 4096, 9472, 5, "f32", False),
                                                  (8, 64, 2048, 9472, 8, "bf16", True),
                                                  (2, 128, 8192, 8000, 1, "bf16", True),
                                                  (4, 32, 3072, 13000, 1, "bf16", False),
                                                  (8, 128, 2048, 7400, 1, "f32", True)]]


@pytest.mark.parametrize("case", BIG_RESIDENT, ids=[c.name for c in BIG_RESIDENT])
def test_affine_resident_decode_16_warps(ql, orc, case):
    rng = np.random.default_rng(case.N)
    rows = np.sort(rng.choice(case.N, size=400, replace=False))
    rows[0], rows[-1] = 0, case.N - 1
    _run_case(ql, orc, case, rows)


def test_affine_rejects_bad_args(ql):
    x = torch.zeros((1, 96), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((4, 12), dtype=torch.int32, device="cuda")
    s = torch.zeros((4, 1), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ql.QlinError) as e:
        ql.matmul(x, codes, s, s, 4, 64)  # K % g != 0
    assert e.value.status == ql.QLIN_ERR_INVALID_ARG
    with pytest.raises(ql.QlinError) as e:
        ql.matmul(x, codes, s, s, 7, 32)  # 7-bit codes
    assert e.value.status == ql.QLIN_ERR_UNSUPPORTED
    assert ql.device_status() == ql.QLIN_OK


PREFILL_SMALL = [
    synth.AffineCase(f"prefill_b4_g{g}_M{M}_K{K}_N{N}_{xd}", M, K, N, 4, g, xd, "bf16", True, seed=17)
    for (M, K, N, g, xd) in [(17, 256, 128, 64, "bf16"), (128, 512, 256, 128, "bf16"), (200, 1024, 300, 32, "bf16"),
                             (300, 2048, 640, 64, "bf16"),
                             # K % 64 == 32 (half of the last stage past K) and K/g % 8 != 0 (scalar parameter windows)
                             (40, 1056, 200, 32, "bf16"),
                             # more 128 x 256 tiles (160) than SMs: a persistent CTA takes a second tile
                             (1280, 512, 4096, 32, "bf16"),
                             # short K: few terms, little cancellation -- the products' own error must meet the bar
                             (1280, 128, 4096, 32, "bf16"), (300, 64, 520, 32, "bf16"), (64, 128, 128, 64, "bf16"),
                             # fp32 x (and output, bias) through the same fp16 tensor-core path
                             (100, 512, 384, 64, "f32"), (33, 128, 64, 128, "f32"),
                             # 384-token tiles (two 192-column accumulators), taken when they need fewer
                             # tile rounds: 1100 tokens x 32 weight tiles -> 3 x 32 (1 round instead of 2),
                             # the last tile holding 332 tokens; 740 x 112 -> 2 x 112 (2 rounds, not 3)
                             (1100, 256, 4096, 64, "bf16"), (1100, 128, 4096, 32, "f32"),
                             (740, 64, 14336, 64, "bf16")]
]
@pytest.mark.parametrize("case", PREFILL_SMALL, ids=[c.name for c in PREFILL_SMALL])
def test_affine_prefill_small(ql, orc, case):
    _run_case(ql, orc, case)


def test_affine_prefill_config_sampled(ql, orc):
    """2048 x 4096 x 14336 (outlier weights), one call; sampled tokens x features."""
    case = synth.AFFINE_PREFILL
    w = case.weight()
    codes, s, b = orc.affine_quantize(w, 4, 64, True)
    x = case.x()
    lb = case.layer_bias()
    y = ql.matmul(x.torch("cuda"), u32_dev(codes), params_dev(s, "bf16"), params_dev(b, "bf16"), 4, 64,
                  lb.torch("cuda"))
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    toks = np.sort(rng.choice(case.M, size=48, replace=False))
    feats = np.sort(rng.choice(case.N, size=96, replace=False))
    feats[-1] = case.N - 1
    yr, mag = orc.affine_matmul(x.vals[toks], codes[feats], s[feats], b[feats], 4, 64, lb.vals[feats])
    ys = y[torch.as_tensor(toks, device="cuda")][:, torch.as_tensor(feats, device="cuda")]
    assert_fp_close(ys, yr, mag, lb.vals[feats], case.name)
