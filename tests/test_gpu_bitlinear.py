"""GPU parity of bitlinear_matmul (ternary weights packed 4:1 along N)."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    return build_lib()


def _run(ql, orc, case: synth.BitLinearCase):
    P = case.packed()
    x = case.x()
    lb = case.layer_bias()
    ws = torch.tensor([case.weight_scale], dtype=torch.float32, device="cuda")
    y = ql.bitlinear_matmul(x.torch("cuda"), to_dev(P), case.N, ws, case.invert,
                            None if lb is None else lb.torch("cuda"))
    torch.cuda.synchronize()
    yr, mag = orc.bitlinear(x.vals, P, case.N, case.weight_scale, case.invert,
                            None if lb is None else lb.vals)
    return assert_fp_close(y, yr, mag, None if lb is None else lb.vals, case.name)


SMALL = [synth.BitLinearCase(f"M{M}_K{K}_N{N}_{'div' if inv else 'mul'}{'_bias' if b else ''}", M, K, N, 0.75,
                             inv, b, seed=11)
         for M in (1, 5, 8, 16) for (K, N) in [(512, 204), (1040, 64), (4096, 260)]
         for inv in (False, True) for b in (False, True)]


@pytest.mark.parametrize("case", SMALL, ids=[c.name for c in SMALL])
def test_bitlinear_small(ql, orc, case):
    _run(ql, orc, case)


# every byte value (code 3 -> weight 2), the one-CTA-per-SM split (N = 4096), 8-row CTAs in waves
# (N > 4736 on 148 SMs), K beyond one register round (K > 4096) and a partial last chunk
# (K % 64 != 0), fewer packed rows than SMs, and M > 16 (16-token slices)
WIDE = [synth.BitLinearCase(f"all_bytes_M{M}_K{K}_N{N}_{'div' if inv else 'mul'}{'_bias' if b else ''}", M, K, N,
                            0.5, inv, b, seed=21, all_bytes=True)
        for (M, K, N, inv, b) in [(1, 4096, 4096, False, False), (8, 4096, 4096, True, False),
                                  (16, 4096, 4096, False, True), (3, 1040, 6000, False, True),
                                  (8, 4112, 1024, True, False), (1, 8192, 512, False, False),
                                  (12, 2064, 64, True, True), (17, 512, 520, False, True),
                                  (40, 1024, 1024, True, False)]]


@pytest.mark.parametrize("case", WIDE, ids=[c.name for c in WIDE])
def test_bitlinear_all_bytes_and_paths(ql, orc, case):
    _run(ql, orc, case)


def test_bitlinear_code3_is_two(ql):
    """All codes 3 (weight 2): y = 2 rowsum(x) * scale, exact for small-integer x."""
    x = torch.randint(-4, 5, (5, 1024), device="cuda").to(torch.bfloat16)
    P = torch.full((16, 1024), 0xFF, dtype=torch.uint8, device="cuda")
    ws = torch.tensor([0.5], device="cuda")
    y = ql.bitlinear_matmul(x, P, 64, ws, False).float()
    expect = x.float().sum(dim=1, keepdim=True).expand(5, 64) * 2 * 0.5
    assert torch.equal(y, expect)


@pytest.mark.parametrize("case", synth.BITLINEAR_DECODE, ids=[c.name for c in synth.BITLINEAR_DECODE])
def test_bitlinear_decode_config_full(ql, orc, case):
    _run(ql, orc, case)


def test_bitlinear_code1_gives_exact_zero(ql):
    x = torch.randn((8, 512), device="cuda").to(torch.bfloat16)
    P = torch.full((64, 512), 0x55, dtype=torch.uint8, device="cuda")
    ws = torch.tensor([0.5], device="cuda")
    y = ql.bitlinear_matmul(x, P, 256, ws, False)
    assert torch.count_nonzero(y).item() == 0


def test_bitlinear_code2_rowsum(ql):
    """All codes 2: y = rowsum(x) * scale, exact for small-integer x."""
    x = torch.randint(-4, 5, (3, 1024), device="cuda").to(torch.bfloat16)
    P = torch.full((16, 1024), 0xAA, dtype=torch.uint8, device="cuda")
    ws = torch.tensor([0.5], device="cuda")
    for inv, f in ((False, 0.5), (True, 2.0)):
        y = ql.bitlinear_matmul(x, P, 64, ws, inv).float()
        expect = x.float().sum(dim=1, keepdim=True).expand(3, 64) * f
        assert torch.equal(y, expect)


def test_bitlinear_rejects_ragged(ql):
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    P = torch.zeros((2, 64), dtype=torch.uint8, device="cuda")
    ws = torch.ones(1, device="cuda")
    with pytest.raises(ql.QlinError) as e:
        ql.bitlinear_matmul(x, P, 6, ws, False)
    assert e.value.status == ql.QLIN_ERR_INVALID_ARG


# M > 16: the tcgen05 GEMM (bf16 x, exact bf16 ternary weights, 32 packed rows x 4 fields per tile)
PREFILL = [synth.BitLinearCase(f"prefill_M{M}_K{K}_N{N}_{'div' if inv else 'mul'}{'_bias' if b else ''}", M, K, N,
                               0.5, inv, b, seed=25, all_bytes=ab)
           for (M, K, N, inv, b, ab) in [(300, 1040, 600, False, True, True),   # K % 32 == 16, ragged tiles
                                         (256, 512, 4096, True, False, False),
                                         (33, 2048, 136, False, False, True),
                                         (512, 4096, 512, False, True, False),
                                         # 384-token tiles (3 x 32 tiles instead of 5 x 32 of 256 on 148
                                         # SMs): the last holds 332 tokens, its second 192-row box 140
                                         (1100, 512, 4096, False, True, False)]]


@pytest.mark.parametrize("case", PREFILL, ids=[c.name for c in PREFILL])
def test_bitlinear_prefill(ql, orc, case):
    _run(ql, orc, case)


def test_bitlinear_prefill_llm_sampled(ql, orc):
    """M = 2048, K = N = 4096 in one call; 48 sampled tokens x all outputs of 64 sampled packed rows."""
    case = synth.BitLinearCase("prefill_2048", 2048, 4096, 4096, 0.5, True, False, seed=27)
    P = case.packed()
    x = case.x()
    ws = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    y = ql.bitlinear_matmul(x.torch("cuda"), to_dev(P), 4096, ws, True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    toks = np.sort(rng.choice(2048, size=48, replace=False))
    prow = np.sort(rng.choice(1024, size=64, replace=False))
    prow[-1] = 1023
    R = 1024
    cols = np.concatenate([prow + j * R for j in range(4)])  # output n = r + j N/4
    yr, mag = orc.bitlinear(x.vals[toks], P[prow], 4 * len(prow), 0.5, True)
    ys = y[torch.as_tensor(toks, device="cuda")][:, torch.as_tensor(cols, device="cuda")]
    assert_fp_close(ys, yr, mag, None, "prefill_2048 sampled")
