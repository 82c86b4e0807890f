"""GPU parity of the per-group INT8 layer (cider/ops.py pergroup_linear) and its weight quantiser
against the oracle: M == 1 (FP activation) and M > 1 (int8 activation quantisation)."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    return build_lib()


@pytest.mark.parametrize("g", [64, 128, 256])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
@pytest.mark.parametrize("aligned", [True, False])
def test_quantize_int8_groups_bit_exact(ql, orc, g, wdt, aligned):
    w = synth.normal(41, (96, 1024), 0.02)
    w[3, 128:256] = 0.0           # zero groups -> scale 1
    w[5, 700] = 0.9               # one group dominated by an outlier
    if wdt == "bf16":
        w = torch.from_numpy(w).to(torch.bfloat16).float().numpy()
    q_ref, s_ref = orc.quantize_int8_groups(w, g)
    wt = torch.from_numpy(w).to(torch.bfloat16 if wdt == "bf16" else torch.float32).cuda()
    if not aligned:  # data one element past a 16-byte boundary: the warp-per-group kernel
        flat = torch.empty(wt.numel() + 1, dtype=wt.dtype, device="cuda")
        wt = flat[1:].view(wt.shape).copy_(wt)
    q, s = ql.quantize_int8_groups(wt, g)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


def _case(ql, orc, M, K, N, g, xd, bias, seed, rows=None):
    w = synth.normal(seed, (N, K), 0.02)
    q, s = orc.quantize_int8_groups(w, g)
    x = synth.activations(seed + 1, (M, K), xd)
    lb = synth.activations(seed + 2, (N,), xd, 0.01) if bias else None
    y = ql.pergroup_linear(x.torch("cuda"), to_dev(q), to_dev(s), g, None if lb is None else lb.torch("cuda"))
    torch.cuda.synchronize()
    if rows is not None:
        q, s = q[rows], s[:, rows]
        y = y[:, torch.as_tensor(rows, device="cuda")]
    bv = None if lb is None else (lb.vals if rows is None else lb.vals[rows])
    yr, mag, _, _ = orc.pergroup_linear(x.vals, q, s, g, bv)
    return assert_fp_close(y, yr, mag, bv, f"pergroup M{M} K{K} N{N} g{g} {xd}")


SMALL = [(M, K, N, g, xd, b) for (M, K, N) in [(1, 512, 200), (2, 1024, 96), (17, 512, 130), (300, 768, 264)]
         for g in (64, 128, 256) if K % g == 0
         for (xd, b) in [("bf16", True), ("f32", False)]]


@pytest.mark.parametrize("M,K,N,g,xd,bias", SMALL, ids=[f"M{c[0]}_K{c[1]}_N{c[2]}_g{c[3]}_{c[4]}" for c in SMALL])
def test_pergroup_small(ql, orc, M, K, N, g, xd, bias):
    _case(ql, orc, M, K, N, g, xd, bias, seed=43)


@pytest.mark.parametrize("M", [1, 4, 256])
def test_pergroup_llm_shape_sampled_rows(ql, orc, M):
    """K = N = 4096, group 128: every token, 256 sampled output rows (the last included)."""
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(4096, size=256, replace=False))
    rows[-1] = 4095
    _case(ql, orc, M, 4096, 4096, 128, "bf16", True, seed=47, rows=rows)


def test_pergroup_two_accumulator_tiles(ql, orc):
    """1100 tokens, N = 4096: 3 x 32 tiles of 384 tokens (two 192-column accumulators) instead of
    5 x 32 of 256 on 148 SMs; the last tile holds 332 tokens.  256 sampled output rows."""
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(4096, size=256, replace=False))
    rows[0], rows[-1] = 0, 4095
    _case(ql, orc, 1100, 256, 4096, 64, "bf16", True, seed=49, rows=rows)


def test_pergroup_dispatch_on_gpu(ql, orc):
    """The page's dispatch on the GPU: the same token alone (M == 1, FP activation) and twice (M == 2,
    int8 activation) gives different results, each matching its own oracle branch."""
    K, N, g = 512, 64, 64
    w = synth.normal(51, (N, K), 0.02)
    q, s = orc.quantize_int8_groups(w, g)
    x = synth.activations(52, (1, K), "bf16")
    y1 = ql.pergroup_linear(x.torch("cuda"), to_dev(q), to_dev(s), g)
    x2 = torch.cat([x.torch("cuda"), x.torch("cuda")])
    y2 = ql.pergroup_linear(x2, to_dev(q), to_dev(s), g)
    torch.cuda.synchronize()
    r1, m1, _, _ = orc.pergroup_linear(x.vals, q, s, g)
    r2, m2, _, _ = orc.pergroup_linear(np.vstack([x.vals, x.vals]), q, s, g)
    assert_fp_close(y1, r1, m1, None, "M == 1")
    assert_fp_close(y2, r2, m2, None, "M == 2")
    assert not torch.equal(y1[0], y2[0])


def test_pergroup_rejects_bad_args(ql):
    x = torch.zeros((2, 512), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((8, 512), dtype=torch.int8, device="cuda")
    s = torch.ones((512 // 64, 8), device="cuda")
    with pytest.raises(ql.QlinError) as e:
        ql.pergroup_linear(x, w, s, 32)
    assert e.value.status == ql.QLIN_ERR_UNSUPPORTED
    with pytest.raises(ql.QlinError) as e:
        ql.pergroup_linear(x, w, s, 64, workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == ql.QLIN_ERR_WORKSPACE
    assert ql.device_status() == ql.QLIN_OK
