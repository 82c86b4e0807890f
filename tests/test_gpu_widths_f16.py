"""GPU parity of the MLX code widths 1, 3, 5 and 6 (codes straddling 32-bit words) and of fp16
activations, weights and group parameters, against the oracle [nuvec-nn QuantizedLinear:
from_linear (bits 1..6, 8), dequantized_weight, forward]."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, host_f32, params_dev, to_dev, u32_dev

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@pytest.fixture(scope="module")
def ql():
    return build_lib()


def _w_dev(w, w_dt):
    """(values the device sees as fp32, device tensor) for weights stored in w_dt."""
    if w_dt == "bf16":
        vals, bits = synth.to_bf16(w)
        return vals, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    if w_dt == "f16":
        vals, bits = synth.to_f16(w)
        return vals, torch.from_numpy(bits.view(np.int16)).view(torch.float16).cuda()
    return w, to_dev(w)


QUANT = [(b, g, p, wd) for b in (1, 3, 5, 6) for g in (32, 64, 128) for p in ("f32", "bf16", "f16")
         for wd in ("f32", "bf16", "f16")] + \
        [(b, g, "f16", wd) for b in (2, 4, 8) for g in (32, 128) for wd in ("f16", "bf16")]


@pytest.mark.parametrize("bits,g,p_dt,w_dt", QUANT, ids=[f"b{c[0]}_g{c[1]}_p{c[2]}_w{c[3]}" for c in QUANT])
def test_quantize_bit_exact(ql, orc, bits, g, p_dt, w_dt):
    N, K = 37, 5 * g
    w = synth.outlier_weights(500 + bits + g, N, K, frac=0.01)
    w[2, g:2 * g] = -0.125  # a constant group
    wv, wd = _w_dev(w, w_dt)
    codes, s, b = ql.quantize(wd, bits, g, TORCH_DT[p_dt])
    torch.cuda.synchronize()
    rc, rs, rb = orc.affine_quantize(wv, bits, g, p_dt)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(host_f32(s), rs)
    assert np.array_equal(host_f32(b), rb)


DEQ = [(b, g, p, o) for b in (1, 3, 5, 6) for g in (32, 128) for p in ("f32", "bf16", "f16")
       for o in ("f32", "bf16", "f16")] + [(b, 64, "f16", "f16") for b in (2, 4, 8)]


@pytest.mark.parametrize("bits,g,p_dt,o_dt", DEQ, ids=[f"b{c[0]}_g{c[1]}_p{c[2]}_o{c[3]}" for c in DEQ])
def test_dequantize_bit_exact(ql, orc, bits, g, p_dt, o_dt):
    N, K = 29, 3 * g
    w = synth.normal(600 + bits, (N, K), 0.02)
    rc, rs, rb = orc.affine_quantize(w, bits, g, p_dt)
    out = ql.dequantize(u32_dev(rc), params_dev(rs, p_dt), params_dev(rb, p_dt), K, bits, g, TORCH_DT[o_dt])
    torch.cuda.synchronize()
    ref = orc.affine_dequantize(rc, rs, rb, K, bits, g)  # fp32, one fma per weight
    got = out.float().cpu().numpy()
    if o_dt == "bf16":
        ref = orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(ref))
    elif o_dt == "f16":
        ref = orc.round_f16(ref)
    assert np.array_equal(got, ref)


def _run_matmul(ql, orc, case: synth.AffineCase):
    w = case.weight()
    codes, s, b = orc.affine_quantize(w, case.bits, case.group_size, case.param_dtype)
    x = case.x()
    lb = case.layer_bias()
    y = ql.matmul(x.torch("cuda"), u32_dev(codes), params_dev(s, case.param_dtype), params_dev(b, case.param_dtype),
                  case.bits, case.group_size, None if lb is None else lb.torch("cuda"))
    torch.cuda.synchronize()
    assert y.dtype == TORCH_DT[case.x_dtype]
    bias_v = None if lb is None else lb.vals
    yr, mag = orc.affine_matmul(x.vals, codes, s, b, case.bits, case.group_size, bias_v)
    return assert_fp_close(y, yr, mag, bias_v, case.name)


# the general decode kernel: odd widths, 2 bits in groups of 32, fp16 anywhere; K a multiple of 32
# that is not one of 256 (a partial last span), N not a multiple of the 32-row warp tile, M across
# the 1 / 2 / 4 / 8-token tiles and past 8 (two launches) and 16
GENERAL = [synth.AffineCase(f"b{b}_g{g}_M{M}_K{K}_N{N}_{xd}_{pd}", M, K, N, b, g, xd, pd, bias, seed=b * 7 + M)
           for (b, g, K, N) in [(1, 32, 544, 70), (3, 32, 800, 133), (3, 128, 1280, 64), (5, 64, 576, 97),
                                (6, 32, 672, 150), (6, 128, 1024, 33), (2, 32, 480, 90)]
           for M in (1, 3, 8, 20)
           for (xd, pd, bias) in [("f16", "f16", True), ("bf16", "f32", False), ("f32", "bf16", True)]]
# fp16 through the power-of-two widths (fp16 x or parameters take the general kernel below 17 tokens)
GENERAL += [synth.AffineCase(f"b{b}_g{g}_M{M}_f16x_{pd}", M, 512, 120, b, g, "f16", pd, True, seed=b + M)
            for b in (2, 4, 8) for g in (64, 128) for M in (1, 9) for pd in ("f16", "bf16")]


@pytest.mark.parametrize("case", GENERAL, ids=[c.name for c in GENERAL])
def test_general_matmul(ql, orc, case):
    _run_matmul(ql, orc, case)


# the tensor-core prefill with fp16 activations / output / bias
PREFILL_F16 = [synth.AffineCase(f"prefill_f16_M{M}_K{K}_N{N}_g{g}", M, K, N, 4, g, "f16", "bf16", True, seed=31)
               for (M, K, N, g) in [(17, 256, 128, 64), (300, 1024, 520, 32), (64, 128, 256, 128)]]


@pytest.mark.parametrize("case", PREFILL_F16, ids=[c.name for c in PREFILL_F16])
def test_prefill_f16(ql, orc, case):
    _run_matmul(ql, orc, case)


def test_long_rows_small_groups_fall_back(ql, orc):
    """K = 16384 in groups of 32: the decode kernel's per-row group parameters (512 groups x 64 rows x
    8 bytes) do not fit in shared memory, so the call runs the general kernel instead of failing."""
    case = synth.AffineCase("b4_g32_M2_K16384_N100", 2, 16384, 100, 4, 32, "bf16", "bf16", True, seed=5)
    _run_matmul(ql, orc, case)


INT_F16 = [synth.IntCase(f"f16_M{M}_K{K}_N{N}", M, K, N, bias=True, x_dtype="f16", seed=M + 3)
           for (M, K, N) in [(1, 512, 256), (9, 1024, 160), (200, 768, 272)]]


@pytest.mark.parametrize("case", INT_F16, ids=[c.name for c in INT_F16])
def test_w8a8_f16(ql, orc, case):
    w = case.weight()
    qw, sw = orc.quantize_int8_rows(w)
    x = case.x()
    lb = case.layer_bias()
    y = ql.w8a8_linear(x.torch("cuda"), to_dev(qw), to_dev(sw), lb.torch("cuda"))
    torch.cuda.synchronize()
    assert y.dtype == torch.float16
    yr, mag, _, _ = orc.w8a8_linear(x.vals, qw, sw, lb.vals)
    assert_fp_close(y, yr, mag, lb.vals, case.name)


@pytest.mark.parametrize("case", INT_F16, ids=[c.name for c in INT_F16])
def test_w4a8_f16(ql, orc, case):
    w = case.weight()
    P, sw = orc.pack_int4_cols(np.ascontiguousarray(w.T))
    x = case.x()
    lb = case.layer_bias()
    y = ql.w4a8_linear(x.torch("cuda"), to_dev(P), to_dev(sw), lb.torch("cuda"))
    torch.cuda.synchronize()
    assert y.dtype == torch.float16
    yr, mag, _, _ = orc.w4a8_linear(x.vals, P, sw, lb.vals)
    assert_fp_close(y, yr, mag, lb.vals, case.name)


@pytest.mark.parametrize("M", [1, 2, 40])
def test_pergroup_f16(ql, orc, M):
    K, N, g = 1024, 136, 128
    w = synth.normal(71, (N, K), 0.02)
    q, s = orc.quantize_int8_groups(w, g)
    x = synth.activations(72, (M, K), "f16")
    lb = synth.activations(73, (N,), "f16", 0.01)
    y = ql.pergroup_linear(x.torch("cuda"), to_dev(q), to_dev(s), g, lb.torch("cuda"))
    torch.cuda.synchronize()
    assert y.dtype == torch.float16
    yr, mag, _, _ = orc.pergroup_linear(x.vals, q, s, g, lb.vals)
    assert_fp_close(y, yr, mag, lb.vals, f"pergroup f16 M{M}")


def test_int8_quantisers_f16_weights(ql, orc):
    """Every int8 weight quantiser reads fp16 weights bit-exactly like fp32 ones of the same values."""
    w = synth.normal(81, (48, 512), 0.02)
    w[4] = 0.0
    wv, wd = _w_dev(w, "f16")
    q, s = ql.quantize_int8_rows(wd)
    rq, rs = orc.quantize_int8_rows(wv)
    assert np.array_equal(q.cpu().numpy(), rq) and np.array_equal(s.cpu().numpy(), rs)
    q, s = ql.quantize_int8_groups(wd, 128)
    rq, rs = orc.quantize_int8_groups(wv, 128)
    assert np.array_equal(q.cpu().numpy(), rq) and np.array_equal(s.cpu().numpy(), rs)
    q, s = ql.quantize_weight_int8(wd, 99.5)
    rq, rs = orc.quantize_weight_int8_clip(wv, 99.5)
    assert np.array_equal(q.cpu().numpy(), rq) and np.array_equal(s.cpu().numpy(), rs)
    wt = np.ascontiguousarray(wv.T)  # [K, N] for the per-column int4 packer
    P, s = ql.pack_int4_cols(torch.from_numpy(wt).to(torch.float16).cuda())
    rP, rs = orc.pack_int4_cols(wt)
    assert np.array_equal(P.cpu().numpy(), rP) and np.array_equal(s.cpu().numpy(), rs)
