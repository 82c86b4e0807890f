"""GPU parity of the quantisers and the dequantiser (bit-exact with the oracle)."""
import numpy as np
import pytest
import torch

import synth
from helpers import build_lib, host_bits16, host_f32, params_dev, to_dev, u32_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    return build_lib()


def _w_dev(w, w_dt):
    if w_dt == "bf16":
        vals, bits = synth.to_bf16(w)
        return vals, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return w, to_dev(w)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("g", [32, 64, 128])
@pytest.mark.parametrize("p_dt", ["f32", "bf16"])
@pytest.mark.parametrize("w_dt", ["f32", "bf16"])
def test_quantize_bit_exact(ql, orc, bits, g, p_dt, w_dt):
    N, K = 75, 6 * g
    w = synth.outlier_weights(100 + bits + g, N, K, frac=0.01)
    w[3, :g] = 0.25  # a constant group
    wv, wd = _w_dev(w, w_dt)
    codes, s, b = ql.quantize(wd, bits, g, torch.bfloat16 if p_dt == "bf16" else torch.float32)
    torch.cuda.synchronize()
    rc, rs, rb = orc.affine_quantize(wv, bits, g, p_dt == "bf16")
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(host_f32(s), rs)
    assert np.array_equal(host_f32(b), rb)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("g", [32, 128])
@pytest.mark.parametrize("p_dt", ["f32", "bf16"])
@pytest.mark.parametrize("o_dt", ["f32", "bf16"])
def test_dequantize_bit_exact(ql, orc, bits, g, p_dt, o_dt):
    N, K = 53, 4 * g
    w = synth.normal(200 + bits, (N, K), 0.02)
    rc, rs, rb = orc.affine_quantize(w, bits, g, p_dt == "bf16")
    out = ql.dequantize(u32_dev(rc), params_dev(rs, p_dt), params_dev(rb, p_dt), K, bits, g,
                        torch.bfloat16 if o_dt == "bf16" else torch.float32)
    torch.cuda.synchronize()
    ref = orc.affine_dequantize(rc, rs, rb, K, bits, g)
    if o_dt == "bf16":
        assert np.array_equal(host_bits16(out), orc.f32_to_bf16_bits(ref))
    else:
        assert np.array_equal(out.cpu().numpy(), ref)


def _offset_copy(t, elems=1):
    """A contiguous copy of t whose data starts `elems` elements past an allocation (not 16-byte
    aligned): the quantiser and dequantiser then take their per-group / per-word kernels."""
    flat = torch.empty(t.numel() + elems, dtype=t.dtype, device=t.device)
    v = flat[elems:].view(t.shape)
    v.copy_(t)
    assert v.data_ptr() % 16 != 0
    return v


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("w_dt", ["f32", "bf16"])
def test_quantize_unaligned_weights_bit_exact(ql, orc, bits, w_dt):
    g = 64
    N, K = 9, 3 * g
    w = synth.outlier_weights(150 + bits, N, K, frac=0.02)
    wv, wd = _w_dev(w, w_dt)
    codes, s, b = ql.quantize(_offset_copy(wd), bits, g, torch.float32)
    torch.cuda.synchronize()
    rc, rs, rb = orc.affine_quantize(wv, bits, g, False)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(host_f32(s), rs)
    assert np.array_equal(host_f32(b), rb)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("aligned", [True, False])
def test_dequantize_word_tail_and_unaligned_bit_exact(ql, orc, bits, aligned):
    # K = g = 32: 32 * bits / 32 words per row; 53 rows give a word count that is not a multiple of 4
    # for 2-bit codes (the vector kernel's tail); unaligned codes take the per-word kernel
    g, N, K = 32, 53, 32
    w = synth.normal(250 + bits, (N, K), 0.02)
    rc, rs, rb = orc.affine_quantize(w, bits, g, True)
    cd = u32_dev(rc)
    if not aligned:
        cd = _offset_copy(cd)
    out = ql.dequantize(cd, params_dev(rs, "bf16"), params_dev(rb, "bf16"), K, bits, g, torch.bfloat16)
    torch.cuda.synchronize()
    ref = orc.affine_dequantize(rc, rs, rb, K, bits, g)
    assert np.array_equal(host_bits16(out), orc.f32_to_bf16_bits(ref))


@pytest.mark.parametrize("w_dt", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 8192), (7, 1000), (33, 4096), (3, 24), (700, 1000), (1024, 8192), (600, 24),
                                   # launches of few rows: 1024 threads per row with 1, 2 and 4 pieces each
                                   # (the last ragged), then 512 threads with 2, 4 and 8; the 296 / 297 rows
                                   # step between the two on a 148-SM part
                                   (150, 12000), (50, 30000), (296, 8192), (297, 8192), (400, 4096),
                                   (500, 9000), (300, 20000)])
def test_quantize_int8_rows_bit_exact(ql, orc, w_dt, shape):
    R, Cc = shape
    w = synth.normal(300 + R, (R, Cc), 1.0)
    if R > 2:
        w[1] = 0.0
        w[2, 5] = 1e4
    wv, wd = _w_dev(w, w_dt)
    q, s = ql.quantize_int8_rows(wd)
    torch.cuda.synchronize()
    rq, rs = orc.quantize_int8_rows(wv)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), rs)


@pytest.mark.parametrize("w_dt", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(3, 64), (200, 4096), (700, 1000)])
def test_quantize_int8_rows_half_integer_ties(ql, orc, w_dt, shape):
    """Rows whose absmax is 127 have scale 1, so half-integers x.5 quantise exactly at a tie (rint
    rounds to even): every piece of eight leaves the multiply path for the division path."""
    R, Cc = shape
    rng = np.random.default_rng(R + Cc)
    w = (rng.integers(-127, 127, size=(R, Cc)) + 0.5).astype(np.float32)
    w[:, 0] = 127.0
    w[::3, 1:9] = np.float32(2.5)  # one piece of ties only
    wv, wd = _w_dev(w, w_dt)
    q, s = ql.quantize_int8_rows(wd)
    torch.cuda.synchronize()
    rq, rs = orc.quantize_int8_rows(wv)
    assert np.all(rs == 1.0)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), rs)


@pytest.mark.parametrize("w_dt", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 4), (64, 96), (512, 300), (8192, 64)])
def test_pack_int4_cols_bit_exact(ql, orc, w_dt, shape):
    K, N = shape
    w = synth.normal(400 + K, (K, N), 0.02)
    if N > 3:
        w[:, 2] = 0.0
    wv, wd = _w_dev(w, w_dt)
    P, s = ql.pack_int4_cols(wd)
    torch.cuda.synchronize()
    rP, rs = orc.pack_int4_cols(wv)
    assert np.array_equal(P.cpu().numpy(), rP)
    assert np.array_equal(s.cpu().numpy(), rs)


def test_quantize_full_prefill_weight_bit_exact(ql, orc):
    """The 14336 x 4096 prefill weight (outliers, 4-bit g64, bf16 params): every code."""
    case = synth.AFFINE_PREFILL
    w = case.weight()
    codes, s, b = ql.quantize(to_dev(w), 4, 64, torch.bfloat16)
    torch.cuda.synchronize()
    rc, rs, rb = orc.affine_quantize(w, 4, 64, True)
    assert np.array_equal(codes.cpu().numpy().view(np.uint32), rc)
    assert np.array_equal(host_f32(s), rs)
    assert np.array_equal(host_f32(b), rb)


CLIP_CASES = [(R, C, p, wdt) for (R, C) in [(7, 1000), (64, 4096), (3, 1), (5, 33), (2, 32768)]
              for p in (99.9, 50.0, 0.0, 100.0, 97.25) for wdt in ("f32", "bf16")]


@pytest.mark.parametrize("R,C,p,wdt", CLIP_CASES, ids=[f"R{c[0]}_C{c[1]}_p{c[2]}_{c[3]}" for c in CLIP_CASES])
def test_quantize_weight_int8_clip_bit_exact(ql, orc, R, C, p, wdt):
    """quantize_weight_int8 with clip_percentile [cider/ops.py]: codes and scales bit-equal to the
    oracle (which is itself pinned to np.percentile)."""
    import synth
    w = synth.normal(71 + C, (R, C), 0.02)
    w[0, : min(C, 3)] = [4.0, -3.0, 2.5][: min(C, 3)]  # outliers the clip cuts
    if R > 1:
        w[1, :] = 0.0                                    # zero row
    if wdt == "bf16":
        w = torch.from_numpy(w).to(torch.bfloat16).float().numpy()
    q_ref, s_ref = orc.quantize_weight_int8_clip(w, p)
    wt = torch.from_numpy(w).to(torch.bfloat16 if wdt == "bf16" else torch.float32).cuda()
    q, s = ql.quantize_weight_int8(wt, p)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quantize_weight_int8_no_clip_is_absmax(ql, orc):
    import synth
    w = synth.normal(72, (16, 512), 0.02)
    q_ref, s_ref = orc.quantize_int8_rows(w)
    q, s = ql.quantize_weight_int8(torch.from_numpy(w).cuda(), None)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("p", [0.0, 12.5, 50.0, 66.7, 99.0, 100.0])
def test_quantize_weight_int8_clip_ties(ql, orc, p):
    """Rows of few distinct magnitudes (every order statistic tied with its neighbours), one row of a
    single value and one with a lone nonzero: the percentile's two order statistics at every rank."""
    import synth
    rng = np.random.default_rng(int(p * 10) + 3)
    w = rng.choice(np.array([-0.5, -0.25, 0.0, 0.25, 0.5, 1.0], np.float32), size=(6, 777)).astype(np.float32)
    w[1, :] = 0.125
    w[2, :] = 0.0
    w[2, 400] = -3.0
    w[3] = synth.normal(5, (777,), 1.0)
    q_ref, s_ref = orc.quantize_weight_int8_clip(w, p)
    q, s = ql.quantize_weight_int8(torch.from_numpy(w).cuda(), p)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)
