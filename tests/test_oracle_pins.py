"""Pins for the CPU oracle: checks it against what the pages and the
mathematics fix, never against a retyped copy of its own formulas.

Every test here runs without a GPU.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([part.split() for part in line.split("|")])
    return rows


def _row_as_bitstream(words_row):
    """A row of uint32 words read as one little-endian integer."""
    return int.from_bytes(np.ascontiguousarray(words_row, dtype="<u4").tobytes(), "little")


# ------------------------------------------------------------------ packing

def test_pack_golden_words(orc):
    """Hand-computed words of the LSB-first b-bit layout (nuvec-nn QuantizedLinear, weight)."""
    for (bits,), codes, words in _golden_rows("pack_words.txt"):
        bits = int(bits)
        q = np.array([[int(c) for c in codes]], np.uint8)
        want = np.array([[int(w, 16) for w in words]], np.uint32)
        got = orc.pack(q, bits)
        assert got.shape == want.shape
        assert np.array_equal(got, want), (bits, got, want)
        assert np.array_equal(orc.unpack(got, q.shape[1], bits), q)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 8])
def test_pack_is_a_little_endian_bitstream(orc, bits):
    """Row of words == sum_k q[k] << (bits*k) as one integer; unpack inverts pack."""
    rng = np.random.default_rng(bits)
    q = rng.integers(0, 2 ** bits, size=(5, 256)).astype(np.uint8)
    words = orc.pack(q, bits)
    assert words.shape == (5, 256 * bits // 32)
    for n in range(q.shape[0]):
        expect = sum(int(c) << (bits * k) for k, c in enumerate(q[n]))
        assert _row_as_bitstream(words[n]) == expect
    assert np.array_equal(orc.unpack(words, 256, bits), q)


def test_pack_8bit_is_byte_order(orc):
    q = np.arange(64, dtype=np.uint8).reshape(2, 32) * 3
    words = orc.pack(q, 8)
    assert np.array_equal(words.view(np.uint8).reshape(2, 32), q)


def test_pack_rejects_out_of_range(orc):
    with pytest.raises(orc.OracleError):
        orc.pack(np.full((1, 8), 16, np.uint8), 4)


# ------------------------------------------------------------------ bf16 rounding

def test_bf16_rounding_matches_torch(orc):
    """The oracle's own bf16 rounding agrees with torch's RNE conversion."""
    v = np.concatenate([synth.normal(5, (4096,), 1.0), synth.normal(6, (4096,), 1e-3),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.4e38, -1e-40], np.float32)])
    _, bits_t = synth.to_bf16(v)
    assert np.array_equal(orc.f32_to_bf16_bits(v), bits_t)
    # halfway cases: 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0)
    assert orc.bf16_bits_to_f32(orc.f32_to_bf16_bits(np.array([1.00390625], np.float32)))[0] == 1.0


# ------------------------------------------------------------------ affine quantize / dequantize

def _dyadic_case(N, K, g, bits, seed):
    """w = bias + q*scale exactly, scale a power of two, each group holding
    both 0 and 2^b-1 so that min-max recovers scale and bias exactly."""
    rng = np.random.default_rng(seed)
    G = K // g
    qmax = 2 ** bits - 1
    q = rng.integers(0, qmax + 1, size=(N, K)).astype(np.uint8)
    for n in range(N):
        for gi in range(G):
            pos = rng.choice(g, size=2, replace=False) + gi * g
            q[n, pos[0]] = 0
            q[n, pos[1]] = qmax
    e = rng.integers(6, 12, size=(N, G))
    scale = np.ldexp(1.0, -e).astype(np.float32)
    bias = (rng.integers(-64, 64, size=(N, G)) * 2.0 ** -6).astype(np.float32)
    w = np.empty((N, K), np.float32)
    for n in range(N):
        for k in range(K):
            w[n, k] = Fraction(float(bias[n, k // g])) + int(q[n, k]) * Fraction(float(scale[n, k // g]))
    return q, scale, bias, w


@pytest.mark.parametrize("bits,g", [(2, 32), (4, 64), (8, 128), (4, 128), (1, 32), (3, 64), (5, 32), (6, 128)])
@pytest.mark.parametrize("bf16", [False, True, "f16"])
def test_quantize_recovers_dyadic_grid(orc, bits, g, bf16):
    """Weights on an exact grid come back as the same codes, scale and bias."""
    q, scale, bias, w = _dyadic_case(6, 2 * g, g, bits, seed=bits * 1000 + g)
    codes, s, b = orc.affine_quantize(w, bits, g, bf16)
    assert np.array_equal(s, scale)
    assert np.array_equal(b, bias)
    assert np.array_equal(orc.unpack(codes, w.shape[1], bits), q)
    # and dequantize reproduces w exactly
    assert np.array_equal(orc.affine_dequantize(codes, s, b, w.shape[1], bits, g), w)


@pytest.mark.parametrize("bits,g", [(2, 64), (4, 64), (4, 128), (8, 64), (4, 32), (1, 32), (3, 64), (5, 128),
                                    (6, 32)])
def test_quantize_roundtrip_within_half_scale(orc, bits, g):
    """|w - dequant(quant(w))| <= scale/2 (plus fp32 rounding of the step) for fp32 params."""
    w = synth.normal(11, (64, 4 * g), 0.02)
    codes, s, b = orc.affine_quantize(w, bits, g, False)
    wh = orc.affine_dequantize(codes, s, b, w.shape[1], bits, g)
    srep = np.repeat(s, g, axis=1).astype(np.float64)
    err = np.abs(w.astype(np.float64) - wh)
    bound = srep * (0.5 + 2.0 ** -21 * 2 ** bits) + np.abs(w) * 2.0 ** -22 + 1e-30
    assert np.all(err <= bound), float((err - bound).max())
    # the group minimum maps to code 0 and the maximum to 2^b - 1
    q = orc.unpack(codes, w.shape[1], bits)
    G = w.shape[1] // g
    wg = w.reshape(64, G, g)
    qg = q.reshape(64, G, g)
    rows = np.arange(64)[:, None]
    grp = np.arange(G)[None, :]
    assert np.all(qg[rows, grp, wg.argmin(axis=2)] == 0)
    assert np.all(qg[rows, grp, wg.argmax(axis=2)] == 2 ** bits - 1)
    # scale and bias are exactly the min-max pair
    assert np.array_equal(b, wg.min(axis=2))


def test_quantize_roundtrip_bf16_params(orc):
    """bf16-stored params: unclipped elements stay within scale_p/2; params are bf16 values."""
    bits, g = 4, 128
    w = synth.normal(12, (64, 512), 0.02)
    codes, s, b = orc.affine_quantize(w, bits, g, True)
    for p in (s, b):
        assert np.all((p.view(np.uint32) & 0xFFFF) == 0)
    wh = orc.affine_dequantize(codes, s, b, 512, bits, g)
    srep = np.repeat(s, g, axis=1).astype(np.float64)
    brep = np.repeat(b, g, axis=1).astype(np.float64)
    t = (w - brep) / srep
    inside = (t >= -0.5) & (t <= 2 ** bits - 1 + 0.5)
    err = np.abs(w.astype(np.float64) - wh)
    bound = srep * (0.5 + 2.0 ** -19) + np.abs(w) * 2.0 ** -22
    assert inside.mean() > 0.9
    assert np.all(err[inside] <= bound[inside])


def test_quantize_constant_group(orc):
    """A constant group gets scale 1, code 0 and dequantizes to itself."""
    w = np.full((2, 64), 0.125, np.float32)
    w[1, :] = -3.0
    codes, s, b = orc.affine_quantize(w, 4, 64, False)
    assert np.all(s == 1.0)
    assert np.array_equal(b[:, 0], np.array([0.125, -3.0], np.float32))
    assert np.all(codes == 0)
    assert np.array_equal(orc.affine_dequantize(codes, s, b, 64, 4, 64), w)


def test_quantize_rejects_bad_group(orc):
    with pytest.raises(orc.OracleError):
        orc.affine_quantize(np.zeros((2, 96), np.float32), 4, 64, False)


# ------------------------------------------------------------------ affine matmul

def _bitstream_codes(words_row, K, bits):
    """Codes of one packed row, read from its little-endian integer (not via orc.unpack)."""
    v = _row_as_bitstream(words_row)
    return [(v >> (bits * k)) & ((1 << bits) - 1) for k in range(K)]


@pytest.mark.parametrize("bits,g,M,N,K", [(4, 32, 3, 5, 64), (2, 64, 2, 7, 128), (8, 32, 4, 3, 96), (3, 32, 2, 4, 64),
                                          (5, 64, 2, 3, 128), (6, 32, 3, 2, 96), (1, 32, 2, 5, 64)])
def test_affine_matmul_brute_force_exact(orc, bits, g, M, N, K):
    """Tiny layers with dyadic x and grid weights: the double sums are exact,
    so the oracle must equal an exact rational brute force."""
    q, scale, bias, w = _dyadic_case(N, K, g, bits, seed=7 + bits)
    codes, s, b = orc.affine_quantize(w, bits, g, False)
    rng = np.random.default_rng(3)
    x = (rng.integers(-8, 9, size=(M, K)) * 0.25).astype(np.float32)
    lb = (rng.integers(-8, 9, size=(N,)) * 0.125).astype(np.float32)
    y, mag = orc.affine_matmul(x, codes, s, b, bits, g, lb)
    for n in range(N):
        qn = _bitstream_codes(codes[n], K, bits)
        for m in range(M):
            acc = Fraction(float(lb[n]))
            absacc = Fraction(0)
            for k in range(K):
                wk = Fraction(float(s[n, k // g])) * qn[k] + Fraction(float(b[n, k // g]))
                acc += Fraction(float(x[m, k])) * wk
                absacc += abs(Fraction(float(x[m, k])) * wk)
            assert y[m, n] == float(acc)
            assert mag[m, n] == float(absacc)


def test_affine_matmul_vs_torch_float64(orc):
    """Random layer: oracle y == torch float64 x @ w_hat^T + bias (w_hat = oracle dequant)."""
    case = synth.AffineCase("t", 3, 256, 40, 4, 64, "f32", "f32", True, seed=21)
    w = case.weight()
    codes, s, b = orc.affine_quantize(w, 4, 64, False)
    wh = orc.affine_dequantize(codes, s, b, 256, 4, 64)
    x = case.x().vals
    lb = case.layer_bias().vals
    y, _ = orc.affine_matmul(x, codes, s, b, 4, 64, lb)
    ref = (torch.from_numpy(x).double() @ torch.from_numpy(wh).double().T
           + torch.from_numpy(lb).double()).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)
    # and without bias
    y0, _ = orc.affine_matmul(x, codes, s, b, 4, 64, None)
    assert np.allclose(y0, y - lb[None, :].astype(np.float64), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ BitLinear

def _ternary_case(M, K, N, seed):
    rng = np.random.default_rng(seed)
    x = rng.integers(-16, 17, size=(M, K)).astype(np.float32)
    return x


@pytest.mark.parametrize("invert", [False, True])
def test_bitlinear_code1_is_zero(orc, invert):
    M, K, N = 3, 64, 16
    x = _ternary_case(M, K, N, 1)
    P = orc.pack_ternary(np.ones((N, K), np.uint8))
    assert np.all(P == 0x55)
    y, _ = orc.bitlinear(x, P, N, 0.5, invert)
    assert np.all(y == 0.0)
    lb = np.linspace(-1, 1, N).astype(np.float32)
    yb, _ = orc.bitlinear(x, P, N, 0.5, invert, lb)
    assert np.array_equal(yb, np.broadcast_to(lb.astype(np.float64), (M, N)))


@pytest.mark.parametrize("invert,factor", [(False, 0.5), (True, 2.0)])
def test_bitlinear_code2_and_code0_are_rowsums(orc, invert, factor):
    M, K, N = 4, 128, 8
    x = _ternary_case(M, K, N, 2)
    rows = x.astype(np.float64).sum(axis=1)
    P2 = orc.pack_ternary(np.full((N, K), 2, np.uint8))
    P0 = orc.pack_ternary(np.zeros((N, K), np.uint8))
    y2, _ = orc.bitlinear(x, P2, N, 0.5, invert)
    y0, _ = orc.bitlinear(x, P0, N, 0.5, invert)
    assert np.array_equal(y2, np.repeat(rows[:, None] * factor, N, axis=1))
    assert np.array_equal(y0, np.repeat(-rows[:, None] * factor, N, axis=1))


def test_bitlinear_one_hot_row_mapping(orc):
    """Code j of byte P[r, k] drives output r + j*N/4 (BitLinear kernel source)."""
    M, K, N = 2, 16, 12
    R = N // 4
    x = _ternary_case(M, K, N, 3)
    for r in range(R):
        for j in range(4):
            for k in (0, 5, K - 1):
                P = np.full((R, K), 0x55, np.uint8)
                P[r, k] = (0x55 & ~(3 << (2 * j))) | (2 << (2 * j))
                y, _ = orc.bitlinear(x, P, N, 1.0, False)
                expect = np.zeros((M, N))
                expect[:, r + j * R] = x[:, k]
                assert np.array_equal(y, expect), (r, j, k)


def test_bitlinear_random_vs_torch(orc):
    """Random ternary codes, packed by the oracle, vs a float64 dense matmul of (code - 1)."""
    M, K, N = 3, 256, 32
    codes = synth.ternary_codes(4, N, K)
    P = orc.pack_ternary(codes)
    x = synth.normal(5, (M, K), 1.0)
    y, mag = orc.bitlinear(x, P, N, 0.75, False)
    wd = torch.from_numpy(codes.astype(np.float64) - 1.0)
    ref = (torch.from_numpy(x).double() @ wd.T).numpy() * 0.75
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(mag, (torch.from_numpy(np.abs(x)).double() @ wd.abs().T).numpy() * 0.75)
    yi, _ = orc.bitlinear(x, P, N, 0.75, True)
    assert np.allclose(yi, ref / 0.75 * float(np.float32(1.0) / np.float32(0.75)), rtol=1e-12)


def test_bitlinear_rejects_ragged_n(orc):
    with pytest.raises(orc.OracleError):
        orc.bitlinear(np.zeros((1, 8), np.float32), np.zeros((1, 8), np.uint8), 6, 1.0, False)


# ------------------------------------------------------------------ int8 / int4

def test_int8_rows_golden(orc):
    (R, Cc), w, q, s = _golden_rows("int8_rows.txt")[0]
    R, Cc = int(R), int(Cc)
    w = np.array([float(v) for v in w], np.float32).reshape(R, Cc)
    got_q, got_s = orc.quantize_int8_rows(w)
    assert np.array_equal(got_q, np.array([int(v) for v in q], np.int8).reshape(R, Cc))
    assert np.array_equal(got_s, np.array([float(v) for v in s], np.float32))


def test_int8_rows_properties(orc):
    w = synth.normal(8, (128, 1000), 0.02)
    w[7] = 0.0
    q, s = orc.quantize_int8_rows(w)
    amax = np.abs(w).max(axis=1)
    nz = amax > 0
    assert np.array_equal(s[nz], (amax[nz] / np.float32(127.0)).astype(np.float32))
    assert s[7] == 1.0 and np.all(q[7] == 0)
    arg = np.abs(w).argmax(axis=1)
    picked = q[np.arange(128), arg]
    assert np.all(np.abs(picked[nz]) == 127)
    assert np.all(np.sign(picked[nz]) == np.sign(w[np.arange(128), arg][nz]))
    err = np.abs(w.astype(np.float64) - q.astype(np.float64) * s[:, None])
    assert np.all(err <= s[:, None] * (0.5 + 2.0 ** -16))


def test_int4_golden_nibbles(orc):
    (K, N), w, packed, s = _golden_rows("int4_nibbles.txt")[0]
    K, N = int(K), int(N)
    w = np.array([float(v) for v in w], np.float32).reshape(K, N)
    P, sc = orc.pack_int4_cols(w)
    assert np.array_equal(P, np.array([int(v, 16) for v in packed], np.uint8).reshape(K // 2, N))
    assert np.array_equal(sc, np.array([float(v) for v in s], np.float32))


def test_int4_properties(orc):
    w = synth.normal(9, (256, 96), 0.02)
    P, s = orc.pack_int4_cols(w)
    hi = (P >> 4).astype(np.int64)
    lo = (P & 15).astype(np.int64)
    c = np.empty((256, 96), np.int64)
    c[0::2] = hi
    c[1::2] = lo
    arg = np.abs(w).argmax(axis=0)
    picked = c[arg, np.arange(96)]
    assert np.all(np.where(w[arg, np.arange(96)] > 0, picked == 15, picked == 1))
    err = np.abs(w.astype(np.float64) - (c - 8) * s[None, :].astype(np.float64))
    assert np.all(err <= s[None, :] * (0.5 + 2.0 ** -16))
    assert c.min() >= 1  # round(w/scale) lies in [-7, 7]


def test_int8_matmul_exact(orc):
    rng = np.random.default_rng(10)
    a = rng.integers(-128, 128, size=(17, 300)).astype(np.int8)
    b = rng.integers(-128, 128, size=(23, 300)).astype(np.int8)
    c = orc.int8_matmul(a, b)
    assert np.array_equal(c.astype(np.int64), a.astype(np.int64) @ b.astype(np.int64).T)


def test_w8a8_vs_float64_library(orc):
    M, K, N = 5, 512, 24
    x = synth.normal(11, (M, K), 1.0)
    w = synth.normal(12, (N, K), 0.02)
    qw, sw = orc.quantize_int8_rows(w)
    lb = synth.normal(13, (N,), 0.01)
    y, mag, qx, sx = orc.w8a8_linear(x, qw, sw, lb)
    qx2, sx2 = orc.quantize_int8_rows(x)
    assert np.array_equal(qx, qx2) and np.array_equal(sx, sx2)
    acc = qx.astype(np.float64) @ qw.astype(np.float64).T
    ref = acc * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64) + lb[None, :]
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)
    # the dequantized product approximates the float product
    assert np.allclose(y - lb, x.astype(np.float64) @ w.astype(np.float64).T, atol=0.05 * np.abs(y).max())


def test_w4a8_matches_w8a8_on_integer_weights(orc):
    """Integer weights in [-7, 7] with a +-7 in every column pack with scale 1,
    so W4A8 must equal W8A8 on the same integers (nibble order and zero point)."""
    rng = np.random.default_rng(14)
    M, K, N = 4, 64, 10
    wint = rng.integers(-7, 8, size=(K, N)).astype(np.float32)
    wint[rng.integers(0, K, size=N), np.arange(N)] = 7.0
    P, s4 = orc.pack_int4_cols(wint)
    assert np.all(s4 == 1.0)
    x = synth.normal(15, (M, K), 1.0)
    y4, m4, qx4, sx4 = orc.w4a8_linear(x, P, s4)
    y8, m8, qx8, sx8 = orc.w8a8_linear(x, wint.T.astype(np.int8), np.ones(N, np.float32))
    assert np.array_equal(y4, y8) and np.array_equal(m4, m8)


def test_quantize_golden_ties(orc):
    """Half steps round to even (hand-computed fixture)."""
    (bits, g), w, codes = _golden_rows("affine_ties.txt")[0]
    bits, g = int(bits), int(g)
    w = np.array([[float(v) for v in w]], np.float32)
    want = np.array([[int(v) for v in codes]], np.uint8)
    for bf16 in (False, True):
        c, s, b = orc.affine_quantize(w, bits, g, bf16)
        assert s[0, 0] == 1.0 and b[0, 0] == 0.0
        assert np.array_equal(orc.unpack(c, g, bits), want)


# ------------------------------------------------------------------ per-group INT8 (pergroup_linear)

def test_int8_groups_properties(orc):
    """Per-group symmetric int8 (the [Q8] rule per group): every group's absmax element maps to
    +-127, a zero group gets scale 1 and zero codes, |w - q s| <= s/2, and the scales sit
    transposed, group-major, as the page's Args give them (scale_w[grp, n])."""
    rng = np.random.default_rng(5)
    N, K, g = 6, 256, 64
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[2, 64:128] = 0.0                                    # a zero group: row 2, group 1
    w[4, 130] = 0.5                                       # group 2 of row 4 dominated by one element
    q, s = orc.quantize_int8_groups(w, g)
    assert s.shape == (K // g, N)
    assert s[1, 2] == 1.0 and not np.any(q[2, 64:128])
    assert s[2, 4] == np.float32(np.float32(0.5) / np.float32(127.0)) and q[4, 130] == 127
    for n in range(N):
        for grp in range(K // g):
            blk = w[n, grp * g:(grp + 1) * g]
            if not np.any(blk):
                continue
            i = int(np.argmax(np.abs(blk)))
            assert abs(int(q[n, grp * g + i])) == 127
            err = np.abs(blk - q[n, grp * g:(grp + 1) * g].astype(np.float64) * s[grp, n])
            assert np.all(err <= s[grp, n] / 2 * (1 + 1e-6))


def test_pergroup_m1_brute_force_exact(orc):
    """M == 1 (FP activation): y[n] = sum_grp s[grp, n] sum_{k in grp} x_k w[n, k] + bias, checked
    exactly with Fractions on dyadic inputs (every product and sum exact in double)."""
    rng = np.random.default_rng(6)
    N, K, g = 5, 128, 64
    w = rng.integers(-128, 128, (N, K)).astype(np.int8)
    s = (2.0 ** rng.integers(-9, -3, (K // g, N))).astype(np.float32)
    x = (rng.integers(-8, 9, (1, K)) / 4.0).astype(np.float32)
    bias = (rng.integers(-4, 5, N) / 8.0).astype(np.float32)
    y, mag, _, _ = orc.pergroup_linear(x, w, s, g, bias)
    for n in range(N):
        want = Fraction(float(bias[n]))
        for grp in range(K // g):
            want += Fraction(float(s[grp, n])) * sum(Fraction(float(x[0, k])) * int(w[n, k])
                                                     for k in range(grp * g, (grp + 1) * g))
        assert Fraction(y[0, n]) == want


def test_pergroup_single_group_equals_w8a8(orc):
    """With one group spanning K, the per-group layer is the per-channel W8A8 layer: M > 1 must give
    exactly the W8A8 result (same quant_a, same scale per output)."""
    rng = np.random.default_rng(7)
    M, N, K = 3, 7, 256
    wf = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    q, s = orc.quantize_int8_groups(wf, 256)
    y, mag, qx, sx = orc.pergroup_linear(x, q, s, 256)
    y8, mag8, qx8, sx8 = orc.w8a8_linear(x, q, s[0], None)
    assert np.array_equal(qx, qx8) and np.array_equal(sx, sx8)
    assert np.allclose(y, y8, rtol=1e-15, atol=0) and np.allclose(mag, mag8, rtol=1e-15, atol=0)


def test_pergroup_m1_vs_float64_library(orc):
    """M == 1 with several groups equals x @ (w * s)^T by torch float64 (the dequantised weight
    built from the transposed scales)."""
    rng = np.random.default_rng(8)
    N, K, g = 33, 512, 128
    wf = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    q, s = orc.quantize_int8_groups(wf, g)
    x = rng.standard_normal((1, K)).astype(np.float32)
    y, _, _, _ = orc.pergroup_linear(x, q, s, g)
    wd = torch.from_numpy(q.astype(np.float64)) * torch.from_numpy(np.repeat(s.T.astype(np.float64), g, axis=1))
    ref = (torch.from_numpy(x.astype(np.float64)) @ wd.T).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_pergroup_dispatch_m1_vs_m2(orc):
    """The page's dispatch: M == 1 uses x as it is, M > 1 its int8 quantisation.  On activations that
    are already on the int8 grid of their row (x = c * amax/127 with integer c) both branches agree;
    on generic activations they differ."""
    rng = np.random.default_rng(9)
    N, K, g = 9, 256, 64
    q, s = orc.quantize_int8_groups((rng.standard_normal((N, K)) * 0.02).astype(np.float32), g)
    c = rng.integers(-127, 128, (1, K)).astype(np.float32)
    c[0, 0] = 127.0
    grid = (c * np.float32(2.0 ** -6)).astype(np.float32)  # amax = 127 / 64, s_x = 1/64 exactly
    y1, _, _, _ = orc.pergroup_linear(grid, q, s, g)
    y2, _, qx, sx = orc.pergroup_linear(np.vstack([grid, grid]), q, s, g)
    assert sx[0] == np.float32(2.0 ** -6) and np.array_equal(qx[0], c[0].astype(np.int8))
    assert np.allclose(y2[0], y1[0], rtol=1e-13, atol=1e-13) and np.allclose(y2[1], y1[0], rtol=1e-13, atol=1e-13)
    xr = rng.standard_normal((1, K)).astype(np.float32)
    r1, _, _, _ = orc.pergroup_linear(xr, q, s, g)
    r2, _, _, _ = orc.pergroup_linear(np.vstack([xr, xr]), q, s, g)
    assert not np.allclose(r1[0], r2[0], rtol=1e-6, atol=0)


# ------------------------------------------------------------------ clip_percentile (quantize_weight_int8)

def test_percentile_linear_equals_numpy(orc):
    """The oracle's percentile (sorting and interpolating in float32) is bit-equal to numpy's
    np.percentile, an independent implementation of the same definition, on random rows of many
    lengths and percentiles, the end points 0 and 100 and the median included."""
    rng = np.random.default_rng(11)
    for trial in range(600):
        n = int(rng.integers(1, 400))
        p = float(rng.choice([0.0, 50.0, 99.0, 99.9, 99.99, 100.0, rng.uniform(0, 100)]))
        v = np.abs(rng.standard_normal(n).astype(np.float32) * np.float32(rng.uniform(1e-3, 1e3)))
        assert orc.percentile_linear(v, p) == float(np.percentile(v, p)), (n, p)


def test_percentile_end_points(orc):
    v = np.array([3.0, 1.0, 2.0, 5.0, 4.0], np.float32)
    assert orc.percentile_linear(v, 0.0) == 1.0 and orc.percentile_linear(v, 100.0) == 5.0
    assert orc.percentile_linear(v, 50.0) == 3.0
    assert orc.percentile_linear(v, 12.5) == 1.5  # h = 4 * 0.125 = 0.5: halfway between 1 and 2


def test_quantize_clip_properties(orc):
    """With a percentile clip: the scale is the clip / 127, elements past the clip saturate at
    +-127, the others follow the absmax rule with that scale; p = 100 is the absmax quantiser
    exactly; a row whose percentile is 0 falls back to its max; an all-zero row gets scale 1."""
    rng = np.random.default_rng(12)
    R, C = 8, 1000
    w = (rng.standard_normal((R, C)) * 0.02).astype(np.float32)
    w[0, :5] = [1.0, -2.0, 1.5, -0.9, 3.0]              # outliers
    w[1, :] = 0.0
    w[1, 7] = 0.25                                      # percentile 0 for p < 99.9 -> max
    w[2, :] = 0.0                                       # all zero
    q, s = orc.quantize_weight_int8_clip(w, 99.0)
    clip = np.array([np.percentile(np.abs(w[r]), 99.0) for r in range(R)], np.float32)
    assert s[1] == np.float32(np.float32(0.25) / np.float32(127.0)) and q[1, 7] == 127
    assert s[2] == 1.0 and not np.any(q[2])
    for r in (0, 3, 4, 5, 6, 7):
        assert s[r] == np.float32(clip[r] / np.float32(127.0))
        over = np.abs(w[r]) >= clip[r]
        assert np.all(np.abs(q[r][over]) == 127)
        inside = ~over
        err = np.abs(w[r][inside] - q[r][inside].astype(np.float64) * s[r])
        assert np.all(err <= s[r] / 2 * (1 + 1e-6))
    q100, s100 = orc.quantize_weight_int8_clip(w, 100.0)
    qa, sa = orc.quantize_int8_rows(w)
    assert np.array_equal(q100, qa) and np.array_equal(s100, sa)



def test_round_f16_equals_numpy(orc):
    """fp16 rounding of the oracle (written from the binary16 format) equals numpy's float32 ->
    float16 conversion on normals, subnormals, ties, the overflow edge and signed zeros."""
    rng = np.random.default_rng(13)
    v = np.concatenate([
        (rng.standard_normal(100000) * np.exp(rng.uniform(-25, 12, 100000))).astype(np.float32),
        np.array([65504, 65519.99, 65520, 65536, -65520, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14,
                  1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 0.0, -0.0, 2.0 ** -26], np.float32)])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).astype(np.float32)
    got = orc.round_f16(v)
    assert np.array_equal(np.signbit(got[np.isfinite(got)]), np.signbit(want[np.isfinite(want)]))
    assert np.array_equal(got, want)
