"""CPU checks of the bit-level decode steps the kernels use, against plain unpacking.

The GPU kernels turn packed codes into MMA operands with byte permutes (PRMT),
masked ORs into a bf16 exponent pattern (LOP3) and one exact bf16x2 FMA.  These
tests emulate those instructions bit for bit and check, for every code value,
that the result equals what a plain unpacking of the formats gives:

- affine 4-bit, a code pair of one byte -> bf16x2 (q, q'), exactly
  [MLX affine format: LSB-first codes in uint32 words];
- BitLinear 2-bit fields of one byte -> code - 1 for output rows r + j N/4
  [BitLinear packing: code j of byte P[r, k] at bits 2j];
- W4 nibbles -> int8 16 (c - 8), even k from the high nibble
  [packed per-column INT4: zero point 8, high nibble = even k].

The constants are read from the kernel sources, so a change there that these
tests do not follow fails here.
"""
from __future__ import annotations

import os
import struct
from fractions import Fraction

import numpy as np
import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bit_quantized_linear_qmm_b200",
                    "csrc")


def _src(name: str) -> str:
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def prmt(a: int, b: int, sel: int) -> int:
    """PRMT default mode: byte i of the result is byte (sel >> 4i) & 7 of {b, a} (a = bytes 0-3)."""
    bs = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    return sum(bs[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def lop3_and_or(a: int, mask: int, orv: int) -> int:
    return ((a & mask) | orv) & 0xFFFFFFFF


def bf16(h: int) -> Fraction:
    """Exact value of a bf16 bit pattern (finite values only)."""
    f = struct.unpack("<f", struct.pack("<I", (h & 0xFFFF) << 16))[0]
    assert np.isfinite(f)
    return Fraction(f)


def halves(w: int):
    return bf16(w & 0xFFFF), bf16(w >> 16)


def fma_exact_pair(v: int, scale: int, bias: int):
    """bf16x2 FMA v * scale + bias, per half, as exact rationals (the kernels rely on the result
    being exactly representable, so the single rounding of fma.rn leaves it unchanged)."""
    (v0, v1), (s0, s1), (b0, b1) = halves(v), halves(scale), halves(bias)
    return v0 * s0 + b0, v1 * s1 + b1


def exact_in_bf16(x: Fraction) -> bool:
    if x == 0:
        return True
    f = float(x)
    h = struct.unpack("<I", struct.pack("<f", f))[0]
    return Fraction(f) == x and (h & 0xFFFF) == 0


# ---------------------------------------------------------------- affine 4-bit pair -> bf16x2

def f16(h: int) -> Fraction:
    """Exact value of an fp16 bit pattern (finite values only)."""
    f = float(np.frombuffer(struct.pack("<H", h & 0xFFFF), dtype=np.float16)[0])
    assert np.isfinite(f)
    return Fraction(f)


def f16_halves(w: int):
    return f16(w & 0xFFFF), f16(w >> 16)


def test_affine_pair_decode_constants_in_source():
    s = _src("k_tc_affine.cu")
    assert "lop3_and_or(prmt(words[w], w1, sel), 0x0078000Fu, 0x64006400u)" in s
    assert "f16x2_fma(v, 0x30003C00u, 0xD800E400u)" in s
    assert "const uint32_t w1 = words[w] >> 1;" in s
    assert "(uint32_t)(e | (e << 4) | ((4 + e) << 8) | ((4 + e) << 12))" in s


@pytest.mark.parametrize("pos", range(4))
def test_affine_pair_decode_every_byte(pos):
    """One byte of a word of 4-bit codes -> the fp16 pair (1024 + q, 1024 + 8 q') -> (q, q') exactly."""
    rng = np.random.default_rng(pos)
    for byte in range(256):
        others = int(rng.integers(0, 2**32))
        w = (others & ~(0xFF << (8 * pos)) | (byte << (8 * pos))) & 0xFFFFFFFF
        q = [(w >> (4 * i)) & 15 for i in range(8)]  # LSB-first codes k = 0..7
        sel = pos | (pos << 4) | ((4 + pos) << 8) | ((4 + pos) << 12)
        v = lop3_and_or(prmt(w, w >> 1, sel), 0x0078000F, 0x64006400)
        lo, hi = f16_halves(v)
        assert (lo, hi) == (1024 + q[2 * pos], 1024 + 8 * q[2 * pos + 1])
        (s0, s1), (b0, b1) = f16_halves(0x30003C00), f16_halves(0xD800E400)
        a, b = lo * s0 + b0, hi * s1 + b1
        assert (a, b) == (q[2 * pos], q[2 * pos + 1])  # column pos holds k = 2 pos, 2 pos + 1


# ---------------------------------------------------------------- BitLinear 2-bit fields

def test_bitlinear_decode_constants_in_source():
    s = _src("k_bitlinear.cu")
    for c in ("kMagic = 0x43004300u", "kScale0 = 0x3F803F80u, kBias0 = 0xC301C301u",
              "kScale1 = 0x3E803E80u, kBias1 = 0xC204C204u", "kScale2 = 0x3D803D80u, kBias2 = 0xC110C110u",
              "kScale3 = 0x3C803C80u, kBias3 = 0xC040C040u", "kTwo = 0x40004000u",
              "prmt(raw, 0u, 0x0100u)", "prmt(raw, 0u, 0x0302u)",
              "f[0] = bf16x2_fma(lop3_and_or(lo, 0x00030003u, kMagic), kScale0, kBias0)",
              "f[1] = bf16x2_fma(lop3_and_or(lo, 0x00300030u, kMagic), kScale2, kBias2)",
              "f[2] = bf16x2_fma(lop3_and_or(hi, 0x00030003u, kMagic), kScale0, kBias0)",
              "f[3] = bf16x2_fma(lop3_and_or(hi, 0x00300030u, kMagic), kScale2, kBias2)",
              "f[4] = bf16x2_fma(lop3_and_or(lo, 0x000C000Cu, kMagic), kScale1, kBias1)",
              "f[5] = bf16x2_min(bf16x2_fma(lop3_and_or(lo, 0x00C000C0u, kMagic), kScale3, kBias3), kTwo)",
              "f[6] = bf16x2_fma(lop3_and_or(hi, 0x000C000Cu, kMagic), kScale1, kBias1)",
              "f[7] = bf16x2_min(bf16x2_fma(lop3_and_or(hi, 0x00C000C0u, kMagic), kScale3, kBias3), kTwo)"):
        assert c in s, c


def _min2(pair, two=0x40004000):
    t0, t1 = halves(two)
    return min(pair[0], t0), min(pair[1], t1)


def _bitlinear_chunk(word: int):
    """The kernel's decode of one 32-bit word (bytes k .. k+3 of one packed row): field j of byte k
    -> value, as the eight A registers f[0..7] produce them."""
    MAGIC = 0x43004300
    S0, B0, S1, B1, S2, B2 = 0x3F803F80, 0xC301C301, 0x3E803E80, 0xC204C204, 0x3D803D80, 0xC110C110
    S3, B3 = 0x3C803C80, 0xC040C040
    lo = prmt(word, 0, 0x0100)  # bytes k, k+1 in the low byte of each half
    hi = prmt(word, 0, 0x0302)  # bytes k+2, k+3
    out = {}
    out[(0, 0)], out[(0, 1)] = fma_exact_pair(lop3_and_or(lo, 0x00030003, MAGIC), S0, B0)
    out[(2, 0)], out[(2, 1)] = fma_exact_pair(lop3_and_or(lo, 0x00300030, MAGIC), S2, B2)
    out[(0, 2)], out[(0, 3)] = fma_exact_pair(lop3_and_or(hi, 0x00030003, MAGIC), S0, B0)
    out[(2, 2)], out[(2, 3)] = fma_exact_pair(lop3_and_or(hi, 0x00300030, MAGIC), S2, B2)
    out[(1, 0)], out[(1, 1)] = fma_exact_pair(lop3_and_or(lo, 0x000C000C, MAGIC), S1, B1)
    out[(3, 0)], out[(3, 1)] = _min2(fma_exact_pair(lop3_and_or(lo, 0x00C000C0, MAGIC), S3, B3))
    out[(1, 2)], out[(1, 3)] = fma_exact_pair(lop3_and_or(hi, 0x000C000C, MAGIC), S1, B1)
    out[(3, 2)], out[(3, 3)] = _min2(fma_exact_pair(lop3_and_or(hi, 0x00C000C0, MAGIC), S3, B3))
    return out  # (field j, k offset) -> value


def test_bitlinear_field3_pattern():
    """Field 3 sits on the exponent's low bit: codes 0..3 read 128, 192, 256, 384 (not affine),
    the FMA gives -1, 0, 1, 3 and the min with 2 gives code 3 its weight 2."""
    for c in range(4):
        v = lop3_and_or(c << 6, 0x00C000C0, 0x43004300)
        assert halves(v)[0] == [128, 192, 256, 384][c]
        raw = fma_exact_pair(v, 0x3C803C80, 0xC040C040)[0]
        assert raw == [-1, 0, 1, 3][c]
        assert _min2((raw, raw))[0] == (c - 1 if c < 3 else 2)


def test_bitlinear_fields_every_byte():
    rng = np.random.default_rng(3)
    for byte in range(256):
        for pos in range(4):
            word = int(rng.integers(0, 2**32))
            word = (word & ~(0xFF << (8 * pos)) | (byte << (8 * pos))) & 0xFFFFFFFF
            got = _bitlinear_chunk(word)
            for kk in range(4):
                b = (word >> (8 * kk)) & 0xFF
                for j in range(4):
                    code = (b >> (2 * j)) & 3  # output row r + j N/4
                    assert got[(j, kk)] == code - 1, (hex(word), j, kk)
                    assert exact_in_bf16(got[(j, kk)])


# ---------------------------------------------------------------- W4 nibbles -> int8 16 (c - 8)

def test_w4_decode_constants_in_source():
    s = _src("k_gemv.cu")
    assert "^ 0x88888888u" in s and "& 0xF0F0F0F0u" in s and "(x << 4) & 0xF0F0F0F0u" in s
    assert "prmt(hi, lo, 0x5140u)" in s and "prmt(hi, lo, 0x7362u)" in s
    s = _src("k_tc_gemm.cu")
    assert "kHi = 0xF0F0F0F0u, kSign = 0x80808080u" in s
    assert "hi[j] = (w[j] & kHi) ^ kSign;" in s and "lo[j] = ((w[j] << 4) & kHi) ^ kSign;" in s


def test_w4_mn_major_split_every_byte():
    """The GEMM's MN-major operand: a packed word holds four columns of one k-pair row; the
    high nibbles give K row 2i and the low nibbles K row 2i + 1, each byte int8 16 (c - 8)."""
    rng = np.random.default_rng(7)
    for byte in range(256):
        for pos in range(4):
            w = int(rng.integers(0, 2**32))
            w = (w & ~(0xFF << (8 * pos)) | (byte << (8 * pos))) & 0xFFFFFFFF
            hi = (w & 0xF0F0F0F0) ^ 0x80808080
            lo = ((w << 4) & 0xF0F0F0F0) ^ 0x80808080
            for col in range(4):
                b = (w >> (8 * col)) & 0xFF
                assert int(np.int8(np.uint8((hi >> (8 * col)) & 0xFF))) == 16 * ((b >> 4) - 8)
                assert int(np.int8(np.uint8((lo >> (8 * col)) & 0xFF))) == 16 * ((b & 15) - 8)


def test_w4_nibbles_every_byte():
    """A word of four packed bytes (k-pair rows i = 0..3 of one column; high nibble = k = 2i) ->
    two words of int8 16 (c - 8) in k order 0..3 and 4..7."""
    rng = np.random.default_rng(5)
    for byte in range(256):
        for pos in range(4):
            t = int(rng.integers(0, 2**32))
            t = (t & ~(0xFF << (8 * pos)) | (byte << (8 * pos))) & 0xFFFFFFFF
            x = t ^ 0x88888888
            hi = x & 0xF0F0F0F0
            lo = (x << 4) & 0xF0F0F0F0
            o = [prmt(hi, lo, 0x5140), prmt(hi, lo, 0x7362)]
            got = [int(np.int8(np.uint8((o[k // 4] >> (8 * (k % 4))) & 0xFF))) for k in range(8)]
            want = []
            for i in range(4):
                b = (t >> (8 * i)) & 0xFF
                want += [16 * ((b >> 4) - 8), 16 * ((b & 15) - 8)]
            assert got == want, (hex(t), got, want)
