"""The quantisers' rint(d / s): a multiply by the once-rounded reciprocal, with the IEEE division
done only when the product lies within 1e-4 of a half-integer (k_quant.cu rint_div: distance to
the nearest integer not under 0.4999).  Emulated here in float32 (numpy
rounds every float32 operation once, as the kernel's _rn intrinsics do) and checked against
rint of the float32 quotient on random and adversarial (near half-integer) quotients."""
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "bit_quantized_linear_qmm_b200", "csrc", "k_quant.cu")
f32 = np.float32


def rint_div_emulated(d, s):
    d = d.astype(f32)
    s = s.astype(f32)
    fast = (s >= f32(1.17549435e-38)) & (s <= f32(8.0e37))
    with np.errstate(all="ignore"):
        r = (f32(1) / s).astype(f32)
        m = (d * r).astype(f32)
        t = np.rint(m)
        use_m = fast & (np.abs((m - t).astype(f32)) < f32(0.4999)) & (np.abs(m) < f32(512.0))
        exact = np.rint((d / s).astype(f32))
    return np.where(use_m, t, exact), use_m


def _check(d, s):
    got, used = rint_div_emulated(d, s)
    with np.errstate(all="ignore"):
        want = np.rint((d.astype(f32) / s.astype(f32)).astype(f32))
    assert np.array_equal(got, want)
    return used


def test_constants_match_the_kernel():
    src = open(SRC).read()
    assert "fabsf(__fsub_rn(m, t)) < 0.4999f && fabsf(m) < 512.0f" in src and "const float t = rintf(m);" in src
    assert "return s >= 1.17549435e-38f && s <= 8.0e37f;" in src
    assert "const float m = __fmul_rn(d, r);" in src and "return rintf(__fdiv_rn(d, s));" in src


def test_random_quotients():
    rng = np.random.default_rng(11)
    n = 2_000_000
    s = (10.0 ** rng.uniform(-30, 30, n)).astype(f32)
    q = rng.uniform(-300, 300, n)
    d = (q * s.astype(np.float64)).astype(f32)
    used = _check(d, s)
    assert used.mean() > 0.99  # the division is the rare path


def test_near_half_integers():
    """Quotients a few float32 ulps from k + 0.5, where a second rounding would flip rint."""
    rng = np.random.default_rng(12)
    n = 400_000
    s = (10.0 ** rng.uniform(-20, 20, n)).astype(f32)
    k = rng.integers(-256, 256, n).astype(np.float64) + 0.5
    d0 = (k * s.astype(np.float64)).astype(f32)
    steps = rng.integers(-6, 7, n).astype(np.int32)
    d = (d0.view(np.int32) + steps).view(f32)  # neighbours of k s in float32
    _check(d, s)


def test_quantiser_shaped_inputs():
    """s = amax / 127 (per-token and per-group int8), s = (max - min) / (2^b - 1) (affine), with
    elements at every code boundary of the grid."""
    rng = np.random.default_rng(13)
    for qmax in (7.0, 15.0, 127.0, 255.0, 3.0):
        for _ in range(200):
            amax = f32(10.0 ** rng.uniform(-8, 8))
            s = (amax / f32(qmax)).astype(f32)
            grid = np.arange(-qmax - 1, qmax + 1) + 0.5
            d = (grid * np.float64(s)).astype(f32)
            d = np.concatenate([d, np.nextafter(d, f32(np.inf)), np.nextafter(d, f32(-np.inf)),
                                rng.uniform(-amax, amax, 256).astype(f32)])
            _check(d, np.full_like(d, s))


def test_subnormal_and_extreme_scales_divide():
    s = np.array([1e-40, 1e-45, 1e38, 3e38, 1.0], f32)
    d = np.array([1e-39, 1e-45, 2e38, -3e38, 0.5], f32)
    got, used = rint_div_emulated(d, s)
    assert not used[:4].any()  # outside the normal range of s and 1/s: always the division
    _check(d, s)


def sym_code_emulated(x, amax):
    """k_quant.cu sym_code for one row: s = amax / 127 (or 1), r = 1/s, each rounded once."""
    x = x.astype(f32)
    with np.errstate(all="ignore"):
        s = f32(amax) / f32(127.0)
        s = f32(1.0) if s == 0 else s
        fast = f32(1.17549435e-38) <= s <= f32(8.0e37)
        r = f32(1) / s
        m = (x * r).astype(f32)
        t = np.rint(m)
        use_m = fast & (np.abs((m - t).astype(f32)) < f32(0.4999))
        slow = np.minimum(np.maximum(np.rint((x / s).astype(f32)), f32(-128)), f32(127))
        # fmaxf / fminf return the other operand for a NaN one
        slow = np.where(np.isnan(slow), f32(-128), slow)
    return np.where(use_m, t, slow).astype(np.int64), use_m


def test_sym_code_matches_clamped_division():
    """The multiply path needs no clamp: |x| <= amax keeps every code in [-127, 127]."""
    assert "return (int)t;" in open(SRC).read()
    rng = np.random.default_rng(14)
    for trial in range(3000):
        amax = f32(10.0 ** rng.uniform(-38, 30))
        n = 64
        x = (rng.uniform(-1, 1, n) * np.float64(amax)).astype(f32)
        x[0] = amax
        x[1] = -amax
        x = np.concatenate([x, (np.arange(-127, 128) + 0.5).astype(np.float64).astype(f32) * (amax / f32(127))])
        x = np.clip(x, -amax, amax)
        got, used = sym_code_emulated(x, float(np.max(np.abs(x))))
        s = f32(np.max(np.abs(x))) / f32(127.0)
        s = f32(1.0) if s == 0 else s
        with np.errstate(all="ignore"):
            want = np.clip(np.rint((x / s).astype(f32)), -128, 127).astype(np.int64)
        assert np.array_equal(got, want), trial
        assert np.all(np.abs(got[used]) <= 127)


def test_sym_code_nan_and_subnormal_scale():
    x = np.array([np.nan, 1.0, -1.0], f32)
    got, used = sym_code_emulated(x, 1.0)
    assert got[0] == -128 and not used[0]
    # a subnormal scale (amax / 127 below 2^-126) always divides and clamps
    amax = f32(1e-40)
    assert 0 < f32(amax) / f32(127.0) < f32(1.17549435e-38)
    x = np.array([amax, -amax, 0.0, f32(3e-41)], f32)
    got, used = sym_code_emulated(x, float(amax))
    assert not used.any() and got.min() >= -128 and got.max() <= 127


def test_pack4_byte_order():
    """pack4 = prmt(prmt(a, b, 0x0040), prmt(c, d, 0x0040), 0x5410): code i in byte i."""
    def prmt(a, b, sel):
        src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
        return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))
    assert "prmt(prmt((uint32_t)a, (uint32_t)b, 0x0040u), prmt((uint32_t)c, (uint32_t)d, 0x0040u), 0x5410u)" in \
        open(SRC).read()
    rng = np.random.default_rng(15)
    for _ in range(500):
        c = [int(v) for v in rng.integers(-128, 128, 4)]
        u = [v & 0xFFFFFFFF for v in c]
        w = prmt(prmt(u[0], u[1], 0x0040), prmt(u[2], u[3], 0x0040), 0x5410)
        assert [int(np.int8(np.uint8((w >> (8 * i)) & 0xFF))) for i in range(4)] == c
