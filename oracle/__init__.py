"""CPU oracle for the quantized linear layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library's product path never does;
it shares no code with the CUDA library (see ``oracle.c`` for the sources each
routine follows and the readings taken where the pages are silent).

This module only marshals numpy arrays into the plain C routines of
``oracle.c`` (built with gcc into ``liboracle.so`` beside it).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, no fast-math, no fp contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-std=c11",
            "-shared", "-fPIC", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # ORACLE_SO_OVERRIDE points the mutation tests at a deliberately broken
        # build of oracle.c; it is never set outside those tests.
        path = os.environ.get("ORACLE_SO_OVERRIDE")
        if not path:
            path = build()
        lib = C.CDLL(path)
        P = C.c_void_p
        I64 = C.c_int64
        lib.orc_pack.argtypes = [P, I64, I64, C.c_int, P]
        lib.orc_unpack.argtypes = [P, I64, I64, C.c_int, P]
        lib.orc_affine_quantize.argtypes = [P, I64, I64, C.c_int, C.c_int, C.c_int, P, P, P]
        lib.orc_affine_dequantize.argtypes = [P, P, P, I64, I64, C.c_int, C.c_int, P]
        lib.orc_affine_matmul.argtypes = [P, I64, I64, P, P, P, I64, C.c_int, C.c_int, P, P, P]
        lib.orc_pack_ternary.argtypes = [P, I64, I64, P]
        lib.orc_bitlinear.argtypes = [P, I64, I64, P, I64, C.c_float, C.c_int, P, P, P]
        lib.orc_quantize_int8_rows.argtypes = [P, I64, I64, P, P]
        lib.orc_pack_int4_cols.argtypes = [P, I64, I64, P, P]
        lib.orc_int8_matmul.argtypes = [P, P, I64, I64, I64, P]
        lib.orc_w8a8_linear.argtypes = [P, I64, I64, P, P, I64, P, P, P, P, P]
        lib.orc_w4a8_linear.argtypes = [P, I64, I64, P, P, I64, P, P, P, P, P]
        lib.orc_quantize_int8_groups.argtypes = [P, I64, I64, C.c_int, P, P]
        lib.orc_percentile_linear.argtypes = [P, I64, C.c_double]
        lib.orc_percentile_linear.restype = C.c_float
        lib.orc_quantize_weight_int8_clip.argtypes = [P, I64, I64, C.c_double, P, P]
        lib.orc_pergroup_linear.argtypes = [P, I64, I64, P, P, I64, C.c_int, P, P, P, P, P]
        lib.orc_f32_to_bf16.argtypes = [P, I64, P]
        lib.orc_round_f16_array.argtypes = [P, I64, P]
        lib.orc_bf16_to_f32.argtypes = [P, I64, P]
        for name in ("orc_pack", "orc_unpack", "orc_affine_quantize", "orc_affine_dequantize",
                     "orc_affine_matmul", "orc_pack_ternary", "orc_bitlinear",
                     "orc_quantize_int8_rows", "orc_pack_int4_cols", "orc_int8_matmul",
                     "orc_w8a8_linear", "orc_w4a8_linear"):
            getattr(lib, name).restype = C.c_int
        lib.orc_f32_to_bf16.restype = None
        lib.orc_bf16_to_f32.restype = None
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc == -2:
        raise OracleError(f"{what}: int32 accumulator overflow")
    if rc != 0:
        raise OracleError(f"{what}: invalid argument (rc={rc})")


# ---------------------------------------------------------------- bf16

def f32_to_bf16_bits(a) -> np.ndarray:
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().orc_f32_to_bf16(_p(a), a.size, _p(out))
    return out


def bf16_bits_to_f32(h) -> np.ndarray:
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    _load().orc_bf16_to_f32(_p(h), h.size, _p(out))
    return out


# ---------------------------------------------------------------- affine format

def pack(q, bits: int) -> np.ndarray:
    q = _c(q, np.uint8)
    N, K = q.shape
    out = np.empty((N, K * bits // 32), np.uint32)
    _check(_load().orc_pack(_p(q), N, K, bits, _p(out)), "pack")
    return out


def unpack(packed, K: int, bits: int) -> np.ndarray:
    packed = _c(packed, np.uint32)
    N = packed.shape[0]
    q = np.empty((N, K), np.uint8)
    _check(_load().orc_unpack(_p(packed), N, K, bits, _p(q)), "unpack")
    return q


def affine_quantize(w, bits: int, group_size: int, bf16_params):
    """Returns (codes uint32 [N,K*b/32], scales f32 [N,K/g], biases f32 [N,K/g]).

    ``bf16_params``: False / "f32" stores fp32 scales/biases; True / "bf16" bf16 values, "f16"
    fp16 values (both held exactly in f32).
    """
    if isinstance(bf16_params, str):
        bf16_params = {"f32": 0, "bf16": 1, "f16": 2}[bf16_params]
    w = _c(w, np.float32)
    N, K = w.shape
    if K % group_size:
        raise OracleError("affine_quantize: K % group_size != 0")
    codes = np.empty((N, K * bits // 32), np.uint32)
    G = K // group_size
    scales = np.empty((N, G), np.float32)
    biases = np.empty((N, G), np.float32)
    _check(_load().orc_affine_quantize(_p(w), N, K, bits, group_size, int(bf16_params),
                                       _p(codes), _p(scales), _p(biases)), "affine_quantize")
    return codes, scales, biases


def affine_dequantize(codes, scales, biases, K: int, bits: int, group_size: int) -> np.ndarray:
    codes = _c(codes, np.uint32)
    scales = _c(scales, np.float32)
    biases = _c(biases, np.float32)
    N = codes.shape[0]
    out = np.empty((N, K), np.float32)
    _check(_load().orc_affine_dequantize(_p(codes), _p(scales), _p(biases), N, K, bits,
                                         group_size, _p(out)), "affine_dequantize")
    return out


def affine_matmul(x, codes, scales, biases, bits: int, group_size: int, bias=None):
    """Returns (y float64 [M,N] unrounded, absdot float64 [M,N])."""
    x = _c(x, np.float32)
    M, K = x.shape
    codes = _c(codes, np.uint32)
    scales = _c(scales, np.float32)
    biases = _c(biases, np.float32)
    N = codes.shape[0]
    bias = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    mag = np.empty((M, N), np.float64)
    _check(_load().orc_affine_matmul(_p(x), M, K, _p(codes), _p(scales), _p(biases), N, bits,
                                     group_size, _p(bias), _p(y), _p(mag)), "affine_matmul")
    return y, mag


# ---------------------------------------------------------------- BitLinear

def pack_ternary(codes) -> np.ndarray:
    codes = _c(codes, np.uint8)
    N, K = codes.shape
    P = np.empty((N // 4, K), np.uint8)
    _check(_load().orc_pack_ternary(_p(codes), N, K, _p(P)), "pack_ternary")
    return P


def bitlinear(x, P, N: int, weight_scale: float, invert: bool, bias=None):
    x = _c(x, np.float32)
    M, K = x.shape
    P = _c(P, np.uint8)
    bias = None if bias is None else _c(bias, np.float32)
    y = np.empty((M, N), np.float64)
    mag = np.empty((M, N), np.float64)
    _check(_load().orc_bitlinear(_p(x), M, K, _p(P), N, float(np.float32(weight_scale)),
                                 int(invert), _p(bias), _p(y), _p(mag)), "bitlinear")
    return y, mag


# ---------------------------------------------------------------- int8 / int4

def quantize_int8_rows(w):
    w = _c(w, np.float32)
    R, Cc = w.shape
    q = np.empty((R, Cc), np.int8)
    s = np.empty((R,), np.float32)
    _check(_load().orc_quantize_int8_rows(_p(w), R, Cc, _p(q), _p(s)), "quantize_int8_rows")
    return q, s


def pack_int4_cols(w):
    w = _c(w, np.float32)
    K, N = w.shape
    P = np.empty((K // 2, N), np.uint8)
    s = np.empty((N,), np.float32)
    _check(_load().orc_pack_int4_cols(_p(w), K, N, _p(P), _p(s)), "pack_int4_cols")
    return P, s


def int8_matmul(a, b) -> np.ndarray:
    a = _c(a, np.int8)
    b = _c(b, np.int8)
    M, K = a.shape
    N = b.shape[0]
    c = np.empty((M, N), np.int32)
    _check(_load().orc_int8_matmul(_p(a), _p(b), M, N, K, _p(c)), "int8_matmul")
    return c


def w8a8_linear(x, w, scale_w, bias=None):
    """Returns (y, absdot, qx, s_x)."""
    x = _c(x, np.float32)
    M, K = x.shape
    w = _c(w, np.int8)
    N = w.shape[0]
    scale_w = _c(scale_w, np.float32)
    bias = None if bias is None else _c(bias, np.float32)
    qx = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    y = np.empty((M, N), np.float64)
    mag = np.empty((M, N), np.float64)
    _check(_load().orc_w8a8_linear(_p(x), M, K, _p(w), _p(scale_w), N, _p(bias), _p(qx), _p(sx),
                                   _p(y), _p(mag)), "w8a8_linear")
    return y, mag, qx, sx


def w4a8_linear(x, P, scale_w, bias=None):
    """Returns (y, absdot, qx, s_x)."""
    x = _c(x, np.float32)
    M, K = x.shape
    P = _c(P, np.uint8)
    N = P.shape[1]
    scale_w = _c(scale_w, np.float32)
    bias = None if bias is None else _c(bias, np.float32)
    qx = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    y = np.empty((M, N), np.float64)
    mag = np.empty((M, N), np.float64)
    _check(_load().orc_w4a8_linear(_p(x), M, K, _p(P), _p(scale_w), N, _p(bias), _p(qx), _p(sx),
                                   _p(y), _p(mag)), "w4a8_linear")
    return y, mag, qx, sx


def quantize_int8_groups(w, g: int):
    """Per-group symmetric int8 weights: returns (q int8 [N, K], scale_w fp32 [K/g, N])."""
    w = _c(w, np.float32)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    scale_w = np.empty((K // g, N), np.float32)
    _check(_load().orc_quantize_int8_groups(_p(w), N, K, g, _p(q), _p(scale_w)), "quantize_int8_groups")
    return q, scale_w


def pergroup_linear(x, w, scale_w, g: int, bias=None):
    """Per-group INT8 linear with the page's M == 1 / M > 1 dispatch.
    Returns (y, absdot, qx, s_x) (qx, s_x meaningful for M > 1 only)."""
    x = _c(x, np.float32)
    M, K = x.shape
    w = _c(w, np.int8)
    N = w.shape[0]
    scale_w = _c(scale_w, np.float32)
    bias = None if bias is None else _c(bias, np.float32)
    qx = np.zeros((M, K), np.int8)
    sx = np.zeros((M,), np.float32)
    y = np.empty((M, N), np.float64)
    mag = np.empty((M, N), np.float64)
    _check(_load().orc_pergroup_linear(_p(x), M, K, _p(w), _p(scale_w), N, g, _p(bias), _p(qx), _p(sx),
                                       _p(y), _p(mag)), "pergroup_linear")
    return y, mag, qx, sx


def percentile_linear(v, p: float) -> float:
    """The p-th percentile of a float32 vector, linear interpolation in float32 arithmetic."""
    v = _c(v, np.float32).ravel()
    return float(np.float32(_load().orc_percentile_linear(_p(v), v.size, float(p))))


def quantize_weight_int8_clip(w, clip_percentile: float):
    """Per-row int8 with a percentile clip: returns (q int8 [R, C], scale fp32 [R])."""
    w = _c(w, np.float32)
    R, Cc = w.shape
    q = np.empty((R, Cc), np.int8)
    s = np.empty((R,), np.float32)
    _check(_load().orc_quantize_weight_int8_clip(_p(w), R, Cc, float(clip_percentile), _p(q), _p(s)),
           "quantize_weight_int8_clip")
    return q, s


def round_f16(v) -> np.ndarray:
    """Values rounded to the nearest binary16 (ties to even), as fp32."""
    v = _c(v, np.float32)
    out = np.empty_like(v)
    _load().orc_round_f16_array(_p(v), v.size, _p(out))
    return out
