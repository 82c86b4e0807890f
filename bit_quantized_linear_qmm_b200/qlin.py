"""Thin ctypes binding of libqlin.so (the C ABI declared in include/qlin.h).

Argument marshalling only: every step of every operation runs in the CUDA
kernels of libqlin.so.  Tensors are torch CUDA tensors (PyTorch provides the
device memory and the current stream); outputs are allocated here with torch
and filled by the library.  A missing library is an error, never a fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libqlin.so")
HEADER = os.path.join(ROOT, "include", "qlin.h")

QLIN_OK = 0
QLIN_ERR_INVALID_ARG = 1
QLIN_ERR_UNSUPPORTED = 2
QLIN_ERR_MISALIGNED = 3
QLIN_ERR_DEVICE = 4
QLIN_ERR_CUDA = 5
QLIN_ERR_TIMEOUT = 6
QLIN_ERR_WORKSPACE = 7

QLIN_F32 = 0
QLIN_BF16 = 1
QLIN_F16 = 2

QLIN_OP_MATMUL = 0
QLIN_OP_BITLINEAR = 1
QLIN_OP_W8A8 = 2
QLIN_OP_W4A8 = 3
QLIN_OP_PERGROUP = 4

_lib = None


class QlinError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def header_functions() -> list[str]:
    """Names of the functions include/qlin.h declares."""
    text = open(HEADER).read()
    return re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\*?\s+\*?(qlin_\w+|bitlinear_\w+|w8a8_\w+|w4a8_\w+|pergroup_\w+)\s*\(",
                      text, re.M)


def lib():
    """Load libqlin.so (building nothing: call bit_quantized_linear_qmm_b200.build first)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libqlin.so not found at {LIB_PATH}; run `python -m bit_quantized_linear_qmm_b200.build`")
    L = C.CDLL(LIB_PATH)
    P, I64, I, SZ = C.c_void_p, C.c_int64, C.c_int, C.c_size_t
    sig = {
        "qlin_status_string": ([I], C.c_char_p),
        "qlin_version": ([], I),
        "qlin_workspace_size": ([I, I64, I64, I64, I, I], SZ),
        "qlin_int8_gemm_tile": ([I, I64, I64, I, P, P], I),
        "qlin_quantize": ([P, I, I64, I64, I, I, P, P, P, I, P], I),
        "qlin_dequantize": ([P, P, P, I, I64, I64, I, I, P, I, P], I),
        "qlin_matmul": ([P, I, I64, I64, P, P, P, I, I64, I, I, P, P, P, SZ, P], I),
        "bitlinear_matmul": ([P, I, I64, I64, P, I64, P, I, P, P, P], I),
        "qlin_quantize_int8_rows": ([P, I, I64, I64, P, P, P], I),
        "qlin_pack_int4_cols": ([P, I, I64, I64, P, P, P], I),
        "qlin_int8_matmul_int32": ([P, P, I64, I64, I64, P, P], I),
        "w8a8_linear": ([P, I, I64, I64, P, P, I64, P, P, P, SZ, P], I),
        "w4a8_linear": ([P, I, I64, I64, P, P, I64, P, P, P, SZ, P], I),
        "w8a8_linear_noalloc": ([P, I, I64, I64, P, P, I64, P, P, P], I),
        "qlin_quantize_int8_groups": ([P, I, I64, I64, I, P, P, P], I),
        "qlin_quantize_weight_int8": ([P, I, I64, I64, C.c_double, P, P, P], I),
        "pergroup_linear": ([P, I, I64, I64, P, P, I64, I, P, P, P, SZ, P], I),
        "qlin_get_device_status": ([P], I),
        "qlin_selftest_wait_timeout": ([C.c_uint, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def status_string(s: int) -> str:
    return lib().qlin_status_string(int(s)).decode()


def _check(status: int, what: str):
    if status != QLIN_OK:
        raise QlinError(status, what)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(device=None):
    return C.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return QLIN_F32
    if t.dtype == torch.bfloat16:
        return QLIN_BF16
    if t.dtype == torch.float16:
        return QLIN_F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _torch_dt(code: int):
    return {QLIN_F32: torch.float32, QLIN_BF16: torch.bfloat16, QLIN_F16: torch.float16}[code]


def _cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("qlin operates on CUDA tensors only")
            if not t.is_contiguous():
                raise ValueError("qlin expects contiguous tensors")


def workspace_size(op: int, M: int, N: int, K: int, bits: int = 0, group_size: int = 0) -> int:
    return int(lib().qlin_workspace_size(op, M, N, K, bits, group_size))


def int8_gemm_tile(op: int, M: int, N: int, sm_count: int) -> tuple[int, int]:
    """(tokens, columns) of the int8 tensor-core GEMM's CTA tile for an M x N output."""
    t, c = C.c_int(0), C.c_int(0)
    _check(lib().qlin_int8_gemm_tile(op, M, N, sm_count, C.byref(t), C.byref(c)), "qlin_int8_gemm_tile")
    return t.value, c.value


def quantize(w: torch.Tensor, bits: int, group_size: int, param_dtype=torch.bfloat16):
    """Affine group quantisation -> (codes uint32-as-int32 [N, K*bits/32], scales, biases [N, K/g])."""
    _cuda(w)
    N, K = w.shape
    codes = torch.empty((N, K * bits // 32), dtype=torch.int32, device=w.device)
    G = K // group_size if group_size else 0
    scales = torch.empty((N, G), dtype=param_dtype, device=w.device)
    biases = torch.empty((N, G), dtype=param_dtype, device=w.device)
    _check(lib().qlin_quantize(_ptr(w), _dt(w), N, K, bits, group_size, _ptr(codes), _ptr(scales), _ptr(biases),
                               _dt(scales), _stream(w.device)), "qlin_quantize")
    return codes, scales, biases


def dequantize(codes, scales, biases, K: int, bits: int, group_size: int, out_dtype=torch.bfloat16):
    _cuda(codes, scales, biases)
    N = codes.shape[0]
    out = torch.empty((N, K), dtype=out_dtype, device=codes.device)
    _check(lib().qlin_dequantize(_ptr(codes), _ptr(scales), _ptr(biases), _dt(scales), N, K, bits, group_size,
                                 _ptr(out), _dt(out), _stream(codes.device)), "qlin_dequantize")
    return out


def matmul(x, codes, scales, biases, bits: int, group_size: int, bias=None, out=None, workspace=None):
    """y = x @ dequant(codes, scales, biases)^T + bias, y in x's dtype."""
    _cuda(x, codes, scales, biases, bias)
    M, K = x.shape
    N = codes.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    ws = workspace_size(QLIN_OP_MATMUL, M, N, K, bits, group_size)
    if ws and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=x.device)
    _check(lib().qlin_matmul(_ptr(x), _dt(x), M, K, _ptr(codes), _ptr(scales), _ptr(biases), _dt(scales), N, bits,
                             group_size, _ptr(bias), _ptr(out), _ptr(workspace),
                             0 if workspace is None else workspace.numel(), _stream(x.device)), "qlin_matmul")
    return out


def bitlinear_matmul(x, packed, N: int, weight_scale, invert: bool, bias=None, out=None):
    """BitLinear ternary layer; weight_scale is a 1-element fp32 CUDA tensor."""
    _cuda(x, packed, weight_scale, bias)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    _check(lib().bitlinear_matmul(_ptr(x), _dt(x), M, K, _ptr(packed), N, _ptr(weight_scale), int(bool(invert)),
                                  _ptr(bias), _ptr(out), _stream(x.device)), "bitlinear_matmul")
    return out


def quantize_int8_rows(w):
    _cuda(w)
    R, Cc = w.shape
    q = torch.empty((R, Cc), dtype=torch.int8, device=w.device)
    s = torch.empty((R,), dtype=torch.float32, device=w.device)
    _check(lib().qlin_quantize_int8_rows(_ptr(w), _dt(w), R, Cc, _ptr(q), _ptr(s), _stream(w.device)),
           "qlin_quantize_int8_rows")
    return q, s


def pack_int4_cols(w):
    _cuda(w)
    K, N = w.shape
    P = torch.empty((K // 2, N), dtype=torch.uint8, device=w.device)
    s = torch.empty((N,), dtype=torch.float32, device=w.device)
    _check(lib().qlin_pack_int4_cols(_ptr(w), _dt(w), K, N, _ptr(P), _ptr(s), _stream(w.device)),
           "qlin_pack_int4_cols")
    return P, s


def int8_matmul_int32(a, b, out=None):
    _cuda(a, b)
    M, K = a.shape
    N = b.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32, device=a.device)
    _check(lib().qlin_int8_matmul_int32(_ptr(a), _ptr(b), M, N, K, _ptr(out), _stream(a.device)),
           "qlin_int8_matmul_int32")
    return out


def w8a8_linear(x, w, scale_w, bias=None, out=None, workspace=None):
    _cuda(x, w, scale_w, bias)
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = torch.empty(workspace_size(QLIN_OP_W8A8, M, N, K), dtype=torch.uint8, device=x.device)
    _check(lib().w8a8_linear(_ptr(x), _dt(x), M, K, _ptr(w), _ptr(scale_w), N, _ptr(bias), _ptr(out),
                             _ptr(workspace), workspace.numel(), _stream(x.device)), "w8a8_linear")
    return out


def w4a8_linear(x, packed_w, scale_w, bias=None, out=None, workspace=None):
    _cuda(x, packed_w, scale_w, bias)
    M, K = x.shape
    N = packed_w.shape[1]
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = torch.empty(workspace_size(QLIN_OP_W4A8, M, N, K), dtype=torch.uint8, device=x.device)
    _check(lib().w4a8_linear(_ptr(x), _dt(x), M, K, _ptr(packed_w), _ptr(scale_w), N, _ptr(bias), _ptr(out),
                             _ptr(workspace), workspace.numel(), _stream(x.device)), "w4a8_linear")
    return out


def w8a8_linear_noalloc(x, w, scale_w, bias=None, out=None):
    """w8a8_linear with the activation scratch inside the library (no workspace)."""
    _cuda(x, w, scale_w, bias)
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    _check(lib().w8a8_linear_noalloc(_ptr(x), _dt(x), M, K, _ptr(w), _ptr(scale_w), N, _ptr(bias), _ptr(out),
                                     _stream(x.device)), "w8a8_linear_noalloc")
    return out


def selftest_wait_timeout(limit_us: int = 1000, device=None):
    """Queues a kernel whose bounded wait runs out after limit_us (see qlin.h)."""
    _check(lib().qlin_selftest_wait_timeout(int(limit_us), _stream(device)), "qlin_selftest_wait_timeout")


def device_status(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device status."""
    return int(lib().qlin_get_device_status(_stream(device)))


def quantize_int8_groups(w, group_size: int):
    """Per-group symmetric int8 weights: (q int8 [N, K], scale_w fp32 [K/group_size, N])."""
    _cuda(w)
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.int8, device=w.device)
    s = torch.empty((K // group_size, N), dtype=torch.float32, device=w.device)
    _check(lib().qlin_quantize_int8_groups(_ptr(w), _dt(w), N, K, group_size, _ptr(q), _ptr(s), _stream(w.device)),
           "qlin_quantize_int8_groups")
    return q, s


def pergroup_linear(x, w, scale_w, group_size: int, bias=None, out=None, workspace=None):
    """Per-group INT8 linear (M == 1: FP activation; M > 1: int8 activation quantisation)."""
    _cuda(x, w, scale_w, bias)
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = torch.empty(workspace_size(QLIN_OP_PERGROUP, M, N, K, 8, group_size), dtype=torch.uint8,
                                device=x.device)
    _check(lib().pergroup_linear(_ptr(x), _dt(x), M, K, _ptr(w), _ptr(scale_w), N, group_size, _ptr(bias), _ptr(out),
                                 _ptr(workspace), workspace.numel(), _stream(x.device)), "pergroup_linear")
    return out


def quantize_weight_int8(w, clip_percentile=None):
    """Per-row int8 weights, optionally clipped at a per-row percentile of |w|: (q [R, C], scale [R])."""
    _cuda(w)
    R, Cc = w.shape
    q = torch.empty((R, Cc), dtype=torch.int8, device=w.device)
    s = torch.empty((R,), dtype=torch.float32, device=w.device)
    p = -1.0 if clip_percentile is None else float(clip_percentile)
    _check(lib().qlin_quantize_weight_int8(_ptr(w), _dt(w), R, Cc, p, _ptr(q), _ptr(s), _stream(w.device)),
           "qlin_quantize_weight_int8")
    return q, s
