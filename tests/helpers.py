"""Shared helpers for the GPU parity tests (the tolerance, device transfer)."""
from __future__ import annotations

import numpy as np
import torch

# Floating-point bar: |y - y_ref| <= REL * (sum_k |x_k w_k| + |bias_n|) + ABS + half an ulp of y in
# the output dtype, with y_ref the oracle's unrounded double result.  REL and ABS bound the
# computation (fp32 accumulation of the products); the half ulp is the one rounding of y to the
# I/O dtype, which no bf16 output can avoid: 2^-8 |y| exceeds REL * sum_k |x_k w_k| whenever
# |y| > 0.51 sum_k |x_k w_k| (few terms of one sign).  The |bias| term covers a bias-dominated
# output.
REL = 2e-3
ABS = 1e-5


def half_ulp(v: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Half a unit in the last place of |v| in `dtype` (bf16: 8 significant bits, fp16: 11 with
    subnormal spacing 2^-24, fp32: 24)."""
    bits = {torch.bfloat16: 8, torch.float16: 11}.get(dtype, 24)
    a = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(a)  # a = f 2^e, f in [0.5, 1)
    if dtype == torch.float16:
        e = np.maximum(e, -13)  # below 2^-14 the spacing stays 2^-24
    return np.where(a > 0, np.ldexp(1.0, e - 1 - bits), 0.0)


def build_lib():
    from bit_quantized_linear_qmm_b200 import build
    build.build()
    from bit_quantized_linear_qmm_b200 import qlin
    return qlin


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def u32_dev(a: np.ndarray) -> torch.Tensor:
    """uint32 numpy -> int32 CUDA tensor with the same bytes."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).cuda()


def bf16_dev_from_f32_values(v: np.ndarray) -> torch.Tensor:
    """fp32 values that are exactly bf16 -> bf16 CUDA tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16).cuda()


def params_dev(vals: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return bf16_dev_from_f32_values(vals)
    if dtype == "f16":  # fp32 values that are exactly fp16
        return torch.from_numpy(np.ascontiguousarray(vals, np.float32).astype(np.float16)).cuda()
    return to_dev(vals.astype(np.float32))


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float32)


def host_bits16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def assert_fp_close(y_gpu: torch.Tensor, y_ref: np.ndarray, absdot: np.ndarray, bias=None, what=""):
    y = y_gpu.double().cpu().numpy()
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    scale = absdot.copy()
    if bias is not None:
        scale = scale + np.abs(np.asarray(bias, np.float64))[None, :]
    tol = REL * scale + ABS + half_ulp(np.maximum(np.abs(y), np.abs(y_ref)), y_gpu.dtype)
    err = np.abs(y - y_ref)
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)[:5]
        worst = float((err / tol).max())
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside tolerance (worst err/tol {worst:.3g}); "
            f"first {[(tuple(i), float(y[tuple(i)]), float(y_ref[tuple(i)])) for i in idx]}")
    return float((err / tol).max())
