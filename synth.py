"""Seeded synthetic inputs for the quantized linear layer.

This module only draws random numbers and rounds them to the storage dtype;
it holds none of the layer's arithmetic (no quantisation, packing or
product).  Both the CUDA library's tests/benchmark and the CPU oracle take
their inputs from here, so the two sides see the same bytes.

Distributions follow the workloads the layer is used for (LLM linear layers):
activations ~ N(0, 1), weights ~ N(0, 0.02), layer bias ~ N(0, 0.01).  Each
tensor of a case has its own seed: weights ``seed``, activations ``seed+1``,
bias ``seed+2`` (and ``seed+3`` for the outlier positions of the prefill
weights).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def normal(seed: int, shape, sigma: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma)).astype(np.float32)


def to_bf16(a: np.ndarray):
    """Round fp32 -> bf16 (round to nearest even, via torch on the CPU).

    Returns (values as fp32, raw bf16 bits as uint16)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16).copy()
    vals = t.to(torch.float32).numpy().copy()
    return vals, bits


def to_f16(a: np.ndarray):
    """Round fp32 -> IEEE binary16 (round to nearest even, numpy's conversion).

    Returns (values as fp32, raw fp16 bits as uint16)."""
    h = np.ascontiguousarray(a, dtype=np.float32).astype(np.float16)
    return h.astype(np.float32), h.view(np.uint16).copy()


def outlier_weights(seed: int, N: int, K: int, sigma: float = 0.02,
                    frac: float = 0.001, factor: float = 20.0) -> np.ndarray:
    """N(0, sigma) weights with round(frac*N*K) positions, drawn uniformly
    without replacement, multiplied by ``factor``."""
    w = normal(seed, (N, K), sigma)
    count = int(round(frac * N * K))
    rng = np.random.default_rng(seed + 3)
    pos = rng.choice(N * K, size=count, replace=False)
    flat = w.reshape(-1)
    flat[pos] *= np.float32(factor)
    return w


# The 81 byte values whose four 2-bit fields all lie in {0, 1, 2}: drawing
# uniformly from them makes every field an independent uniform draw from
# {0, 1, 2}, i.e. a random ternary weight for each of the four output rows a
# byte serves.
_TERNARY_BYTES = np.array(
    [v for v in range(256) if all(((v >> (2 * j)) & 3) < 3 for j in range(4))], dtype=np.uint8)


def ternary_bytes(seed: int, rows: int, K: int) -> np.ndarray:
    """uint8 [rows, K], each 2-bit field uniform in {0, 1, 2}."""
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, len(_TERNARY_BYTES), size=(rows, K))
    return _TERNARY_BYTES[idx]


def any_bytes(seed: int, rows: int, K: int) -> np.ndarray:
    """uint8 [rows, K] uniform over all 256 values (2-bit fields 0..3, code 3 included)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 256, size=(rows, K)).astype(np.uint8)


def random_words(seed: int, shape) -> np.ndarray:
    """uint32 words with every bit uniform (packed codes of any width, drawn directly)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 2**32, size=shape, dtype=np.uint32)


def ternary_codes(seed: int, N: int, K: int) -> np.ndarray:
    """uint8 [N, K] codes uniform in {0, 1, 2} (unpacked form)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 3, size=(N, K)).astype(np.uint8)


@dataclass
class Activations:
    vals: np.ndarray            # fp32 values (exactly representable in `dtype`)
    bits: np.ndarray | None     # uint16 bf16 / fp16 bits when dtype is "bf16" / "f16"
    dtype: str

    def torch(self, device="cpu"):
        if self.dtype == "bf16":
            t = torch.from_numpy(self.bits.view(np.int16)).view(torch.bfloat16)
        elif self.dtype == "f16":
            t = torch.from_numpy(self.bits.view(np.int16)).view(torch.float16)
        else:
            t = torch.from_numpy(self.vals)
        return t.to(device)


def activations(seed: int, shape, dtype: str, sigma: float = 1.0) -> Activations:
    v = normal(seed, shape, sigma)
    if dtype == "bf16":
        vals, bits = to_bf16(v)
        return Activations(vals, bits, "bf16")
    if dtype == "f16":
        vals, bits = to_f16(v)
        return Activations(vals, bits, "f16")
    if dtype == "f32":
        return Activations(v, None, "f32")
    raise ValueError(dtype)


# ---------------------------------------------------------------- workloads

@dataclass
class AffineCase:
    """MLX-affine quantized linear: x [M,K], weight [N,K] quantized in groups."""
    name: str
    M: int
    K: int
    N: int
    bits: int
    group_size: int
    x_dtype: str        # "f32" | "bf16" | "f16" (output and bias use the same dtype)
    param_dtype: str    # "f32" | "bf16" | "f16" (scales, biases)
    bias: bool = True
    outliers: bool = False
    seed: int = 0

    def weight(self) -> np.ndarray:
        if self.outliers:
            return outlier_weights(self.seed, self.N, self.K)
        return normal(self.seed, (self.N, self.K), 0.02)

    def x(self) -> Activations:
        return activations(self.seed + 1, (self.M, self.K), self.x_dtype)

    def layer_bias(self) -> Activations | None:
        if not self.bias:
            return None
        return activations(self.seed + 2, (self.N,), self.x_dtype, 0.01)


@dataclass
class BitLinearCase:
    name: str
    M: int
    K: int
    N: int
    weight_scale: float = 0.5
    invert: bool = False
    bias: bool = False
    x_dtype: str = "bf16"
    seed: int = 0
    all_bytes: bool = False  # fields uniform in 0..3 (code 3 included) instead of {0, 1, 2}

    def packed(self) -> np.ndarray:
        if self.all_bytes:
            return any_bytes(self.seed, self.N // 4, self.K)
        return ternary_bytes(self.seed, self.N // 4, self.K)

    def x(self) -> Activations:
        return activations(self.seed + 1, (self.M, self.K), self.x_dtype)

    def layer_bias(self) -> Activations | None:
        if not self.bias:
            return None
        return activations(self.seed + 2, (self.N,), self.x_dtype, 0.01)


@dataclass
class IntCase:
    """W8A8 / W4A8: weight ~ N(0, 0.02) [N, K] (W4 quantizes its transpose [K, N])."""
    name: str
    M: int
    K: int
    N: int
    bias: bool = False
    x_dtype: str = "bf16"
    seed: int = 0

    def weight(self) -> np.ndarray:
        return normal(self.seed, (self.N, self.K), 0.02)

    def x(self) -> Activations:
        return activations(self.seed + 1, (self.M, self.K), self.x_dtype)

    def layer_bias(self) -> Activations | None:
        if not self.bias:
            return None
        return activations(self.seed + 2, (self.N,), self.x_dtype, 0.01)


# Case 1: small MLX-affine layer (4-bit, group 64, fp32 x / params, with bias).
AFFINE_SMALL = AffineCase("affine_b4_g64_M4_K512_N512_f32", 4, 512, 512, 4, 64, "f32", "f32", True)

# Case 2: BitLinear ternary decode, K = N = 4096, M in {1, 8}, both scale modes.
BITLINEAR_DECODE = [BitLinearCase(f"bitlinear_M{M}_K4096_N4096_{'div' if inv else 'mul'}", M, 4096, 4096,
                                  0.5, inv)
                    for M in (1, 8) for inv in (False, True)]

# Case 3: Llama-7B-shaped decode, bf16 x / params.
AFFINE_DECODE = (
    [AffineCase(f"affine_b4_g128_M{M}_K{K}_N{N}", M, K, N, 4, 128, "bf16", "bf16", True)
     for (K, N) in ((4096, 4096), (4096, 11008), (11008, 4096)) for M in (1, 4, 16)]
    + [AffineCase(f"affine_b{b}_g64_M{M}_K4096_N4096", M, 4096, 4096, b, 64, "bf16", "bf16", True)
       for b in (2, 8) for M in (1, 4, 16)]
)

# Case 4: prefill GEMM, 4-bit group 64, 0.1% x20 outliers in W.
AFFINE_PREFILL = AffineCase("affine_b4_g64_M2048_K4096_N14336", 2048, 4096, 14336, 4, 64,
                            "bf16", "bf16", True, outliers=True)

# Case 5: W8A8 / W4A8, K = N = 8192.
INT_LINEAR = [IntCase(f"int_M{M}_K8192_N8192", M, 8192, 8192) for M in (1, 256, 4096)]
