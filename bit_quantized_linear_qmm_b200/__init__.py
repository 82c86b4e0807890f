"""Quantized linear layers on the NVIDIA B200 (sm_100a), computed straight from
packed low-bit weights.  The compute lives in libqlin.so (C ABI: include/qlin.h);
this package holds its sources (csrc/), its build script and a thin binding."""
from . import qlin  # noqa: F401
from .qlin import (  # noqa: F401
    QlinError, bitlinear_matmul, dequantize, device_status, int8_matmul_int32, matmul,
    pack_int4_cols, quantize, quantize_int8_rows, w4a8_linear, w8a8_linear, workspace_size,
)
