"""Host-only checks of the C ABI: the library builds, loads and exports every
function include/qlin.h declares, and argument validation answers before any
device work (no GPU needed)."""
import ctypes as C

import pytest

from helpers import build_lib


@pytest.fixture(scope="module")
def ql():
    return build_lib()


def test_exports_every_declared_function(ql):
    names = ql.header_functions()
    assert len(names) >= 13
    L = ql.lib()
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(ql):
    for s in range(8):
        assert ql.status_string(s).startswith("QLIN_")
    assert "unknown" in ql.status_string(99)


def test_workspace_sizes(ql):
    assert ql.workspace_size(ql.QLIN_OP_MATMUL, 16, 4096, 4096, 4, 128) == 0
    # tensor-core prefill: fp16 x [M, K] and group parameters [N, K/g] x 2, token and row scales
    M, N, K, g = 2048, 14336, 4096, 64
    a = lambda v: (v + 255) // 256 * 256  # noqa: E731
    assert ql.workspace_size(ql.QLIN_OP_MATMUL, M, N, K, 4, g) == \
        a(M * K * 2) + 2 * a(N * (K // g) * 2) + a(-(-M // 256) * 256 * 4) + a(N * 4)
    assert ql.workspace_size(ql.QLIN_OP_MATMUL, M, N, K, 2, g) == 0  # 2-bit codes: no prefill GEMM
    assert ql.workspace_size(ql.QLIN_OP_BITLINEAR, 8, 4096, 4096) == 0
    assert ql.workspace_size(ql.QLIN_OP_W8A8, 4096, 8192, 8192) == 4096 * 8192 + 4096 * 4
    assert ql.workspace_size(ql.QLIN_OP_W8A8, 1, 8192, 8192) == 8192 + 256
    assert ql.workspace_size(ql.QLIN_OP_W4A8, 1, 8192, 8192) == 8192 + 256


P16 = C.c_void_p(256)  # a non-null, 16-byte aligned stand-in; never dereferenced on these paths


def test_validation_before_device(ql):
    L = ql.lib()
    # null pointers
    assert L.qlin_quantize(None, 0, 4, 64, 4, 64, P16, P16, P16, 0, None) == ql.QLIN_ERR_INVALID_ARG
    # unsupported bits / group
    assert L.qlin_quantize(P16, 0, 4, 64, 7, 64, P16, P16, P16, 0, None) == ql.QLIN_ERR_UNSUPPORTED
    assert L.qlin_quantize(P16, 0, 4, 64, 0, 64, P16, P16, P16, 0, None) == ql.QLIN_ERR_UNSUPPORTED
    assert L.qlin_quantize(P16, 3, 4, 64, 4, 64, P16, P16, P16, 0, None) == ql.QLIN_ERR_UNSUPPORTED  # no dtype 3
    assert L.qlin_quantize(P16, 0, 4, 64, 4, 48, P16, P16, P16, 0, None) == ql.QLIN_ERR_UNSUPPORTED
    # K not a multiple of the group
    assert L.qlin_dequantize(P16, P16, P16, 0, 4, 96, 4, 64, P16, 0, None) == ql.QLIN_ERR_INVALID_ARG
    # codes not 4-byte aligned (a 4-byte aligned pointer that breaks the 16-byte rule takes the
    # general kernel instead), x not 16-byte aligned
    assert L.qlin_matmul(P16, 1, 1, 128, C.c_void_p(258), P16, P16, 1, 64, 4, 64, None, P16, None, 0,
                         None) == ql.QLIN_ERR_MISALIGNED
    assert L.qlin_matmul(C.c_void_p(264), 2, 1, 96, P16, P16, P16, 1, 64, 3, 32, None, P16, None, 0,
                         None) == ql.QLIN_ERR_MISALIGNED
    # BitLinear needs N % 4 == 0 and K % 16 == 0
    assert L.bitlinear_matmul(P16, 1, 1, 64, P16, 6, P16, 0, None, P16, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.bitlinear_matmul(P16, 1, 1, 60, P16, 8, P16, 0, None, P16, None) == ql.QLIN_ERR_INVALID_ARG
    # int4 needs even K
    assert L.qlin_pack_int4_cols(P16, 0, 3, 8, P16, P16, None) == ql.QLIN_ERR_INVALID_ARG


def test_valid_call_without_gpu_reports_device(ql):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = ql.lib()
    assert L.qlin_matmul(P16, 1, 1, 128, P16, P16, P16, 1, 64, 4, 64, None, P16, None, 0,
                         None) == ql.QLIN_ERR_DEVICE
    assert L.qlin_get_device_status(None) == ql.QLIN_ERR_DEVICE


def test_empty_inputs_rejected_before_device(ql):
    """M, N or K = 0 is an invalid argument for every entry (checked before any device access)."""
    L = ql.lib()
    assert L.qlin_matmul(P16, 1, 0, 128, P16, P16, P16, 1, 64, 4, 64, None, P16, None, 0, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_matmul(P16, 1, 1, 128, P16, P16, P16, 1, 0, 4, 64, None, P16, None, 0, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_matmul(P16, 1, 1, 0, P16, P16, P16, 1, 64, 4, 64, None, P16, None, 0, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.bitlinear_matmul(P16, 1, 0, 64, P16, 8, P16, 0, None, P16, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.bitlinear_matmul(P16, 1, 1, 64, P16, 0, P16, 0, None, P16, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize(P16, 0, 0, 64, 4, 64, P16, P16, P16, 0, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_dequantize(P16, P16, P16, 0, 4, 0, 4, 64, P16, 0, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_int8_rows(P16, 1, 0, 64, P16, P16, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_pack_int4_cols(P16, 1, 64, 0, P16, P16, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_int8_matmul_int32(P16, P16, 0, 16, 16, P16, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.w8a8_linear(P16, 1, 0, 64, P16, P16, 16, None, P16, P16, 4096, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.w4a8_linear(P16, 1, 1, 64, P16, P16, 0, None, P16, P16, 4096, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.pergroup_linear(P16, 1, 0, 128, P16, P16, 16, 64, None, P16, P16, 4096, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_int8_groups(P16, 1, 16, 0, 64, P16, P16, None) == ql.QLIN_ERR_INVALID_ARG
    assert L.qlin_quantize_weight_int8(P16, 1, 0, 64, -1.0, P16, P16, None) == ql.QLIN_ERR_INVALID_ARG


@pytest.mark.parametrize("op,M,N,want", [
    # int8 weights, K = N = 8192 on 148 SMs: 148 tiles of 128 x 112 at 256 tokens (one round; 256 x 112
    # tiles took 41.6 us there against 30.9), 148 tiles of 256 x 112 at 384 and 512 tokens (41.6 / 43.6 us
    # against 50.2 / 51.8 for two rounds of 128 x 112), 128 x 256 once they fill every SM
    ("W8A8", 256, 8192, (128, 112)), ("W8A8", 384, 8192, (256, 112)), ("W8A8", 512, 8192, (256, 112)),
    ("W8A8", 4096, 8192, (128, 256)), ("W8A8", 512, 4096, (128, 112)), ("W8A8", 1, 8192, (128, 112)),
    # packed int4 weights: 128 x 128 at 256 tokens (39.1 us; 128 x 256: 48.5), 128 x 256 at 384 (49.4 us
    # against 66.8 for two rounds of 128 x 128)
    ("W4A8", 256, 8192, (128, 128)), ("W4A8", 384, 8192, (128, 256)), ("W4A8", 4096, 8192, (128, 256)),
])
def test_int8_gemm_tile_choice(ql, op, M, N, want):
    """The int8 tensor-core GEMM's CTA tile on a 148-SM part, pinned to the shapes that timed fastest."""
    assert ql.int8_gemm_tile(getattr(ql, "QLIN_OP_" + op), M, N, 148) == want


def test_int8_gemm_tile_rejects(ql):
    t, c = C.c_int(0), C.c_int(0)
    L = ql.lib()
    for args in [(ql.QLIN_OP_MATMUL, 256, 8192, 148), (ql.QLIN_OP_W8A8, 0, 8192, 148),
                 (ql.QLIN_OP_W8A8, 256, 0, 148), (ql.QLIN_OP_W4A8, 256, 8192, 0)]:
        assert L.qlin_int8_gemm_tile(*args, C.byref(t), C.byref(c)) == ql.QLIN_ERR_INVALID_ARG, args
    assert L.qlin_int8_gemm_tile(ql.QLIN_OP_W8A8, 256, 8192, 148, None, C.byref(c)) == ql.QLIN_ERR_INVALID_ARG
