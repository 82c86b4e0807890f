"""The column-parallel split with the CUDA kernels, its ranks emulated on one GPU: every rank's block
of outputs is computed by the library on that rank's weight shard (made contiguous, as a rank would
hold it), the blocks are assembled in global output order, and the result matches the oracle on the
unsplit layer.  (The collective itself is covered by the two-rank gloo test on CPU.)"""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, to_dev

pytestmark = pytest.mark.gpu


def _dev(t):
    return None if t is None else to_dev(np.ascontiguousarray(t))


@pytest.mark.parametrize("world", [2, 3])
def test_split_layers_on_one_gpu(orc, world):
    ql = build_lib()
    from bit_quantized_linear_qmm_b200 import colsplit
    M, K = 20, 1024
    xa = synth.activations(96, (M, K), "bf16")
    x = xa.torch("cuda")
    N = 384
    w = synth.normal(97, (N, K), 0.02)
    bias = synth.activations(98, (N,), "bf16", 0.01)
    # affine 4-bit g64 bf16 params (M > 16: the tcgen05 prefill on each shard)
    codes, s, b = orc.affine_quantize(w, 4, 64, True)
    full = {"codes": codes, "scales": s, "biases": b, "bias": bias.vals}
    parts = []
    for r in range(world):
        t = colsplit.shard("affine", full, N, world, r)
        parts.append(ql.matmul(x, _dev(t["codes"]).view(torch.int32),
                               _dev(t["scales"]).to(torch.bfloat16), _dev(t["biases"]).to(torch.bfloat16), 4, 64,
                               _dev(t["bias"]).to(torch.bfloat16)))
    y = colsplit.assemble_torch("affine", parts, N)
    yr, mag = orc.affine_matmul(xa.vals, codes, s, b, 4, 64, bias.vals)
    assert_fp_close(y, yr, mag, bias.vals, f"affine split {world}")
    # W4A8 (columns of the packed [K/2, N] weight; blocks of 16 columns)
    P4, s4 = orc.pack_int4_cols(synth.normal(99, (K, N), 0.02))
    full = {"packed": P4, "scale_w": s4, "bias": None}
    parts = []
    for r in range(world):
        t = colsplit.shard("w4a8", full, N, world, r)
        parts.append(ql.w4a8_linear(x, _dev(t["packed"]), _dev(t["scale_w"])))
    y = colsplit.assemble_torch("w4a8", parts, N)
    yr, mag, _, _ = orc.w4a8_linear(xa.vals, P4, s4, None)
    assert_fp_close(y, yr, mag, None, f"w4a8 split {world}")
    # BitLinear (packed rows; outputs r + j N/4)
    P = synth.any_bytes(100, N // 4, K)
    ws = torch.tensor([0.5], device="cuda")
    full = {"packed": P, "bias": bias.vals}
    parts = []
    for r in range(world):
        t = colsplit.shard("bitlinear", full, N, world, r)
        parts.append(ql.bitlinear_matmul(x, _dev(t["packed"]), 4 * t["packed"].shape[0], ws, False,
                                         _dev(t["bias"]).to(torch.bfloat16)))
    y = colsplit.assemble_torch("bitlinear", parts, N)
    yr, mag = orc.bitlinear(xa.vals, P, N, 0.5, False, bias.vals)
    assert_fp_close(y, yr, mag, bias.vals, f"bitlinear split {world}")
    torch.cuda.synchronize()
    assert ql.device_status() == ql.QLIN_OK
