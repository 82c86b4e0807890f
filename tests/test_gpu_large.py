"""Maximum sizes: layers with 2^32 packed codes (2 GiB of weights), so every element index and byte
offset passes 2^31; checked on sampled output rows against the oracle."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib, to_dev, u32_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    return build_lib()


def _rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(n, size=count, replace=False))
    rows[0], rows[-1] = 0, n - 1
    return rows


def test_affine_decode_2gib_codes(ql, orc):
    """4-bit g128, 2 tokens x 16384 -> 262144 (2 GiB of codes): the ring-streaming decode kernel."""
    M, K, N, g = 2, 16384, 262144, 128
    codes = synth.random_words(901, (N, K * 4 // 32))
    s_vals, _ = synth.to_bf16(np.abs(synth.normal(902, (N, K // g), 0.002)) + np.float32(1e-3))
    b_vals, _ = synth.to_bf16(synth.normal(903, (N, K // g), 0.01))
    x = synth.activations(904, (M, K), "bf16")
    lb = synth.activations(905, (N,), "bf16", 0.01)
    y = ql.matmul(x.torch("cuda"), u32_dev(codes), to_dev(s_vals, torch.bfloat16), to_dev(b_vals, torch.bfloat16),
                  4, g, lb.torch("cuda"))
    torch.cuda.synchronize()
    rows = _rows(N, 64, 906)
    yr, mag = orc.affine_matmul(x.vals, codes[rows], s_vals[rows], b_vals[rows], 4, g, lb.vals[rows])
    assert_fp_close(y[:, torch.as_tensor(rows, device="cuda")], yr, mag, lb.vals[rows], "affine 2 GiB")


def test_bitlinear_decode_2gib_packed(ql, orc):
    """BitLinear, 1 token x 16384 -> 524288 (packed [131072, 16384] = 2 GiB, every byte value):
    the 8-row-CTA path; sampled packed rows r with all four outputs r + j N/4."""
    K, R = 16384, 131072
    N = 4 * R
    P = synth.random_words(911, (R, K // 4)).view(np.uint8)
    x = synth.activations(912, (1, K), "bf16")
    ws = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    y = ql.bitlinear_matmul(x.torch("cuda"), torch.from_numpy(P).cuda(), N, ws, True)
    torch.cuda.synchronize()
    rows = _rows(R, 32, 913)
    yr, mag = orc.bitlinear(x.vals, np.ascontiguousarray(P[rows]), 4 * len(rows), 0.5, True)
    cols = np.concatenate([rows + j * R for j in range(4)])  # the oracle's outputs i + j S
    assert_fp_close(y[:, torch.as_tensor(cols, device="cuda")], yr, mag, None, "bitlinear 2 GiB")


def test_w8a8_decode_2gib_weights(ql, orc):
    """W8A8, 1 token x 16384 -> 131072 (int8 weights [131072, 16384] = 2 GiB): the int8 GEMV."""
    K, N = 16384, 131072
    qw = synth.random_words(921, (N, K // 4)).view(np.int8)
    sw = (np.abs(synth.normal(922, (N,), 1e-4)) + np.float32(1e-5)).astype(np.float32)
    x = synth.activations(923, (1, K), "bf16")
    y = ql.w8a8_linear(x.torch("cuda"), torch.from_numpy(qw).cuda(), to_dev(sw))
    torch.cuda.synchronize()
    rows = _rows(N, 64, 924)
    yr, mag, _, _ = orc.w8a8_linear(x.vals, np.ascontiguousarray(qw[rows]), sw[rows])
    assert_fp_close(y[:, torch.as_tensor(rows, device="cuda")], yr, mag, None, "w8a8 2 GiB")
