"""The tests' fp bar (helpers.assert_fp_close) against what a bf16 / fp16 / fp32 output can represent."""
import numpy as np
import torch

from helpers import half_ulp


def test_half_ulp_bounds_round_to_nearest():
    """Rounding any value to bf16 / fp32 moves it by at most half_ulp, and by exactly half_ulp at a
    tie: the term the bar adds for the output's one rounding is neither loose nor short."""
    rng = np.random.default_rng(0)
    # fp32 values (the kernels round fp32 results; a float64 -> bf16 cast in torch goes through fp32)
    v = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32).astype(np.float64)
    for dt in (torch.bfloat16, torch.float32):
        r = torch.from_numpy(v).to(dt).double().numpy()
        assert np.all(np.abs(r - v) <= half_ulp(v, dt))
    # fp16: finite range only (|v| < 65504), subnormals included (spacing 2^-24 below 2^-14)
    f = v[np.abs(v) < 65000.0]
    r = torch.from_numpy(f).to(torch.float16).double().numpy()
    assert np.all(np.abs(r - f) <= half_ulp(f, torch.float16))
    assert half_ulp(np.array([1e-7]), torch.float16)[0] == 2.0**-25
    assert half_ulp(np.array([1.0]), torch.float16)[0] == 2.0**-11
    # a bf16 tie: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    tie = np.array([1.0 + 2.0**-8])
    assert half_ulp(tie, torch.bfloat16)[0] == 2.0**-8
    assert abs(float(torch.tensor(tie).to(torch.bfloat16).double()) - tie[0]) == 2.0**-8
