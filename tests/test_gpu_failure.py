"""Failure handling on the GPU without a fault: a bounded wait that runs out."""
import pytest
import torch

import synth
from helpers import assert_fp_close, build_lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ql():
    return build_lib()


def test_bounded_wait_reports_timeout_and_context_stays_usable(ql, orc):
    assert ql.device_status() == ql.QLIN_OK
    ql.selftest_wait_timeout(1000)  # a wait on a barrier nothing completes, limited to 1 ms
    assert ql.device_status() == ql.QLIN_ERR_TIMEOUT
    assert ql.device_status() == ql.QLIN_OK  # the status word was cleared
    # the library still computes correctly afterwards
    case = synth.BITLINEAR_DECODE[0]
    P = case.packed()
    x = case.x()
    ws = torch.tensor([case.weight_scale], dtype=torch.float32, device="cuda")
    y = ql.bitlinear_matmul(x.torch("cuda"), torch.from_numpy(P).cuda(), case.N, ws, case.invert)
    torch.cuda.synchronize()
    assert ql.device_status() == ql.QLIN_OK
    yr, mag = orc.bitlinear(x.vals, P, case.N, case.weight_scale, case.invert)
    assert_fp_close(y, yr, mag, None, case.name)


def test_selftest_rejects_bad_limit(ql):
    with pytest.raises(ql.QlinError) as e:
        ql.selftest_wait_timeout(0)
    assert e.value.status == ql.QLIN_ERR_INVALID_ARG
    with pytest.raises(ql.QlinError) as e:
        ql.selftest_wait_timeout(3_000_000)
    assert e.value.status == ql.QLIN_ERR_INVALID_ARG
