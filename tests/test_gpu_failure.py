"""Failure detection without a GPU fault.

Every wait inside the library's kernels is bounded (one second of
%globaltimer); a wait that runs out records IVIT_ERR_TIMEOUT in the device
status word and the kernel returns.  ivit_selftest_wait_timeout enqueues a
kernel whose wait nothing ever satisfies, so the test sees the status once,
sees it cleared, and then runs an operator bit-exactly in the same context.
The wait takes about one second.
"""
import numpy as np
import pytest
import torch

import integer_only_quantized_int8_b200 as ivit
import oracle
import synthetic
from integer_only_quantized_int8_b200 import build as ivit_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    ivit_build.build()


def test_wait_that_runs_out_reports_timeout_and_context_stays_usable():
    assert ivit.ivit_stream_status() == 0
    ivit.ivit_selftest_wait_timeout()
    assert ivit.ivit_status_string(ivit.ivit_stream_status()) == "IVIT_ERR_TIMEOUT"
    assert ivit.ivit_stream_status() == 0          # reported once, then cleared
    gc = synthetic.gelu_case(4099, seed=5)
    I0 = ivit.ivit_i0_from_scale(gc.S_h)
    go = ivit.ivit_dyadic_from_double(gc.out_ratio)
    x = torch.from_numpy(gc.x).cuda()
    y = torch.empty_like(x)
    ivit.ivit_shiftgelu(x, I0, 30, 8, go, y)
    assert ivit.ivit_stream_status() == 0
    np.testing.assert_array_equal(y.cpu().numpy(), oracle.shiftgelu(gc.x, I0, 30, 8, go))
