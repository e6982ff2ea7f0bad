"""Failure detection without a GPU fault.

Every wait inside the library's kernels is bounded (one second of
%globaltimer); a wait that runs out records IVIT_ERR_TIMEOUT in the device
status word and the kernel returns.  ivit_selftest_wait_timeout enqueues a
kernel whose wait nothing ever satisfies, so the test sees the status once,
sees it cleared, and then runs an operator bit-exactly in the same context.
ivit_selftest_withhold makes the production kernels take the same path: the
TMA producer of the GEMM (plain and residual epilogue) or of the attention
kernel stops before one load, the tensor-core issuer's bounded wait runs out,
every role gives up, drains and frees its tensor memory, and the same
operator then runs again bit-exactly.  Each timeout takes about one second.
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


def _timeout_then_exact(run, want):
    assert ivit.ivit_stream_status() == 0
    run()
    assert ivit.ivit_status_string(ivit.ivit_stream_status()) == "IVIT_ERR_TIMEOUT"
    assert ivit.ivit_stream_status() == 0          # reported once, then cleared
    got = run()
    assert ivit.ivit_stream_status() == 0
    np.testing.assert_array_equal(got, want)


# K = 1024 takes the shared-tile GEMM kernel, K = 384 the own-tile one
@pytest.mark.parametrize("K,residual", [(1024, False), (1024, True), (384, False), (384, True)])
def test_gemm_producer_stops_and_the_gemm_reports_timeout(K, residual):
    lc = synthetic.linear_case(1000, K, 512, seed=31, with_skip=residual)
    b, c = zip(*[ivit.ivit_dyadic_from_double(r) for r in lc.ratio])
    b = np.array(b, dtype=np.int32)
    c = np.array(c, dtype=np.int8)
    res = ivit.ivit_residual_from_double(*lc.res_ratio) if residual else None
    X, W = torch.from_numpy(lc.X).cuda(), torch.from_numpy(lc.W).cuda()
    bias, bd, cd = (torch.from_numpy(a).cuda() for a in (lc.bias, b, c))
    skip = torch.from_numpy(lc.skip).cuda() if residual else None
    Y = torch.empty((1000, 512), dtype=torch.int8, device="cuda")
    state = {"first": True}

    def run():
        if state.pop("first", False):
            ivit.ivit_selftest_withhold(ivit.SELFTEST_GEMM, 2)   # the third k-slice of CTA 0
        Y.fill_(0)
        ivit.ivit_linear_requant(X, W, bias, bd, cd, Y, skip=skip, res=res)
        torch.cuda.synchronize()
        return Y.cpu().numpy()

    want = oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, skip=lc.skip if residual else None,
                                 res=res if residual else (0, 0, 0))
    _timeout_then_exact(run, want)


def test_attention_producer_stops_and_the_attention_reports_timeout():
    B, N, H = 4, 197, 3
    ac = synthetic.attention_case(B, N, H, seed=32, tails="laplace")
    logit, out = ivit.ivit_dyadic_from_double(ac.logit_ratio), ivit.ivit_dyadic_from_double(ac.out_ratio)
    I0 = ivit.ivit_i0_from_scale(ac.S_logit)
    qkv = torch.from_numpy(ac.qkv).cuda()
    ctx = torch.empty((B * N, H * 64), dtype=torch.int8, device="cuda")
    state = {"first": True}

    def run():
        if state.pop("first", False):
            ivit.ivit_selftest_withhold(ivit.SELFTEST_ATTENTION, 0)   # CTA 0's first item
        ctx.fill_(0)
        ivit.ivit_attention(qkv, B, N, H, logit, 8, I0, 30, 8, out, ctx)
        torch.cuda.synchronize()
        return ctx.cpu().numpy()

    _timeout_then_exact(run, oracle.attention(ac.qkv, B, N, H, logit, 8, I0, 30, 8, out))
