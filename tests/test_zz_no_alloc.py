"""The allocation-free block forward (collected last on purpose).

``ivit_block_forward_static`` serves callers that cannot allocate device
memory -- a plugin whose host gives it no allocator, code inside a framework
whose allocator already holds the whole device, a loop that cannot afford
cudaMalloc -- by keeping the block's intermediates in the library's own fixed
device array.  These tests call it through the C ABI and check that two calls
in a row reproduce the workspace-based ``ivit_block_forward`` exactly (the
bit-exact bar of every other test here), and that a batch whose intermediates
do not fit is refused.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import integer_only_quantized_int8_b200 as ivit
import synthetic
from integer_only_quantized_int8_b200 import build as ivit_build
from integer_only_quantized_int8_b200 import params as ivit_params

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_static_scratch_matches_workspace_forward_twice():
    ivit_build.build()
    L = ivit.lib()
    dev = torch.device("cuda", 0)
    B, N = 3, 197
    for seed, tails in ((21, "normal"), (22, "laplace")):   # two calls in a row, different inputs
        wl = synthetic.make_workload(B=B, N=N, D=192, H=3, Dm=768, seed=seed, n_cal=2, tails=tails)
        dp = ivit_params.to_device(ivit_params.integer_params(wl.blocks[0]), dev)
        x = torch.from_numpy(wl.x).to(dev)
        want = torch.empty_like(x)
        ws = torch.empty(ivit.ivit_block_workspace_bytes(B, N, wl.D, wl.Dm), dtype=torch.uint8, device=dev)
        ivit.ivit_block_forward(dp, x, want, ws, B, N)
        got = torch.full_like(x, 77)
        st = L.ivit_block_forward_static(C.byref(dp.c), C.c_void_p(x.data_ptr()), C.c_void_p(got.data_ptr()),
                                         B, N, C.c_void_p(_stream()))
        assert st == 0, ivit.ivit_status_string(st)
        torch.cuda.synchronize()
        assert ivit.ivit_stream_status() == 0
        np.testing.assert_array_equal(got.cpu().numpy(), want.cpu().numpy())


def test_static_scratch_refuses_oversized_batch():
    ivit_build.build()
    L = ivit.lib()
    dev = torch.device("cuda", 0)
    wl = synthetic.make_workload(B=1, N=197, D=192, H=3, Dm=768, seed=23, n_cal=1)
    dp = ivit_params.to_device(ivit_params.integer_params(wl.blocks[0]), dev)
    x = torch.from_numpy(wl.x).to(dev)
    y = torch.empty_like(x)
    B = 100                                                   # 37.8 MB of intermediates > 32 MiB
    assert ivit.ivit_block_workspace_bytes(B, 197, 192, 768) > ivit.STATIC_SCRATCH_BYTES
    st = L.ivit_block_forward_static(C.byref(dp.c), C.c_void_p(x.data_ptr()), C.c_void_p(y.data_ptr()),
                                     B, 197, C.c_void_p(_stream()))
    assert st == 2, ivit.ivit_status_string(st)               # IVIT_ERR_UNSUPPORTED, nothing enqueued
    with pytest.raises(ivit.IvitError):
        ivit.ivit_block_forward_static(dp, x, y, B, 197)
