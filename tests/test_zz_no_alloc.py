"""The allocation-free block forward (collected last on purpose).

``ivit_block_forward_static`` serves callers that cannot allocate device
memory -- a plugin whose host gives it no allocator, code inside a framework
whose allocator already holds the whole device, a loop that cannot afford
cudaMalloc -- by keeping the block's intermediates in the library's own fixed
device array.  These tests call it through the C ABI and check that calls in a
row reproduce the workspace-based ``ivit_block_forward`` exactly (the
bit-exact bar of every other test here), at a small width and at the largest
ViT-B batch the array holds; that the next batch up is refused with nothing
enqueued; and that repeated calls leave the device's free memory unchanged.
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

N_TOK = 197


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _largest_batch(D, Dm):
    B = 0
    while ivit.ivit_block_workspace_bytes(B + 1, N_TOK, D, Dm) <= ivit.STATIC_SCRATCH_BYTES:
        B += 1
    return B


def _static_call(L, dp, x, y, B):
    return L.ivit_block_forward_static(C.byref(dp.c), C.c_void_p(x.data_ptr()), C.c_void_p(y.data_ptr()),
                                       B, N_TOK, C.c_void_p(_stream()))


def _check_against_workspace_forward(L, wl, dev):
    B = wl.B
    dp = ivit_params.to_device(ivit_params.integer_params(wl.blocks[0]), dev)
    x = torch.from_numpy(wl.x).to(dev)
    want = torch.empty_like(x)
    ws = torch.empty(ivit.ivit_block_workspace_bytes(B, N_TOK, wl.D, wl.Dm), dtype=torch.uint8, device=dev)
    ivit.ivit_block_forward(dp, x, want, ws, B, N_TOK)
    got = torch.full_like(x, 77)
    st = _static_call(L, dp, x, got, B)
    assert st == 0, ivit.ivit_status_string(st)
    torch.cuda.synchronize()
    assert ivit.ivit_stream_status() == 0
    np.testing.assert_array_equal(got.cpu().numpy(), want.cpu().numpy())
    return dp, x


def test_static_scratch_matches_workspace_forward_twice():
    ivit_build.build()
    L = ivit.lib()
    dev = torch.device("cuda", 0)
    for seed, tails in ((21, "normal"), (22, "laplace")):   # two calls in a row, different inputs
        wl = synthetic.make_workload(B=3, N=N_TOK, D=192, H=3, Dm=768, seed=seed, n_cal=2, tails=tails)
        _check_against_workspace_forward(L, wl, dev)


def test_static_scratch_largest_vit_b_batch():
    """The largest ViT-B batch whose intermediates fit the array, twice, then
    the next batch up, which must be refused by the library and the binding."""
    ivit_build.build()
    L = ivit.lib()
    dev = torch.device("cuda", 0)
    D, H, Dm = 768, 12, 3072
    Bmax = _largest_batch(D, Dm)
    assert Bmax == 22                                           # 22 x 197 x 7680 bytes <= 32 MiB < 23 x ...
    for seed in (24, 25):
        wl = synthetic.make_workload(B=Bmax, N=N_TOK, D=D, H=H, Dm=Dm, seed=seed, n_cal=2, chan_std=(0.1, 20.0))
        dp, x = _check_against_workspace_forward(L, wl, dev)
    # the next batch: x and y sized for it, so the refusal is the library's
    big = torch.zeros(((Bmax + 1) * N_TOK, D), dtype=torch.int8, device=dev)
    out = torch.empty_like(big)
    st = _static_call(L, dp, big, out, Bmax + 1)
    assert st == 2, ivit.ivit_status_string(st)                # IVIT_ERR_UNSUPPORTED, nothing enqueued
    with pytest.raises(ivit.IvitError):
        ivit.ivit_block_forward_static(dp, big, out, Bmax + 1, N_TOK)
    with pytest.raises(ivit.IvitError):                         # tensors too small: still the size refusal
        ivit.ivit_block_forward_static(dp, x, out, 100, N_TOK)


def test_static_scratch_allocates_nothing():
    """Repeated calls leave the device's free memory exactly where it was."""
    ivit_build.build()
    L = ivit.lib()
    dev = torch.device("cuda", 0)
    wl = synthetic.make_workload(B=2, N=N_TOK, D=192, H=3, Dm=768, seed=26, n_cal=1)
    dp = ivit_params.to_device(ivit_params.integer_params(wl.blocks[0]), dev)
    x = torch.from_numpy(wl.x).to(dev)
    y = torch.empty_like(x)
    assert _static_call(L, dp, x, y, wl.B) == 0                 # first call: symbol lookup, module loaded
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    for _ in range(2):
        assert _static_call(L, dp, x, y, wl.B) == 0
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info(dev)[0] == free0
    assert ivit.ivit_stream_status() == 0


def test_static_scratch_empty_batch_needs_no_device_work():
    ivit_build.build()
    L = ivit.lib()
    dev = torch.device("cuda", 0)
    wl = synthetic.make_workload(B=1, N=N_TOK, D=192, H=3, Dm=768, seed=27, n_cal=1)
    dp = ivit_params.to_device(ivit_params.integer_params(wl.blocks[0]), dev)
    x = torch.from_numpy(wl.x).to(dev)
    y = torch.empty_like(x)
    assert _static_call(L, dp, x, y, 0) == 0
    # argument errors come before the capacity check, as in ivit_block_forward
    st = L.ivit_block_forward_static(C.byref(dp.c), C.c_void_p(x.data_ptr()), C.c_void_p(x.data_ptr()),
                                     1000, N_TOK, C.c_void_p(_stream()))
    assert st == 1, ivit.ivit_status_string(st)                # x aliases y: IVIT_ERR_INVALID_ARG
