"""Host-side size checks of the Python binding (no GPU needed).

Every wrapper checks, before it touches the library, that each tensor holds at
least as many elements as the library will read or write through its pointer.
A valid call made with host tensors gets past those checks and stops at the
device check ("must be a CUDA tensor"), so no call here reaches the library's
compute entry points on any machine.
"""
import pytest
import torch

import integer_only_quantized_int8_b200 as ivit
from integer_only_quantized_int8_b200 import build as ivit_build


@pytest.fixture(scope="module", autouse=True)
def built():
    ivit_build.build()


def i8(*shape):
    return torch.zeros(shape, dtype=torch.int8)


def i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


def u8(n):
    return torch.zeros(n, dtype=torch.uint8)


def expect_size_error(fn, *a, **k):
    with pytest.raises(ValueError, match="holds|must be \\[|shape|channels"):
        fn(*a, **k)


def expect_past_checks(fn, *a, **k):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn(*a, **k)


def test_linear_tables_hold_one_entry_per_channel():
    M, K, N = 32, 64, 48
    X, W, Y = i8(M, K), i8(N, K), i8(M, N)
    expect_past_checks(ivit.ivit_linear_requant, X, W, i32(N), i32(N), i8(N), Y)
    expect_past_checks(ivit.ivit_linear_requant, X, W, None, i32(N), i8(N), Y)  # bias is optional
    expect_size_error(ivit.ivit_linear_requant, X, W, i32(N), i32(N - 1), i8(N), Y)
    expect_size_error(ivit.ivit_linear_requant, X, W, i32(N), i32(N), i8(N - 16), Y)
    expect_size_error(ivit.ivit_linear_requant, X, W, i32(1), i32(N), i8(N), Y)
    g = (1, 0)
    expect_past_checks(ivit.ivit_linear_shiftgelu, X, W, i32(N), i32(N), i8(N), 4, 30, 8, g, Y)
    expect_size_error(ivit.ivit_linear_shiftgelu, X, W, i32(N), i32(N), i8(1), 4, 30, 8, g, Y)


def test_block_activations_hold_the_batch():
    p = ivit.BlockParams()
    p.D, p.H, p.Dm = 64, 1, 256
    B, N = 2, 9
    ws = u8(ivit.ivit_block_workspace_bytes(B, N, 64, 256))
    expect_past_checks(ivit.ivit_block_forward, p, i8(B * N, 64), i8(B * N, 64), ws, B, N)
    expect_size_error(ivit.ivit_block_forward, p, i8(B * N - 1, 64), i8(B * N, 64), ws, B, N)
    expect_size_error(ivit.ivit_block_forward, p, i8(B * N, 64), i8(B, 64), ws, B, N)
    expect_past_checks(ivit.ivit_block_forward_static, p, i8(B * N, 64), i8(B * N, 64), B, N)
    expect_size_error(ivit.ivit_block_forward_static, p, i8(B * N, 64), i8(B * N, 32), B, N)


def test_patch_embed_sizes():
    B, C, Hi, Wi, P, D = 2, 3, 32, 48, 16, 64
    Ntok = (Hi // P) * (Wi // P) + 1
    img = i8(B, C, Hi, Wi)
    W = i8(D, C * P * P)
    ws = u8(ivit.ivit_patch_embed_workspace_bytes(B, C, Hi, Wi, P, D))
    ok = dict(W=W, bias=i32(D), b=i32(D), c=i8(D), cls=i8(D), pos=i8(Ntok, D), x=i8(B * Ntok, D))

    def call(**over):
        a = {**ok, **over}
        return ivit.ivit_patch_embed(img, P, a["W"], a["bias"], a["b"], a["c"], a["cls"], a["pos"], (1, 1, 1),
                                     ws, a["x"])

    expect_past_checks(call)
    expect_past_checks(call, W=i8(D, C, P, P))       # the convolution layout holds the same bytes
    expect_size_error(call, W=i8(D, C * P * P - 16))
    expect_size_error(call, pos=i8(Ntok - 1, D))
    expect_size_error(call, cls=i8(D - 16))
    expect_size_error(call, x=i8(B * (Ntok - 1), D))
    expect_size_error(call, c=i8(D - 1))


def test_head_sizes():
    B, Ntok, D, Ncls = 3, 5, 64, 32
    ws = u8(ivit.ivit_head_workspace_bytes(B, D))
    ok = dict(x=i8(B * Ntok, D), gamma=i8(D), beta=i32(D), W=i8(Ncls, D), bias=i32(Ncls), b=i32(Ncls),
              c=i8(Ncls), logits=i8(B, Ncls))

    def call(**over):
        a = {**ok, **over}
        return ivit.ivit_head(a["x"], B, Ntok, a["gamma"], a["beta"], 7, 23, (1, 0), a["W"], a["bias"], a["b"],
                              a["c"], ws, a["logits"])

    expect_past_checks(call)
    expect_size_error(call, x=i8(B * Ntok - 1, D))
    expect_size_error(call, W=i8(Ncls, D - 16))
    expect_size_error(call, beta=i32(D - 1))
    expect_size_error(call, b=i32(Ncls - 16))
    expect_size_error(call, logits=i8(B - 1, Ncls))


def test_model_forward_sizes():
    m = ivit.ModelParams()
    m.C, m.P, m.D, m.Ncls = 3, 16, 64, 32
    img = i8(2, 3, 32, 32)
    expect_past_checks(ivit.ivit_model_forward, m, img, u8(1 << 16), i8(2, 32))
    expect_size_error(ivit.ivit_model_forward, m, i8(2, 1, 32, 32), u8(1 << 16), i8(2, 32))
    expect_size_error(ivit.ivit_model_forward, m, img, u8(1 << 16), i8(1, 32))
