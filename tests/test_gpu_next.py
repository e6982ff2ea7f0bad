"""GPU parity of the variant operators against the CPU oracle, bit for bit:
ShiftGELU with a row maximum, attention with Log-Int-Softmax, and I-LayerNorm
with power-of-two input factors.  Outputs sit between canary bytes (a write
past either end fails the test without faulting)."""
import numpy as np
import pytest
import torch

import integer_only_quantized_int8_b200 as ivit
import oracle
import synthetic
from integer_only_quantized_int8_b200 import build as ivit_build

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0x5A


@pytest.fixture(scope="module", autouse=True)
def built():
    ivit_build.build()
    yield
    assert ivit.ivit_stream_status() == 0


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def guarded(shape):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
    view = buf[GUARD:GUARD + n].view(torch.int8).view(shape)

    def untouched():
        h = host(buf)
        return bool((h[:GUARD] == CANARY).all() and (h[GUARD + n:] == CANARY).all())

    return view, untouched


# ---------------------------------------------------------------- row-max ShiftGELU

@pytest.mark.parametrize("rows,cols", [(1, 16), (5, 48), (64, 768), (394, 3072), (3, 16384)])
def test_shiftgelu_rowmax_parity(rows, cols):
    gc = synthetic.gelu_case(rows * cols, seed=rows + cols)
    x = gc.x.reshape(rows, cols).copy()
    x[0, :] = -np.arange(cols) % 129                       # a row with no positive exponent (I_max = 0)
    I0 = oracle.recip_i0(gc.S_h)
    out = oracle.dyadic(gc.out_ratio)
    y, untouched = guarded((rows, cols))
    ivit.ivit_shiftgelu_rowmax(dev(x, torch.int8), I0, 30, 8, out, y)
    np.testing.assert_array_equal(host(y), oracle.shiftgelu_rowmax(x, I0, 30, 8, out))
    assert untouched()


@pytest.mark.parametrize("rows,cols", [(20000, 256), (12000, 592), (6000, 1536), (4000, 2560), (3000, 4096),
                                       (600, 4112)])
def test_shiftgelu_rowmax_many_rows(rows, cols):
    """More rows than the kernel's warps, so that warps take several rows
    (the next row loads while the current one is looked up), at row lengths
    that cover every register-resident width and the two-pass fallback; row
    maxima vary at random, so a warp's rows switch between the shared table
    of rows that reach 127 and its own tables."""
    gc = synthetic.gelu_case(rows * cols, seed=rows ^ cols)
    x = gc.x.reshape(rows, cols).copy()
    caps = np.random.default_rng(cols).choice([127, 127, 127, 126, 100, 40, 1, 0, -5, -128], size=rows)
    x = np.minimum(x, caps[:, None].astype(np.int8))
    I0 = oracle.recip_i0(gc.S_h)
    out = oracle.dyadic(gc.out_ratio)
    y, untouched = guarded((rows, cols))
    ivit.ivit_shiftgelu_rowmax(dev(x, torch.int8), I0, 30, 8, out, y)
    np.testing.assert_array_equal(host(y), oracle.shiftgelu_rowmax(x, I0, 30, 8, out))
    assert untouched()


@pytest.mark.parametrize("I0,M,k_out", [(1, 30, 8), (2, 30, 8), (13, 20, 6), (4096, 30, 8)])
def test_shiftgelu_rowmax_parameters(I0, M, k_out):
    """Every int8 value in every row, at I0 = 2 (both exponentials underflow
    for most elements: the 0 / 0 reading), I0 = 1, a large I0 and a narrow
    IntDiv."""
    r = np.random.default_rng(I0 + M)
    x = np.stack([r.permutation(np.arange(-128, 128)) for _ in range(8)]).astype(np.int8)
    x[3] = np.clip(x[3], -128, 0)
    y = torch.empty((8, 256), dtype=torch.int8, device="cuda")
    ivit.ivit_shiftgelu_rowmax(dev(x, torch.int8), I0, M, k_out, (3, 9), y)
    np.testing.assert_array_equal(host(y), oracle.shiftgelu_rowmax(x, I0, M, k_out, (3, 9)))


# ---------------------------------------------------------------- Log-Int-Softmax attention

LIS_CASES = [(1, 1, 1, "normal", 8, 30), (2, 5, 1, "laplace", 8, 30), (2, 33, 2, "normal", 6, 20),
             (3, 130, 2, "laplace", 8, 15), (2, 197, 3, "normal", 8, 30), (1, 256, 2, "laplace", 8, 30),
             (1, 300, 1, "laplace", 8, 30), (1, 577, 2, "laplace", 8, 30), (1, 640, 1, "normal", 8, 24)]


@pytest.mark.parametrize("B,N,H,tails,k_s,M", LIS_CASES)
def test_attention_lis_parity(B, N, H, tails, k_s, M):
    ac = synthetic.attention_case(B, N, H, seed=B * 100 + N + H, tails=tails, k_s=k_s)
    logit = oracle.dyadic(ac.logit_ratio)
    I0 = oracle.recip_i0(ac.S_logit)
    out = oracle.dyadic(ac.out_ratio * 2.0 ** -8)              # S_v 2^-15 / S_ctx
    qkv = dev(ac.qkv, torch.int8)
    ctx, untouched = guarded((B * N, H * 64))
    ivit.ivit_attention_lis(qkv, B, N, H, logit, k_s, I0, M, out, ctx)
    want = oracle.attention_lis(ac.qkv, B, N, H, logit, k_s, I0, M, out)
    np.testing.assert_array_equal(host(ctx), want)
    assert untouched()
    assert np.unique(want).size > 8                            # the case is not degenerate


def test_attention_lis_refusals():
    qkv = torch.zeros((5, 3 * 64), dtype=torch.int8, device="cuda")
    ctx = torch.empty((5, 64), dtype=torch.int8, device="cuda")
    with pytest.raises(ivit.IvitError):                        # M < 15: no 16-bit probability
        ivit.ivit_attention_lis(qkv, 1, 5, 1, (1, 8), 8, 10, 14, (1, 20), ctx)
    with pytest.raises(ivit.IvitError):                        # wider logits than the table
        ivit.ivit_attention_lis(qkv, 1, 5, 1, (1, 8), 10, 10, 30, (1, 20), ctx)
    ivit.ivit_attention_lis(qkv, 0, 5, 1, (1, 8), 8, 10, 30, (1, 20), ctx)   # empty batch: nothing to do


# ---------------------------------------------------------------- PTF I-LayerNorm

@pytest.mark.parametrize("rows,cols,M_ln", [(1, 16, 20), (7, 192, 20), (100, 768, 20), (33, 2048, 18),
                                            (12608, 768, 20)])
def test_layernorm_ptf_parity(rows, cols, M_ln):
    pc = synthetic.ptf_case(rows, cols, seed=rows + cols)
    x = pc.x_ptf.copy()
    x[0] = 9                                                   # a row constant before the factors
    out = oracle.dyadic(pc.out_ratio)
    y, untouched = guarded((rows, cols))
    ivit.ivit_layernorm_ptf(dev(x, torch.int8), dev(pc.alpha, torch.uint8), dev(pc.gamma, torch.int8),
                            dev(pc.beta, torch.int32), 7, M_ln, out, y)
    np.testing.assert_array_equal(host(y), oracle.layernorm_ptf(x, pc.alpha, pc.gamma, pc.beta, 7, M_ln, out))
    assert untouched()


def test_layernorm_ptf_extremes():
    """Every channel at factor 3 and the int8 extremes: |x << alpha| = 1024 and
    the largest sums the 32-bit accumulation must hold (2048 columns)."""
    cols = 2048
    x = np.tile(np.array([-128, 127], dtype=np.int8), (4, cols // 2))
    x[1] = -128
    x[2, ::3] = 0
    alpha = np.full(cols, 3, dtype=np.uint8)
    alpha[::5] = 0
    r = np.random.default_rng(8)
    gamma = r.integers(-128, 128, size=cols).astype(np.int8)
    beta = r.integers(-(1 << 30), 1 << 30, size=cols).astype(np.int32)
    for out in ((1 << 30, 31), (12345, 20), (2147483647, 31)):
        y = torch.empty((4, cols), dtype=torch.int8, device="cuda")
        ivit.ivit_layernorm_ptf(dev(x, torch.int8), dev(alpha, torch.uint8), dev(gamma, torch.int8),
                                dev(beta, torch.int32), 7, 20, out, y)
        np.testing.assert_array_equal(host(y), oracle.layernorm_ptf(x, alpha, gamma, beta, 7, 20, out))
