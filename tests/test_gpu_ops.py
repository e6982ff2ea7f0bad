"""GPU parity of every operator against the CPU oracle, bit for bit.

Inputs are seeded synthetic tensors (``synthetic``); each side derives its
integer parameters from the same real scales with its own code (the library's
host helpers vs the oracle's).  Sizes span several tiles and ragged tails;
edge cases cover single rows/keys, empty inputs and the maximum key count.
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
    yield
    assert ivit.ivit_stream_status() == 0


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


GUARD = 4096   # canary bytes on each side of a guarded output (keeps 16-byte alignment)
CANARY = 0x5A


def guarded(shape):
    """An int8 output inside a larger buffer whose canary bytes on both sides
    must survive the call: a check for writes past either end of the output
    (they land in the test's own memory, so they cannot fault)."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
    view = buf[GUARD:GUARD + n].view(torch.int8).view(shape)

    def untouched():
        h = host(buf)
        return bool((h[:GUARD] == CANARY).all() and (h[GUARD + n:] == CANARY).all())

    return view, untouched


# ---------------------------------------------------------------------------
# INT8 linear + dyadic requant (tcgen05 GEMM)
# ---------------------------------------------------------------------------

LINEAR_SHAPES = [
    (1, 16, 16), (5, 32, 48), (197, 192, 576), (130, 384, 384), (300, 768, 3072),
    (256, 3072, 768), (129, 64, 272), (1000, 1024, 512),
]


@pytest.mark.parametrize("M,K,N", LINEAR_SHAPES)
def test_linear_requant_parity(M, K, N):
    lc = synthetic.linear_case(M, K, N, seed=M + K + N, with_skip=True)
    bq = [ivit.ivit_dyadic_from_double(r) for r in lc.ratio]
    bo = [oracle.dyadic(r) for r in lc.ratio]
    b_d, c_d = np.array([x[0] for x in bq], np.int32), np.array([x[1] for x in bq], np.int8)
    b_o, c_o = np.array([x[0] for x in bo], np.int32), np.array([x[1] for x in bo], np.int32)
    X, W = dev(lc.X, torch.int8), dev(lc.W, torch.int8)
    Y, untouched = guarded((M, N))
    for use_bias in (True, False):
        bias = lc.bias if use_bias else None
        ivit.ivit_linear_requant(X, W, None if bias is None else dev(bias, torch.int32), dev(b_d, torch.int32),
                                 dev(c_d, torch.int8), Y)
        want = oracle.linear_requant(lc.X, lc.W, bias, b_o, c_o)
        np.testing.assert_array_equal(host(Y), want)
    # residual epilogue
    res_d = ivit.ivit_residual_from_double(*lc.res_ratio)
    res_o = oracle.dyadic_pair(*lc.res_ratio)
    ivit.ivit_linear_requant(X, W, dev(lc.bias, torch.int32), dev(b_d, torch.int32), dev(c_d, torch.int8), Y,
                             skip=dev(lc.skip, torch.int8), res=res_d)
    want = oracle.linear_requant(lc.X, lc.W, lc.bias, b_o, c_o, skip=lc.skip, res=res_o)
    np.testing.assert_array_equal(host(Y), want)
    # a narrower output width, alone and before the residual addition
    ivit.ivit_linear_requant(X, W, dev(lc.bias, torch.int32), dev(b_d, torch.int32), dev(c_d, torch.int8), Y,
                             out_bits=4)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(lc.X, lc.W, lc.bias, b_o, c_o, out_bits=4))
    ivit.ivit_linear_requant(X, W, dev(lc.bias, torch.int32), dev(b_d, torch.int32), dev(c_d, torch.int8), Y,
                             out_bits=5, skip=dev(lc.skip, torch.int8), res=res_d)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(lc.X, lc.W, lc.bias, b_o, c_o, out_bits=5,
                                                                 skip=lc.skip, res=res_o))
    assert untouched()


# Shapes whose token-tile width (chosen for the fewest rounds of tiles over
# 148 SMs) covers every width of both GEMM kernels: the shared-tile kernel
# at 256 (three-stage ring, one MMA issuer), 224, 192, 176 (twice, the second
# with a ragged channel tile), 160 and 128 (two issuers), and the own-tile
# kernel (three accumulators, K <= 512) at 160, 144 and 128.  Every M leaves
# a ragged last token tile, and the k-slice counts are odd and even.  Each
# shape runs the plain, residual, narrow-output and fused ShiftGELU
# epilogues (the ShiftGELU one takes the own-tile kernel up to K = 768).
TILE_WIDTH_SHAPES = [
    # shared-tile kernel (K > 512; the ShiftGELU epilogue at K > 768)
    (5421, 1024, 768),    # 256 tokens
    (4655, 896, 768),     # 224
    (4226, 1024, 768),    # 192
    (3890, 640, 768),     # 176
    (2881, 1152, 1008),   # 176, ragged channel tile
    (3121, 896, 768),     # 160
    (1013, 1024, 768),    # 128
    # own-tile kernel (K <= 512): 160, 144 and 128 tokens
    (3461, 384, 768),
    (3076, 512, 768),
    (2593, 384, 1008),    # ragged channel tile
    (2306, 256, 1008),
    (1013, 384, 768),
]


@pytest.mark.parametrize("M,K,N", TILE_WIDTH_SHAPES)
def test_linear_parity_every_tile_width(M, K, N):
    lc = synthetic.linear_case(M, K, N, seed=M + 2 * K + N, with_skip=True)
    bq = [ivit.ivit_dyadic_from_double(r) for r in lc.ratio]
    b = np.array([x[0] for x in bq], np.int32)
    c = np.array([x[1] for x in bq], np.int32)
    X, W = dev(lc.X, torch.int8), dev(lc.W, torch.int8)
    bd, cd, biasd = dev(b, torch.int32), dev(c, torch.int8), dev(lc.bias, torch.int32)
    Y, untouched = guarded((M, N))
    ivit.ivit_linear_requant(X, W, biasd, bd, cd, Y)
    plain = oracle.linear_requant(lc.X, lc.W, lc.bias, b, c)
    np.testing.assert_array_equal(host(Y), plain)
    res = ivit.ivit_residual_from_double(*lc.res_ratio)
    skip = dev(lc.skip, torch.int8)
    ivit.ivit_linear_requant(X, W, biasd, bd, cd, Y, skip=skip, res=res)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, skip=lc.skip, res=res))
    # the narrow-output and fused ShiftGELU epilogues at the same tile width
    ivit.ivit_linear_requant(X, W, biasd, bd, cd, Y, out_bits=4)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, out_bits=4))
    ivit.ivit_linear_requant(X, W, biasd, bd, cd, Y, out_bits=6, skip=skip, res=res)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, out_bits=6,
                                                                 skip=lc.skip, res=res))
    gc = synthetic.gelu_case(1024, seed=M)
    I0 = ivit.ivit_i0_from_scale(gc.S_h)
    go = ivit.ivit_dyadic_from_double(gc.out_ratio)
    ivit.ivit_linear_shiftgelu(X, W, biasd, bd, cd, I0, 30, 8, go, Y)
    np.testing.assert_array_equal(host(Y), oracle.shiftgelu(plain, I0, 30, 8, go))
    assert untouched()


@pytest.mark.parametrize("K", [4096, 16384])
def test_linear_saturation_and_extremes(K):
    """Saturating operands with b = 2^31 - 1 and every shift 0..31 (the wide
    and clamped requant forms).  K = 16384 is the largest reduction the ABI
    accepts; with |bias| up to 2^30 the accumulator reaches 2^28 + 2^30, the
    int32 range the ABI guarantees."""
    r = np.random.default_rng(30)
    M, N = 64, 32
    X = np.full((M, K), -128, np.int8)
    X[1::2] = 127
    W = r.choice(np.array([-128, 127], np.int8), size=(N, K))
    W[0] = -128                                  # row 0 of X times W[0]: 2^14 K = 2^28 at K = 16384
    b = np.zeros(N, np.int32); b[:] = 2 ** 31 - 1
    c = (np.arange(N) % 32).astype(np.int32)
    bias = r.integers(-2 ** 20, 2 ** 20, size=N).astype(np.int32)
    bias[0], bias[1] = 2 ** 30, -2 ** 30
    Y, untouched = guarded((M, N))
    ivit.ivit_linear_requant(dev(X, torch.int8), dev(W, torch.int8), dev(bias, torch.int32), dev(b, torch.int32),
                             dev(c, torch.int8), Y)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(X, W, bias, b, c))
    assert untouched()


@pytest.mark.parametrize("M,K,N", [(197, 192, 576), (300, 768, 3072), (129, 64, 272)])
def test_linear_round_half_up_parity(M, K, N):
    """The round-half-up variant of the linear requant: plain, residual and
    narrow outputs, and the fused fc1 + ShiftGELU."""
    lc = synthetic.linear_case(M, K, N, seed=3 * M + N, with_skip=True)
    bq = [ivit.ivit_dyadic_from_double(r) for r in lc.ratio]
    b = np.array([x[0] for x in bq], np.int32)
    c = np.array([x[1] for x in bq], np.int32)
    X, W = dev(lc.X, torch.int8), dev(lc.W, torch.int8)
    bd, cd, biasd = dev(b, torch.int32), dev(c, torch.int8), dev(lc.bias, torch.int32)
    Y = torch.empty((M, N), dtype=torch.int8, device="cuda")
    ivit.ivit_linear_requant(X, W, biasd, bd, cd, Y, rounding=1)
    want = oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, rounding=1)
    np.testing.assert_array_equal(host(Y), want)
    assert not np.array_equal(want, oracle.linear_requant(lc.X, lc.W, lc.bias, b, c))  # the variant differs
    res = ivit.ivit_residual_from_double(*lc.res_ratio)
    ivit.ivit_linear_requant(X, W, biasd, bd, cd, Y, skip=dev(lc.skip, torch.int8), res=res, rounding=1)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, skip=lc.skip, res=res,
                                                                 rounding=1))
    ivit.ivit_linear_requant(X, W, biasd, bd, cd, Y, out_bits=4, rounding=1)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, out_bits=4, rounding=1))
    gc = synthetic.gelu_case(1024, seed=M)
    I0 = ivit.ivit_i0_from_scale(gc.S_h)
    go = ivit.ivit_dyadic_from_double(gc.out_ratio)
    ivit.ivit_linear_shiftgelu(X, W, biasd, bd, cd, I0, 30, 8, go, Y, rounding=1)
    h = oracle.linear_requant(lc.X, lc.W, lc.bias, b, c, rounding=1)
    np.testing.assert_array_equal(host(Y), oracle.shiftgelu(h, I0, 30, 8, go))


def test_linear_round_half_up_extremes():
    """Wide and clamped requant forms (b = 2^31 - 1, every shift 0..31) with
    rounding, at K = 4096 with saturating inputs."""
    r = np.random.default_rng(31)
    M, K, N = 64, 4096, 32
    X = r.integers(-128, 128, (M, K), dtype=np.int8)
    X[::3] = -128
    W = r.choice(np.array([-128, 127, 1, -1], np.int8), size=(N, K))
    b = np.full(N, 2 ** 31 - 1, np.int32)
    b[::2] = r.integers(1, 1 << 12, N // 2)
    c = (np.arange(N) % 32).astype(np.int32)
    bias = r.integers(-2 ** 20, 2 ** 20, size=N).astype(np.int32)
    Y = torch.empty((M, N), dtype=torch.int8, device="cuda")
    ivit.ivit_linear_requant(dev(X, torch.int8), dev(W, torch.int8), dev(bias, torch.int32), dev(b, torch.int32),
                             dev(c, torch.int8), Y, rounding=1)
    np.testing.assert_array_equal(host(Y), oracle.linear_requant(X, W, bias, b, c, rounding=1))


# ---------------------------------------------------------------------------
# fused attention with Shiftmax
# ---------------------------------------------------------------------------

ATTN_CASES = [
    (1, 1, 1, "normal", 8), (2, 5, 1, "normal", 8), (2, 197, 3, "normal", 8), (1, 577, 2, "laplace", 8),
    (3, 130, 2, "normal", 8), (1, 128, 1, "laplace", 8), (2, 256, 1, "normal", 8), (1, 300, 1, "laplace", 8),
    (1, 640, 1, "laplace", 8), (2, 197, 2, "laplace", 4), (1, 33, 2, "normal", 6),
    # logits wider than 8 bits: ShiftExp computed per score
    (2, 197, 3, "normal", 16), (1, 256, 2, "laplace", 16), (2, 5, 1, "normal", 12), (3, 130, 2, "laplace", 12),
    (1, 33, 2, "normal", 10),
]


@pytest.mark.parametrize("B,N,H,tails,k_s", ATTN_CASES)
def test_attention_parity(B, N, H, tails, k_s):
    ac = synthetic.attention_case(B, N, H, seed=B * 1000 + N + H, tails=tails, k_s=k_s)
    logit_d, logit_o = ivit.ivit_dyadic_from_double(ac.logit_ratio), oracle.dyadic(ac.logit_ratio)
    out_d, out_o = ivit.ivit_dyadic_from_double(ac.out_ratio), oracle.dyadic(ac.out_ratio)
    I0_d, I0_o = ivit.ivit_i0_from_scale(ac.S_logit), oracle.recip_i0(ac.S_logit)
    qkv = dev(ac.qkv, torch.int8)
    ctx, untouched = guarded((B * N, H * 64))
    ivit.ivit_attention(qkv, B, N, H, logit_d, k_s, I0_d, 30, 8, out_d, ctx)
    want = oracle.attention(ac.qkv, B, N, H, logit_o, k_s, I0_o, 30, 8, out_o)
    np.testing.assert_array_equal(host(ctx), want)
    assert untouched()


# Short sequences with 8-bit logits: key counts that change how the 16-key
# chunks split over the two half rows (a ragged last chunk or none, chunks
# that stop short of the 32-key MMA step), both tails, and enough heads and
# images that every CTA takes many items through both softmax groups
SHORT_CASES = [(3, 1, 2, "normal"), (2, 17, 3, "laplace"), (4, 64, 2, "normal"), (2, 100, 3, "laplace"),
                 (1, 129, 2, "normal"), (2, 160, 3, "normal"), (2, 176, 2, "laplace"), (3, 193, 4, "normal"),
                 (64, 197, 12, "normal"), (5, 197, 3, "laplace"), (2, 200, 5, "laplace"), (3, 208, 4, "normal"),
                 (2, 209, 3, "laplace"), (4, 224, 4, "normal"), (1, 197, 1, "normal")]


@pytest.mark.parametrize("B,N,H,tails", SHORT_CASES)
def test_attention_short_parity(B, N, H, tails):
    ac = synthetic.attention_case(B, N, H, seed=7 * N + H, tails=tails, k_s=8)
    I0 = oracle.recip_i0(ac.S_logit)
    logit, out = oracle.dyadic(ac.logit_ratio), oracle.dyadic(ac.out_ratio)
    qkv = dev(ac.qkv, torch.int8)
    ctx, untouched = guarded((B * N, H * 64))
    ivit.ivit_attention(qkv, B, N, H, logit, 8, I0, 30, 8, out, ctx)
    np.testing.assert_array_equal(host(ctx), oracle.attention(ac.qkv, B, N, H, logit, 8, I0, 30, 8, out))
    assert untouched()


@pytest.mark.parametrize("I0,M,k_out", [(1, 30, 8), (2, 20, 8), (255, 30, 8), (97, 30, 5), (40, 12, 8),
                                        (256, 30, 8), (4096, 30, 8)])
def test_attention_short_shiftmax_parameters(I0, M, k_out):
    """N = 197 at I0 = 1 (a hard maximum), I0 at and past one byte, large I0,
    a small IntDiv M (the exact 32-bit product path instead of mul.hi) and
    k_out < 8."""
    ac = synthetic.attention_case(3, 197, 2, seed=300 + I0, tails="laplace")
    qkv = dev(ac.qkv, torch.int8)
    ctx = torch.empty((3 * 197, 128), dtype=torch.int8, device="cuda")
    logit = oracle.dyadic(ac.logit_ratio)
    out = oracle.dyadic(ac.out_ratio * 2 ** (8 - k_out))
    ivit.ivit_attention(qkv, 3, 197, 2, logit, 8, I0, M, k_out, out, ctx)
    np.testing.assert_array_equal(host(ctx), oracle.attention(ac.qkv, 3, 197, 2, logit, 8, I0, M, k_out, out))


@pytest.mark.parametrize("k_s", [8, 12, 16])
def test_attention_hardmax_wide_logits(k_s):
    """I_0 = 1 (the division by I_0 is the identity) and (b_s, c_s) = (1, 0):
    every key below the row maximum gets ShiftExp 0, at any logit width."""
    r = np.random.default_rng(40 + k_s)
    B, N, H = 2, 61, 2
    D = H * 64
    qkv = r.integers(-3, 5, size=(B * N, 3 * D)).astype(np.int8)
    ctx = torch.full((B * N, D), 99, dtype=torch.int8, device="cuda")
    ivit.ivit_attention(dev(qkv, torch.int8), B, N, H, (1, 0), k_s, 1, 30, 8, (1, 4), ctx)
    np.testing.assert_array_equal(host(ctx), oracle.attention(qkv, B, N, H, (1, 0), k_s, 1, 30, 8, (1, 4)))


@pytest.mark.parametrize("I0,M,k_out", [(1, 30, 8), (3, 20, 8), (97, 30, 5), (4096, 30, 8)])
def test_attention_shiftmax_parameters(I0, M, k_out):
    ac = synthetic.attention_case(2, 70, 2, seed=I0, tails="laplace")
    qkv = dev(ac.qkv, torch.int8)
    ctx = torch.empty((140, 128), dtype=torch.int8, device="cuda")
    logit = oracle.dyadic(ac.logit_ratio)
    out = oracle.dyadic(ac.out_ratio * 2 ** (8 - k_out))
    ivit.ivit_attention(qkv, 2, 70, 2, logit, 8, I0, M, k_out, out, ctx)
    np.testing.assert_array_equal(host(ctx), oracle.attention(ac.qkv, 2, 70, 2, logit, 8, I0, M, k_out, out))


# ---------------------------------------------------------------------------
# ShiftGELU
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 4099, 1 << 20, (1 << 20) + 13])
def test_shiftgelu_parity(n):
    gc = synthetic.gelu_case(max(n, 1), seed=n)
    x = gc.x[:n]
    I0_d, out_d = ivit.ivit_i0_from_scale(gc.S_h), ivit.ivit_dyadic_from_double(gc.out_ratio)
    I0_o, out_o = oracle.recip_i0(gc.S_h), oracle.dyadic(gc.out_ratio)
    xd = dev(x, torch.int8) if n else torch.empty(0, dtype=torch.int8, device="cuda")
    y, untouched = guarded((n,))
    ivit.ivit_shiftgelu(xd, I0_d, 30, 8, out_d, y)
    np.testing.assert_array_equal(host(y), oracle.shiftgelu(x, I0_o, 30, 8, out_o))
    assert untouched()


@pytest.mark.parametrize("I0", [1, 2, 5, 16, 25, 64, 1000])
def test_shiftgelu_all_inputs(I0):
    x = np.tile(np.arange(-128, 128, dtype=np.int8), 4)
    out = oracle.dyadic(1.0 / 128)
    y = torch.empty(x.size, dtype=torch.int8, device="cuda")
    ivit.ivit_shiftgelu(dev(x, torch.int8), I0, 30, 8, out, y)
    np.testing.assert_array_equal(host(y), oracle.shiftgelu(x, I0, 30, 8, out))


# ---------------------------------------------------------------------------
# I-LayerNorm
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(1, 16), (7, 192), (1000, 384), (4099, 768), (33, 1024), (9, 2048),
                                       (5, 48)])
def test_layernorm_parity(rows, cols):
    nc = synthetic.layernorm_case(rows, cols, seed=rows + cols)
    x = nc.x.copy()
    x[0] = 17                                    # a constant row (variance 0)
    out_d, out_o = ivit.ivit_dyadic_from_double(nc.out_ratio), oracle.dyadic(nc.out_ratio)
    y, untouched = guarded((rows, cols))
    ivit.ivit_layernorm(dev(x, torch.int8), dev(nc.gamma, torch.int8), dev(nc.beta, torch.int32), 7, 23, out_d, y)
    np.testing.assert_array_equal(host(y), oracle.layernorm(x, nc.gamma, nc.beta, 7, 23, out_o))
    assert untouched()


def test_layernorm_extreme_rows():
    cols = 256
    x = np.zeros((4, cols), np.int8)
    x[0, ::2], x[0, 1::2] = -128, 127            # maximum spread
    x[1, 0] = 1                                  # V floors to 0
    x[2] = -128
    x[3] = np.arange(cols) - 128
    gamma = np.full(cols, -128, np.int8)
    beta = np.arange(cols, dtype=np.int32) * 1000 - 100000
    out = (3, 2)
    y = torch.empty((4, cols), dtype=torch.int8, device="cuda")
    ivit.ivit_layernorm(dev(x, torch.int8), dev(gamma, torch.int8), dev(beta, torch.int32), 7, 23, out, y)
    np.testing.assert_array_equal(host(y), oracle.layernorm(x, gamma, beta, 7, 23, out))


def test_layernorm_variance_sweep():
    """Rows of two values a apart (half each, a = 0..255) have variance
    floor(a^2 / 4), from 0 up to 16256, the largest an int8 row can have: the
    Newton square root and the reciprocal 2^M / sigma are checked across the
    whole range, with M_ln = 23 and with a small M_ln."""
    cols = 64
    amp = np.arange(256)
    x = np.zeros((256, cols), np.int16)
    x[:, ::2] = -128
    x[:, 1::2] = (-128 + amp)[:, None]
    x = x.astype(np.int8)
    rng = np.random.default_rng(3)
    gamma = rng.integers(-128, 128, cols).astype(np.int8)
    beta = rng.integers(-(1 << 20), 1 << 20, cols).astype(np.int32)
    out = ivit.ivit_dyadic_from_double(1.0 / 3000.0)
    for F, M_ln in ((7, 23), (3, 9)):
        y = torch.empty((256, cols), dtype=torch.int8, device="cuda")
        ivit.ivit_layernorm(dev(x, torch.int8), dev(gamma, torch.int8), dev(beta, torch.int32), F, M_ln, out, y)
        np.testing.assert_array_equal(host(y), oracle.layernorm(x, gamma, beta, F, M_ln, oracle.dyadic(1.0 / 3000.0)))


@pytest.mark.parametrize("F", [0, 7, 14])
@pytest.mark.parametrize("side", [0.9, 1.1])
def test_layernorm_extreme_beta(F, side):
    """|beta| at its limit 2^30 and an output ratio on either side of the point
    where the product b acc can leave int32 (the kernel then clamps acc first)."""
    cols, rows = 64, 6
    rng = np.random.default_rng(F + int(10 * side))
    x = rng.integers(-128, 128, (rows, cols)).astype(np.int8)
    x[0, ::2], x[0, 1::2] = -128, 127
    gamma = np.where(np.arange(cols) % 2 == 0, -128, 127).astype(np.int8)
    beta = np.where(np.arange(cols) % 3 == 0, 1 << 30, -(1 << 30)).astype(np.int32)
    beta[5] = 0
    amax = 255.0 * 128.0 * 2.0**F + 2.0**30
    ratio = side * 2.0**30 / amax
    out_d, out_o = ivit.ivit_dyadic_from_double(ratio), oracle.dyadic(ratio)
    y = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
    ivit.ivit_layernorm(dev(x, torch.int8), dev(gamma, torch.int8), dev(beta, torch.int32), F, 23, out_d, y)
    np.testing.assert_array_equal(host(y), oracle.layernorm(x, gamma, beta, F, 23, out_o))


@pytest.mark.parametrize("M,K,N", [(1, 16, 16), (197, 192, 768), (300, 768, 3072), (129, 384, 1552)])
def test_linear_shiftgelu_parity(M, K, N):
    """fc1 with ShiftGELU in the epilogue == oracle linear, then oracle ShiftGELU."""
    lc = synthetic.linear_case(M, K, N, seed=7 * M + N)
    gc = synthetic.gelu_case(1024, seed=N)
    bq = [ivit.ivit_dyadic_from_double(r) for r in lc.ratio]
    bo = [oracle.dyadic(r) for r in lc.ratio]
    b_d, c_d = np.array([x[0] for x in bq], np.int32), np.array([x[1] for x in bq], np.int8)
    b_o, c_o = np.array([x[0] for x in bo], np.int32), np.array([x[1] for x in bo], np.int32)
    I0_d, out_d = ivit.ivit_i0_from_scale(gc.S_h), ivit.ivit_dyadic_from_double(gc.out_ratio)
    I0_o, out_o = oracle.recip_i0(gc.S_h), oracle.dyadic(gc.out_ratio)
    Y = torch.empty((M, N), dtype=torch.int8, device="cuda")
    ivit.ivit_linear_shiftgelu(dev(lc.X, torch.int8), dev(lc.W, torch.int8), dev(lc.bias, torch.int32),
                               dev(b_d, torch.int32), dev(c_d, torch.int8), I0_d, 30, 8, out_d, Y)
    h = oracle.linear_requant(lc.X, lc.W, lc.bias, b_o, c_o)
    np.testing.assert_array_equal(host(Y), oracle.shiftgelu(h, I0_o, 30, 8, out_o))


# ---------------------------------------------------------------------------
# steps either side of the blocks, and a whole model
# ---------------------------------------------------------------------------

from integer_only_quantized_int8_b200 import params as ivit_params  # noqa: E402


def _model_case_params(mc):
    ip = ivit_params.model_integer_params(mc)
    om = oracle.model_params(mc)
    # the library's host helpers and the oracle derive the same integers
    for k in ("b_pe", "c_pe", "b_head", "c_head"):
        np.testing.assert_array_equal(np.asarray(ip[k], np.int64), np.asarray(om[k], np.int64))
    assert tuple(ip["pos_add"]) == tuple(om["pos_add"]) and tuple(ip["head_ln_out"]) == tuple(om["head_ln_out"])
    return ip, om


@pytest.mark.parametrize("Hi,Wi,P", [(64, 48, 16), (24, 40, 8), (224, 224, 16)])
def test_patch_embed_parity(Hi, Wi, P):
    mc = synthetic.model_case(B=2, Hi=Hi, Wi=Wi, P=P, D=192, H=3, Dm=768, blocks=1, Ncls=100, seed=Hi + Wi + P)
    ip, om = _model_case_params(mc)
    B, Np = 2, (Hi // P) * (Wi // P)
    t = {k: dev(ip[k], dt) for k, dt in (("w_pe", torch.int8), ("bias_pe", torch.int32), ("b_pe", torch.int32),
                                         ("c_pe", torch.int8), ("cls", torch.int8), ("pos", torch.int8))}
    ws = torch.empty(ivit.ivit_patch_embed_workspace_bytes(B, 3, Hi, Wi, P, 192), dtype=torch.uint8, device="cuda")
    x = torch.full((B * (Np + 1), 192), 99, dtype=torch.int8, device="cuda")
    ivit.ivit_patch_embed(dev(mc.img, torch.int8), P, t["w_pe"], t["bias_pe"], t["b_pe"], t["c_pe"], t["cls"],
                          t["pos"], ip["pos_add"], ws, x)
    want = oracle.patch_embed(mc.img, P, mc.w_pe, mc.bias_pe, om["b_pe"], om["c_pe"], mc.cls, mc.pos, om["pos_add"])
    np.testing.assert_array_equal(host(x), want)


def test_head_parity():
    mc = synthetic.model_case(B=3, Hi=32, Wi=32, P=16, D=192, H=3, Dm=768, blocks=1, Ncls=100, seed=5)
    ip, om = _model_case_params(mc)
    B, Ntok, D = 5, 9, 192
    x = np.random.default_rng(6).integers(-128, 128, (B * Ntok, D), dtype=np.int8)
    ws = torch.empty(ivit.ivit_head_workspace_bytes(B, D), dtype=torch.uint8, device="cuda")
    logits = torch.full((B, mc.w_head.shape[0]), 99, dtype=torch.int8, device="cuda")
    ivit.ivit_head(dev(x, torch.int8), B, Ntok, dev(mc.head_gamma, torch.int8), dev(mc.head_beta, torch.int32),
                   7, 23, ip["head_ln_out"], dev(mc.w_head, torch.int8), dev(mc.bias_head, torch.int32),
                   dev(ip["b_head"], torch.int32), dev(ip["c_head"], torch.int8), ws, logits)
    want = oracle.head(x, B, Ntok, mc.head_gamma, mc.head_beta, 7, 23, om["head_ln_out"], mc.w_head, mc.bias_head,
                       om["b_head"], om["c_head"])
    np.testing.assert_array_equal(host(logits), want)


def test_model_forward_parity():
    """Patch embedding, two DeiT-Tiny-width blocks and the head through
    ivit_model_forward, against the oracle's composition of the same steps."""
    mc = synthetic.model_case(B=2, Hi=224, Wi=224, P=16, D=192, H=3, Dm=768, blocks=2, Ncls=1000, seed=9)
    ip, om = _model_case_params(mc)
    dm = ivit_params.model_to_device(ip)
    ws = torch.empty(ivit.ivit_model_workspace_bytes(dm, 2, 224, 224), dtype=torch.uint8, device="cuda")
    logits = torch.full((2, mc.w_head.shape[0]), 99, dtype=torch.int8, device="cuda")
    ivit.ivit_model_forward(dm, dev(mc.img, torch.int8), ws, logits)
    assert ivit.ivit_stream_status() == 0
    np.testing.assert_array_equal(host(logits), oracle.model_forward(om, mc))
