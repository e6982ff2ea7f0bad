"""Pins of the oracle's variants: ShiftGELU with a row maximum, Log-Int-Softmax
attention and I-LayerNorm with power-of-two factors.

Each is pinned to something other than its own code: a hand-derived worked
example (tests/golden), the textbook log2 by brute force over every input,
closed forms on inputs where the result is known, and reductions to the
already pinned base operators on inputs where the variant must agree with
them.
"""
import math
import os

import numpy as np
import pytest

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, *v = line.split()
                vals[k] = [int(t) for t in v]
    return vals


# ---------------------------------------------------------------- row-max ShiftGELU

def test_rowmax_shiftgelu_worked_example():
    g = read_golden("shiftgelu_rowmax_worked_example.txt")
    I0, M, k_out = g["I0"][0], g["M"][0], g["k_out"][0]
    x = np.array([g["x"]], dtype=np.int8)
    sigma = g["sigma"]
    # out = (1, 0): y = sat8(x sigma); out = (1, 4): y = (x sigma) >> 4
    y0 = oracle.shiftgelu_rowmax(x, I0, M, k_out, (1, 0))[0]
    y4 = oracle.shiftgelu_rowmax(x, I0, M, k_out, (1, 4))[0]
    for xi, s, a, b in zip(g["x"], sigma, y0, y4):
        assert a == max(-128, min(127, xi * s))
        assert b == max(-128, min(127, (xi * s) >> 4))
    # the exponentials of the derivation are the oracle's shift-exponential
    for ip, e1 in zip(g["I_p"], g["e1"]):
        assert oracle.shift_exp(ip - max(g["I_p"]), I0) == e1
    assert oracle.shift_exp(-max(g["I_p"]), I0) == g["e2"][0]


def test_rowmax_shiftgelu_reduces_to_per_element_reading():
    """Where the row maximum equals the element's own exponent offset, the two
    readings coincide: rows with no positive exponent (I_max = 0 everywhere),
    and the element that holds the row's maximum."""
    r = np.random.default_rng(5)
    I0 = 13
    x = -r.integers(0, 129, size=(6, 96)).astype(np.int8)       # all <= 0: I_max = 0
    np.testing.assert_array_equal(oracle.shiftgelu_rowmax(x, I0, 30, 8, (1, 3)),
                                  oracle.shiftgelu(x, I0, 30, 8, (1, 3)))
    x = r.integers(-128, 128, size=(8, 64)).astype(np.int8)
    y_row = oracle.shiftgelu_rowmax(x, I0, 30, 8, (1, 4))
    y_elt = oracle.shiftgelu(x, I0, 30, 8, (1, 4))
    for i in range(x.shape[0]):
        j = int(np.argmax(x[i]))                                 # I_p is non-decreasing in x
        assert y_row[i, j] == y_elt[i, j]


def test_rowmax_shiftgelu_zero_over_zero_gives_zero():
    """I_0 = 2 and a row holding 127: I_max = 212, so ShiftExp(-I_max) = 0 and
    the element -128 has both exponentials 0 (the reading: sigma = 0)."""
    x = np.array([[127, -128, 0]], dtype=np.int8)
    assert oracle.shift_exp(-212, 2) == 0
    y = oracle.shiftgelu_rowmax(x, 2, 30, 8, (1, 7))
    assert y[0, 1] == 0 and y[0, 2] == 0
    assert y[0, 0] == 127                                        # sigma = 128: (127 * 128) >> 7


# ---------------------------------------------------------------- Log-Int-Softmax

def test_log2_code_against_textbook_log2_every_input():
    """k = clip(15 - round(log2 P16), 0, 15) for every P16 in [0, 2^15], against
    the floating-point log2 (no input sits exactly on a rounding tie: the ties
    are at 2^b sqrt 2, irrational)."""
    for P in range(0, (1 << 15) + 1):
        want = 15 if P == 0 else min(15, max(0, 15 - int(math.floor(math.log2(P) + 0.5))))
        assert oracle.log2_code(P) == want, P
    # the thresholds either side of 2^7 sqrt 2 = 181.02 and 2^14 sqrt 2 = 23170.48
    assert [oracle.log2_code(p) for p in (181, 182, 23170, 23171)] == [8, 7, 1, 0]


def test_lis_row_single_key_and_equal_keys():
    # a single key: P16 = 2^15, code 0 (probability 1)
    assert list(oracle.lis_row([5], I0=20)) == [0]
    # 2^m equal logits with I_0 a power of two: P16 = 2^(15 - m) exactly, code m
    for m in range(0, 8):
        assert set(oracle.lis_row(np.zeros(1 << m, dtype=np.int32), I0=16)) == {m}


def test_lis_row_codes_track_the_probabilities():
    """Codes never increase with the logit, and each is within half a binade of
    -log2 of the row's 16-bit probability (the rounding of log2)."""
    r = np.random.default_rng(9)
    for trial in range(50):
        n = int(r.integers(1, 300))
        I0 = int(r.integers(1, 200))
        L = r.integers(-128, 128, size=n).astype(np.int32)
        codes = oracle.lis_row(L, I0)
        order = np.argsort(L, kind="stable")
        assert np.all(np.diff(codes[order]) <= 0)
        mx = int(L.max())
        e = np.array([oracle.shift_exp(int(l) - mx, I0) for l in L])
        P16 = np.array([oracle.int_div(int(v), int(e.sum()), 30, 16) for v in e])
        for p, k in zip(P16, codes):
            if p >= 1 and 0 < k < 15:
                assert abs(-math.log2(p / 2 ** 15) - k) <= 0.5


def test_attention_lis_closed_forms():
    """Q = 0: every logit is 0, so with N = 2^m keys and I_0 = 16 each code is
    m and ctx_d = requant(2^(15 - m) sum_j V_jd).  N = 1: code 0, ctx = requant(V 2^15)."""
    r = np.random.default_rng(3)
    H = 2
    D = 64 * H
    for N in (1, 2, 8, 64):
        m = int(math.log2(N))
        qkv = r.integers(-128, 128, size=(N, 3 * D)).astype(np.int8)
        qkv[:, :D] = 0
        out = (1, 15 + 3)                                   # ctx = (acc >> 18)
        ctx = oracle.attention_lis(qkv, 1, N, H, (1, 0), 8, 16, 30, out)
        V = qkv[:, 2 * D:].astype(np.int64)
        acc = (1 << (15 - m)) * V.sum(axis=0)
        want = np.clip(acc >> 18, -128, 127)
        np.testing.assert_array_equal(ctx[0] if N == 1 else ctx[0], want)
        np.testing.assert_array_equal(ctx, np.tile(want, (N, 1)))


# ---------------------------------------------------------------- PTF I-LayerNorm

def test_layernorm_ptf_factor_zero_is_i_layernorm():
    r = np.random.default_rng(21)
    x = r.integers(-128, 128, size=(7, 192)).astype(np.int8)
    gamma = r.integers(-128, 128, size=192).astype(np.int8)
    beta = r.integers(-5000, 5000, size=192).astype(np.int32)
    np.testing.assert_array_equal(oracle.layernorm_ptf(x, np.zeros(192, np.uint8), gamma, beta, 7, 20, (3, 12)),
                                  oracle.layernorm(x, gamma, beta, 7, 20, (3, 12)))


def test_layernorm_ptf_is_i_layernorm_of_the_shifted_input():
    """Where x << alpha still fits int8 (|x| <= 15, alpha <= 3), PTF I-LayerNorm
    is the (pinned) I-LayerNorm of the shifted row."""
    r = np.random.default_rng(22)
    cols = 256
    x = r.integers(-15, 16, size=(9, cols)).astype(np.int8)
    alpha = r.integers(0, 4, size=cols).astype(np.uint8)
    gamma = r.integers(-128, 128, size=cols).astype(np.int8)
    beta = r.integers(-5000, 5000, size=cols).astype(np.int32)
    shifted = (x.astype(np.int32) << alpha.astype(np.int32)).astype(np.int8)
    np.testing.assert_array_equal(oracle.layernorm_ptf(x, alpha, gamma, beta, 7, 20, (3, 12)),
                                  oracle.layernorm(shifted, gamma, beta, 7, 20, (3, 12)))


def test_layernorm_ptf_beats_per_tensor_input_on_outlier_channels(capsys):
    """The point of the factors (reported, and required to hold on this input):
    on LayerNorm inputs whose channel scales span 0.1 .. 20 (the ViT-B recipe),
    PTF-quantised inputs give a smaller error against floating-point LayerNorm
    than one per-tensor scale does."""
    pc = synthetic.ptf_case(rows=64, cols=768, seed=4)
    ln_f = pc.ln_float
    out = oracle.dyadic(pc.out_ratio)
    y_ptf = oracle.layernorm_ptf(pc.x_ptf, pc.alpha, pc.gamma, pc.beta, 7, 20, out) * pc.S_out
    y_pt = oracle.layernorm(pc.x_tensor, pc.gamma, pc.beta, 7, 20, out) * pc.S_out
    e_ptf = float(np.abs(y_ptf - ln_f).mean())
    e_pt = float(np.abs(y_pt - ln_f).mean())
    with capsys.disabled():
        print(f"\n[fp report] LayerNorm mean |error| on outlier channels: PTF {e_ptf:.4f}, per tensor {e_pt:.4f}")
    assert e_ptf < e_pt
