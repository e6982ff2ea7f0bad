"""CPU oracle for the integer-only ViT encoder block (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library (``integer_only_quantized_int8_b200``) never imports it and shares no
code with it; the two meet only in the seeded input generator (``synthetic``),
which holds none of the method's arithmetic.

The arithmetic lives in ``ivit_oracle.c`` (plain single-threaded C, built with
gcc).  This module builds it on first use and exposes numpy-friendly wrappers,
plus the oracle's own derivation of integer parameters from real scales
(dyadic numbers, I_0 values) following "I-ViT: Integer-only Quantization for
Efficient Vision Transformer Inference", sections 3.2-3.5.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ivit_oracle.c")
_LIB = os.path.join(_HERE, "libivit_oracle.so")
_lock = threading.Lock()
_lib = None


def compile_source(src: str, out: str) -> str:
    """Compile one C source of the oracle into the shared library `out`."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ivit_oracle.c into a shared library next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def _i8p(a):
    return a.ctypes.data_as(C.POINTER(C.c_int8))


def _i32p(a):
    return a.ctypes.data_as(C.POINTER(C.c_int32))


def _opt_i32p(a):
    return None if a is None else _i32p(a)


class BlockParamsC(C.Structure):
    _fields_ = [(n, t) for n, t in [
        ("D", C.c_int32), ("H", C.c_int32), ("Dm", C.c_int32),
        ("ln1_gamma", C.c_void_p), ("ln1_beta", C.c_void_p), ("ln1_b", C.c_int32), ("ln1_c", C.c_int32),
        ("w_qkv", C.c_void_p), ("bias_qkv", C.c_void_p), ("b_qkv", C.c_void_p), ("c_qkv", C.c_void_p),
        ("logit_b", C.c_int32), ("logit_c", C.c_int32), ("k_s", C.c_int32), ("attn_I0", C.c_int32),
        ("attn_M", C.c_int32), ("attn_k_out", C.c_int32), ("attn_out_b", C.c_int32), ("attn_out_c", C.c_int32),
        ("w_o", C.c_void_p), ("bias_o", C.c_void_p), ("b_o", C.c_void_p), ("c_o", C.c_void_p),
        ("res1_b_skip", C.c_int32), ("res1_b_branch", C.c_int32), ("res1_c", C.c_int32),
        ("ln2_gamma", C.c_void_p), ("ln2_beta", C.c_void_p), ("ln2_b", C.c_int32), ("ln2_c", C.c_int32),
        ("w1", C.c_void_p), ("bias1", C.c_void_p), ("b1", C.c_void_p), ("c1", C.c_void_p),
        ("gelu_I0", C.c_int32), ("gelu_M", C.c_int32), ("gelu_k_out", C.c_int32), ("gelu_b", C.c_int32),
        ("gelu_c", C.c_int32),
        ("w2", C.c_void_p), ("bias2", C.c_void_p), ("b2", C.c_void_p), ("c2", C.c_void_p),
        ("res2_b_skip", C.c_int32), ("res2_b_branch", C.c_int32), ("res2_c", C.c_int32),
        ("ln_F", C.c_int32), ("ln_M", C.c_int32),
    ]]


def use_library(path: str):
    """Bind the oracle's functions to another build of its C source from now
    on (the planted-mistake test uses this on copies it has altered)."""
    global _lib
    with _lock:
        _lib = _bind(C.CDLL(path))


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(C.CDLL(build()))
    return _lib


def _bind(L):
    """Declare the argument and result types of every exported function."""
    L.orc_quantize.restype = C.c_int32
    L.orc_quantize.argtypes = [C.c_double, C.c_double, C.c_int]
    L.orc_dyadic.restype = C.c_int
    L.orc_dyadic.argtypes = [C.c_double, C.POINTER(C.c_int32), C.POINTER(C.c_int32)]
    L.orc_dyadic_pair.restype = C.c_int
    L.orc_dyadic_pair.argtypes = [C.c_double, C.c_double, C.POINTER(C.c_int32),
                                  C.POINTER(C.c_int32), C.POINTER(C.c_int32)]
    L.orc_recip_i0.restype = C.c_int32
    L.orc_recip_i0.argtypes = [C.c_double]
    L.orc_requant.restype = C.c_int64
    L.orc_requant.argtypes = [C.c_int64, C.c_int32, C.c_int32, C.c_int]
    L.orc_linear_requant.restype = None
    L.orc_linear_requant.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p, C.c_int32,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                     C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]
    L.orc_shift_exp.restype = C.c_int64
    L.orc_shift_exp.argtypes = [C.c_int64, C.c_int64]
    L.orc_int_div.restype = C.c_int64
    L.orc_int_div.argtypes = [C.c_int64, C.c_int64, C.c_int, C.c_int]
    L.orc_shiftmax_row.restype = None
    L.orc_shiftmax_row.argtypes = [C.c_void_p, C.c_int, C.c_int32, C.c_int, C.c_int, C.c_void_p]
    L.orc_attention.restype = None
    L.orc_attention.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32,
                                C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]
    L.orc_shift_sigmoid.restype = C.c_int64
    L.orc_shift_sigmoid.argtypes = [C.c_int64, C.c_int64, C.c_int32, C.c_int32]
    L.orc_shiftgelu_one.restype = C.c_int32
    L.orc_shiftgelu_one.argtypes = [C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                    C.c_int32, C.POINTER(C.c_int32)]
    L.orc_shiftgelu.restype = None
    L.orc_shiftgelu.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_int32, C.c_int32,
                                C.c_int32, C.c_int32, C.c_void_p]
    L.orc_isqrt_newton.restype = C.c_int64
    L.orc_isqrt_newton.argtypes = [C.c_int64]
    L.orc_layernorm.restype = None
    L.orc_layernorm.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p, C.c_void_p,
                                C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]
    L.orc_shiftgelu_rowmax.restype = None
    L.orc_shiftgelu_rowmax.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                       C.c_int32, C.c_int32, C.c_void_p]
    L.orc_log2_code.restype = C.c_int32
    L.orc_log2_code.argtypes = [C.c_int64]
    L.orc_lis_row.restype = None
    L.orc_lis_row.argtypes = [C.c_void_p, C.c_int, C.c_int32, C.c_int, C.c_void_p]
    L.orc_attention_lis.restype = None
    L.orc_attention_lis.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                    C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]
    L.orc_layernorm_ptf.restype = None
    L.orc_layernorm_ptf.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]
    L.orc_patch_embed.restype = C.c_int
    L.orc_patch_embed.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32,
                                  C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]
    L.orc_head.restype = C.c_int
    L.orc_head.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                           C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_int32,
                           C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    L.orc_set_linear_rounding.restype = None
    L.orc_set_linear_rounding.argtypes = [C.c_int]
    L.orc_block_forward.restype = C.c_int
    L.orc_block_forward.argtypes = [C.POINTER(BlockParamsC), C.c_void_p, C.c_void_p,
                                    C.c_int32, C.c_int32]
    return L


# ---------------------------------------------------------------------------
# scalar helpers
# ---------------------------------------------------------------------------

def quantize(R: float, m: float, k: int = 8) -> int:
    return int(lib().orc_quantize(float(R), float(m), int(k)))


def dyadic(s: float):
    """DN(s) -> (b, c) with b / 2^c ~ s (I-ViT section 3.2)."""
    b, c = C.c_int32(), C.c_int32()
    if lib().orc_dyadic(float(s), C.byref(b), C.byref(c)) != 0:
        raise ValueError(f"no dyadic number for {s!r}")
    return int(b.value), int(c.value)


def dyadic_pair(s1: float, s2: float):
    b1, b2, c = C.c_int32(), C.c_int32(), C.c_int32()
    if lib().orc_dyadic_pair(float(s1), float(s2), C.byref(b1), C.byref(b2), C.byref(c)) != 0:
        raise ValueError(f"no dyadic pair for {s1!r}, {s2!r}")
    return int(b1.value), int(b2.value), int(c.value)


def recip_i0(S: float) -> int:
    return int(lib().orc_recip_i0(float(S)))


def requant(acc: int, b: int, c: int, bits: int = 8) -> int:
    return int(lib().orc_requant(int(acc), int(b), int(c), int(bits)))


def shift_exp(I_delta: int, I0: int) -> int:
    return int(lib().orc_shift_exp(int(I_delta), int(I0)))


def int_div(e: int, total: int, M: int = 30, k_out: int = 8) -> int:
    return int(lib().orc_int_div(int(e), int(total), int(M), int(k_out)))


def isqrt_newton(V: int) -> int:
    return int(lib().orc_isqrt_newton(int(V)))


def shift_sigmoid(I_p: int, I0: int, M: int = 30, k_out: int = 8) -> int:
    """Integer sigmoid of S*I_p (S = 1/I0), scale 2^-(k_out-1) (I-ViT section 3.4)."""
    return int(lib().orc_shift_sigmoid(int(I_p), int(I0), int(M), int(k_out)))


def shiftgelu_one(I: int, I0: int, M: int = 30, k_out: int = 8, b_g: int = 1, c_g: int = 0):
    """Returns (g, sigma_int) for one int8 input."""
    s = C.c_int32()
    g = lib().orc_shiftgelu_one(int(I), int(I0), int(M), int(k_out), int(b_g), int(c_g), C.byref(s))
    return int(g), int(s.value)


# ---------------------------------------------------------------------------
# tensor ops (numpy in, numpy out)
# ---------------------------------------------------------------------------

def shiftmax_row(L, I0: int, M: int = 30, k_out: int = 8):
    L = np.ascontiguousarray(L, dtype=np.int32)
    P = np.zeros_like(L)
    lib().orc_shiftmax_row(L.ctypes.data, int(L.size), int(I0), int(M), int(k_out), P.ctypes.data)
    return P


class linear_rounding:
    """Context manager: the linear layers' requant rounds half up (mode 1)
    instead of the floor shift (mode 0) inside the block."""

    def __init__(self, mode: int):
        self.mode = int(mode)

    def __enter__(self):
        lib().orc_set_linear_rounding(self.mode)
        return self

    def __exit__(self, *exc):
        lib().orc_set_linear_rounding(0)
        return False


def linear_requant(X, W, bias, b, c, out_bits: int = 8, skip=None, res=(0, 0, 0), rounding: int = 0):
    """X [M x K] int8, W [N x K] int8, bias/b/c [N] -> Y [M x N] int8
    (rounding 1: the requant rounds half up)."""
    if rounding:
        with linear_rounding(rounding):
            return linear_requant(X, W, bias, b, c, out_bits, skip, res)
    X = np.ascontiguousarray(X, dtype=np.int8)
    W = np.ascontiguousarray(W, dtype=np.int8)
    M, K = X.shape
    N = W.shape[0]
    assert W.shape[1] == K
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.int32)
    b = np.ascontiguousarray(b, dtype=np.int32)
    c = np.ascontiguousarray(c, dtype=np.int32)
    Y = np.zeros((M, N), dtype=np.int8)
    sk = None
    if skip is not None:
        sk = np.ascontiguousarray(skip, dtype=np.int8)
        assert sk.shape == (M, N)
    lib().orc_linear_requant(X.ctypes.data, M, K, W.ctypes.data, N,
                             None if bias is None else bias.ctypes.data, b.ctypes.data, c.ctypes.data,
                             int(out_bits), None if sk is None else sk.ctypes.data,
                             int(res[0]), int(res[1]), int(res[2]), Y.ctypes.data)
    return Y


def attention(qkv, B: int, N: int, H: int, logit, k_s: int, I0: int, M: int, k_out: int, out):
    """qkv [B*N x 3*H*64] int8 -> ctx [B*N x H*64] int8."""
    qkv = np.ascontiguousarray(qkv, dtype=np.int8)
    assert qkv.shape == (B * N, 3 * H * 64)
    ctx = np.zeros((B * N, H * 64), dtype=np.int8)
    lib().orc_attention(qkv.ctypes.data, B, N, H, int(logit[0]), int(logit[1]), int(k_s), int(I0),
                        int(M), int(k_out), int(out[0]), int(out[1]), ctx.ctypes.data)
    return ctx


def shiftgelu(x, I0: int, M: int, k_out: int, out):
    x = np.ascontiguousarray(x, dtype=np.int8)
    y = np.zeros_like(x)
    lib().orc_shiftgelu(x.ctypes.data, x.size, int(I0), int(M), int(k_out), int(out[0]), int(out[1]),
                        y.ctypes.data)
    return y


def layernorm(x, gamma, beta, F: int, M_ln: int, out):
    x = np.ascontiguousarray(x, dtype=np.int8)
    rows, cols = x.shape
    gamma = np.ascontiguousarray(gamma, dtype=np.int8)
    beta = np.ascontiguousarray(beta, dtype=np.int32)
    y = np.zeros_like(x)
    lib().orc_layernorm(x.ctypes.data, rows, cols, gamma.ctypes.data, beta.ctypes.data,
                        int(F), int(M_ln), int(out[0]), int(out[1]), y.ctypes.data)
    return y


# ---------------------------------------------------------------------------
# variants: row-max ShiftGELU, Log-Int-Softmax attention, PTF I-LayerNorm
# ---------------------------------------------------------------------------

def shiftgelu_rowmax(x, I0: int, M: int, k_out: int, out):
    """x [rows x cols] int8 -> ShiftGELU with I_max the row's largest exponent."""
    x = np.ascontiguousarray(x, dtype=np.int8)
    rows, cols = x.shape
    y = np.zeros_like(x)
    lib().orc_shiftgelu_rowmax(x.ctypes.data, rows, cols, int(I0), int(M), int(k_out), int(out[0]), int(out[1]),
                               y.ctypes.data)
    return y


def log2_code(P16: int) -> int:
    return int(lib().orc_log2_code(int(P16)))


def lis_row(L, I0: int, M: int = 30):
    """4-bit log2 codes of one row of integer logits (Log-Int-Softmax)."""
    L = np.ascontiguousarray(L, dtype=np.int32)
    codes = np.zeros(L.size, dtype=np.int32)
    lib().orc_lis_row(L.ctypes.data, L.size, int(I0), int(M), codes.ctypes.data)
    return codes


def attention_lis(qkv, B: int, N: int, H: int, logit, k_s: int, I0: int, M: int, out):
    """qkv [B*N x 3*H*64] int8 -> ctx [B*N x H*64] int8 with Log-Int-Softmax."""
    qkv = np.ascontiguousarray(qkv, dtype=np.int8)
    assert qkv.shape == (B * N, 3 * H * 64)
    ctx = np.zeros((B * N, H * 64), dtype=np.int8)
    lib().orc_attention_lis(qkv.ctypes.data, B, N, H, int(logit[0]), int(logit[1]), int(k_s), int(I0), int(M),
                            int(out[0]), int(out[1]), ctx.ctypes.data)
    return ctx


def layernorm_ptf(x, alpha, gamma, beta, F: int, M_ln: int, out):
    """I-LayerNorm of x [rows x cols] whose channel i carries the power-of-two factor 2^alpha[i]."""
    x = np.ascontiguousarray(x, dtype=np.int8)
    rows, cols = x.shape
    alpha = np.ascontiguousarray(alpha, dtype=np.uint8)
    gamma = np.ascontiguousarray(gamma, dtype=np.int8)
    beta = np.ascontiguousarray(beta, dtype=np.int32)
    assert alpha.size == cols and int(alpha.max(initial=0)) <= 3
    y = np.zeros_like(x)
    lib().orc_layernorm_ptf(x.ctypes.data, rows, cols, alpha.ctypes.data, gamma.ctypes.data, beta.ctypes.data,
                            int(F), int(M_ln), int(out[0]), int(out[1]), y.ctypes.data)
    return y


# ---------------------------------------------------------------------------
# integer parameters of a block, derived from the real scales
# ---------------------------------------------------------------------------

def block_params(q, attn_M: int = 30, attn_k_out: int = 8, k_s: int = 8,
                 gelu_M: int = 30, gelu_k_out: int = 8, ln_F: int = 7, ln_M: int = 23):
    """Integer parameters of one block from a ``synthetic.QuantBlock``.

    Every multiplier is the oracle's own DN of a ratio of real scales
    (I-ViT section 3.2); I_0 values are the oracle's own reciprocal rounding
    (section 3.3).  Returns a dict of numpy arrays / ints.
    """
    S = q.scales
    D, H, Dm = q.D, q.H, q.Dm

    def per_channel(s_in, s_w, s_out):
        bc = [dyadic(s_in * float(sw) / float(so)) for sw, so in zip(s_w, s_out)]
        return (np.array([x[0] for x in bc], dtype=np.int32), np.array([x[1] for x in bc], dtype=np.int32))

    qkv_out = np.concatenate([np.full(D, S["q"]), np.full(D, S["k"]), np.full(D, S["v"])])
    p = dict(D=D, H=H, Dm=Dm, ln_F=ln_F, ln_M=ln_M, k_s=k_s,
             attn_M=attn_M, attn_k_out=attn_k_out, gelu_M=gelu_M, gelu_k_out=gelu_k_out)
    p["ln1_gamma"], p["ln1_beta"] = q.ln1_gamma, q.ln1_beta
    p["ln1_out"] = dyadic(S["gamma1"] * 2.0 ** -ln_F / S["ln1"])
    p["w_qkv"], p["bias_qkv"] = q.w_qkv, q.bias_qkv
    p["b_qkv"], p["c_qkv"] = per_channel(S["ln1"], q.s_w_qkv, qkv_out)
    p["logit"] = dyadic(S["q"] * S["k"] / (8.0 * S["logit"]))
    p["attn_I0"] = recip_i0(S["logit"])
    p["attn_out"] = dyadic(S["v"] * 2.0 ** -(attn_k_out - 1) / S["ctx"])
    p["w_o"], p["bias_o"] = q.w_o, q.bias_o
    p["b_o"], p["c_o"] = per_channel(S["ctx"], q.s_w_o, np.full(D, S["o"]))
    p["res1"] = dyadic_pair(S["x"] / S["xh"], S["o"] / S["xh"])
    p["ln2_gamma"], p["ln2_beta"] = q.ln2_gamma, q.ln2_beta
    p["ln2_out"] = dyadic(S["gamma2"] * 2.0 ** -ln_F / S["ln2"])
    p["w1"], p["bias1"] = q.w1, q.bias1
    p["b1"], p["c1"] = per_channel(S["ln2"], q.s_w1, np.full(Dm, S["h"]))
    p["gelu_I0"] = recip_i0(S["h"])
    p["gelu_out"] = dyadic(S["h"] * 2.0 ** -(gelu_k_out - 1) / S["g"])
    p["w2"], p["bias2"] = q.w2, q.bias2
    p["b2"], p["c2"] = per_channel(S["g"], q.s_w2, np.full(D, S["f"]))
    p["res2"] = dyadic_pair(S["xh"] / S["y"], S["f"] / S["y"])
    return p


def block_forward(p, x, B: int, N: int):
    """x [B*N x D] int8 -> y [B*N x D] int8 through one block (the linear
    layers round half up when p["linear_round"] is set)."""
    if p.get("linear_round", 0):
        with linear_rounding(1):
            return _block_forward(p, x, B, N)
    return _block_forward(p, x, B, N)


def _block_forward(p, x, B: int, N: int):
    x = np.ascontiguousarray(x, dtype=np.int8)
    s, keep = _block_struct(p)
    y = np.zeros_like(x)
    rc = lib().orc_block_forward(C.byref(s), x.ctypes.data, y.ctypes.data, int(B), int(N))
    if rc != 0:
        raise MemoryError("oracle block forward could not allocate scratch")
    return y


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - non-Linux
        return os.cpu_count() or 1


def block_forward_images(p, x, B: int, N: int, threads: int = 0):
    """The same result as ``block_forward(p, x, B, N)``, computed one image per
    task on ``threads`` host threads (default: every core this process may
    use).  Images never interact in the block, and each task is one call of
    the single-threaded C oracle on its own image (ctypes releases the
    interpreter lock for the call), so the output is identical to the
    single-call one.  Returns (y, threads used)."""
    from concurrent.futures import ThreadPoolExecutor
    x = np.ascontiguousarray(x, dtype=np.int8)
    threads = max(1, min(int(threads) or host_cores(), max(1, int(B))))
    if p.get("linear_round", 0):
        lib().orc_set_linear_rounding(1)
    try:
        s, keep = _block_struct(p)
        y = np.zeros_like(x)
        D = int(p["D"])
        row = N * D

        def one(img):
            off = img * row
            return lib().orc_block_forward(C.byref(s), x.ctypes.data + off, y.ctypes.data + off, 1, int(N))

        with ThreadPoolExecutor(max_workers=threads) as ex:
            rcs = list(ex.map(one, range(int(B))))
    finally:
        if p.get("linear_round", 0):
            lib().orc_set_linear_rounding(0)
    if any(rcs):
        raise MemoryError("oracle block forward could not allocate scratch")
    return y, threads


def _block_struct(p):
    """The C parameter struct of a block, and the arrays it points into."""
    keep = []

    def arr(a, dt):
        a = np.ascontiguousarray(a, dtype=dt)
        keep.append(a)
        return a.ctypes.data

    s = BlockParamsC()
    s.D, s.H, s.Dm = p["D"], p["H"], p["Dm"]
    s.ln1_gamma, s.ln1_beta = arr(p["ln1_gamma"], np.int8), arr(p["ln1_beta"], np.int32)
    s.ln1_b, s.ln1_c = p["ln1_out"]
    s.w_qkv, s.bias_qkv = arr(p["w_qkv"], np.int8), arr(p["bias_qkv"], np.int32)
    s.b_qkv, s.c_qkv = arr(p["b_qkv"], np.int32), arr(p["c_qkv"], np.int32)
    s.logit_b, s.logit_c = p["logit"]
    s.k_s, s.attn_I0, s.attn_M, s.attn_k_out = p["k_s"], p["attn_I0"], p["attn_M"], p["attn_k_out"]
    s.attn_out_b, s.attn_out_c = p["attn_out"]
    s.w_o, s.bias_o = arr(p["w_o"], np.int8), arr(p["bias_o"], np.int32)
    s.b_o, s.c_o = arr(p["b_o"], np.int32), arr(p["c_o"], np.int32)
    s.res1_b_skip, s.res1_b_branch, s.res1_c = p["res1"]
    s.ln2_gamma, s.ln2_beta = arr(p["ln2_gamma"], np.int8), arr(p["ln2_beta"], np.int32)
    s.ln2_b, s.ln2_c = p["ln2_out"]
    s.w1, s.bias1 = arr(p["w1"], np.int8), arr(p["bias1"], np.int32)
    s.b1, s.c1 = arr(p["b1"], np.int32), arr(p["c1"], np.int32)
    s.gelu_I0, s.gelu_M, s.gelu_k_out = p["gelu_I0"], p["gelu_M"], p["gelu_k_out"]
    s.gelu_b, s.gelu_c = p["gelu_out"]
    s.w2, s.bias2 = arr(p["w2"], np.int8), arr(p["bias2"], np.int32)
    s.b2, s.c2 = arr(p["b2"], np.int32), arr(p["c2"], np.int32)
    s.res2_b_skip, s.res2_b_branch, s.res2_c = p["res2"]
    s.ln_F, s.ln_M = p["ln_F"], p["ln_M"]
    return s, keep


# ---------------------------------------------------------------------------
# steps either side of the blocks
# ---------------------------------------------------------------------------

def patch_embed(img, P: int, W, bias, b, c, cls, pos, add):
    """img [B x C x Hi x Wi] int8 -> tokens [B*(Np+1) x D] int8.

    Flattened P x P patches through an int8 linear layer (W [D x C*P*P]),
    the class token first, then the position embedding added with the
    two-scale dyadic pair ``add`` = (b_u, b_v, c)."""
    img = np.ascontiguousarray(img, dtype=np.int8)
    B, Cin, Hi, Wi = img.shape
    W = np.ascontiguousarray(W, dtype=np.int8)
    D = W.shape[0]
    assert W.shape[1] == Cin * P * P and Hi % P == 0 and Wi % P == 0
    Np = (Hi // P) * (Wi // P)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.int32)
    b = np.ascontiguousarray(b, dtype=np.int32)
    c = np.ascontiguousarray(c, dtype=np.int32)
    cls = np.ascontiguousarray(cls, dtype=np.int8)
    pos = np.ascontiguousarray(pos, dtype=np.int8)
    assert cls.shape == (D,) and pos.shape == (Np + 1, D)
    x = np.zeros((B * (Np + 1), D), dtype=np.int8)
    if lib().orc_patch_embed(img.ctypes.data, B, Cin, Hi, Wi, P, W.ctypes.data,
                             None if bias is None else bias.ctypes.data, b.ctypes.data, c.ctypes.data, D,
                             cls.ctypes.data, pos.ctypes.data, int(add[0]), int(add[1]), int(add[2]),
                             x.ctypes.data) != 0:
        raise MemoryError("orc_patch_embed")
    return x


def head(x, B: int, Ntok: int, gamma, beta, F: int, M_ln: int, ln_out, W, bias, b, c):
    """x [B*Ntok x D] int8 -> logits [B x Ncls] int8 (class token, LN, linear)."""
    x = np.ascontiguousarray(x, dtype=np.int8)
    D = x.shape[1]
    W = np.ascontiguousarray(W, dtype=np.int8)
    Ncls = W.shape[0]
    gamma = np.ascontiguousarray(gamma, dtype=np.int8)
    beta = np.ascontiguousarray(beta, dtype=np.int32)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.int32)
    b = np.ascontiguousarray(b, dtype=np.int32)
    c = np.ascontiguousarray(c, dtype=np.int32)
    out = np.zeros((B, Ncls), dtype=np.int8)
    if lib().orc_head(x.ctypes.data, B, Ntok, D, gamma.ctypes.data, beta.ctypes.data, int(F), int(M_ln),
                      int(ln_out[0]), int(ln_out[1]), W.ctypes.data, Ncls,
                      None if bias is None else bias.ctypes.data, b.ctypes.data, c.ctypes.data,
                      out.ctypes.data) != 0:
        raise MemoryError("orc_head")
    return out



def model_params(mc, **consts):
    """The oracle's own integer parameters of a whole model (``synthetic.ModelCase``):
    per-channel DN for the patch projection and the classifier, the DN pair
    (S_e / S_x, S_pos / S_x) for the position term, DN(S_gamma 2^-F / S_ln) for
    the head's I-LayerNorm; the blocks as ``block_params``."""
    S = mc.scales
    ln_F = consts.get("ln_F", 7)
    ln_M = consts.get("ln_M", 23)
    D = mc.w_pe.shape[0]

    def per_channel(s_in, s_w, s_out):
        bc = [dyadic(s_in * float(sw) / float(s_out)) for sw in s_w]
        return (np.array([x[0] for x in bc], dtype=np.int32), np.array([x[1] for x in bc], dtype=np.int32))

    m = dict(P=mc.P, ln_F=ln_F, ln_M=ln_M)
    m["b_pe"], m["c_pe"] = per_channel(S["img"], mc.s_w_pe, S["e"])
    m["pos_add"] = dyadic_pair(S["e"] / S["x"], S["pos"] / S["x"])
    m["head_ln_out"] = dyadic(S["head_gamma"] * 2.0 ** -ln_F / S["head_ln"])
    m["b_head"], m["c_head"] = per_channel(S["head_ln"], mc.s_w_head, S["logits"])
    m["blocks"] = [block_params(q, **{k: v for k, v in consts.items() if k != "ln_M"}, ln_M=ln_M)
                   for q in mc.wl.blocks]
    return m


def model_forward(m, mc, images=None):
    """Oracle logits [len(images) x Ncls_pad] of the model on the chosen images
    (default: all) of ``mc.img``: patch embedding, every block, the head
    (every linear layer rounds half up when m["linear_round"] is set)."""
    if m.get("linear_round", 0):
        with linear_rounding(1):
            return _model_forward(m, mc, images)
    return _model_forward(m, mc, images)


def _model_forward(m, mc, images=None):
    img = mc.img if images is None else mc.img[list(images)]
    B = img.shape[0]
    x = patch_embed(img, mc.P, mc.w_pe, mc.bias_pe, m["b_pe"], m["c_pe"], mc.cls, mc.pos, m["pos_add"])
    Ntok = x.shape[0] // B
    for p in m["blocks"]:
        x = block_forward(p, x, B, Ntok)
    return head(x, B, Ntok, mc.head_gamma, mc.head_beta, m["ln_F"], m["ln_M"], m["head_ln_out"], mc.w_head,
                mc.bias_head, m["b_head"], m["c_head"])
