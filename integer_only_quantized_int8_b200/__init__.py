"""Integer-only ViT encoder block (I-ViT) on B200: Python binding.

A thin ctypes layer over ``libivit_b200.so`` (the C ABI in ``include/ivit.h``).
Functions keep the C names and only marshal arguments: torch tensors become
device pointers, ``stream=None`` becomes torch's current CUDA stream, and a
non-OK status raises :class:`IvitError`.  Every operator runs in the library's
CUDA kernels; there is no fallback path.  If the shared library has not been
built, importing works but the first call raises (build it with
``python -m integer_only_quantized_int8_b200.build``).
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

__all__ = [
    "IvitError", "lib", "library_path", "Dyadic", "Residual", "BlockParams",
    "ivit_status_string", "ivit_dyadic_from_double", "ivit_residual_from_double", "ivit_i0_from_scale",
    "ivit_linear_requant", "ivit_linear_shiftgelu", "ivit_attention", "ivit_shiftgelu", "ivit_layernorm",
    "ivit_block_workspace_bytes", "ivit_block_forward", "ivit_stream_status", "ivit_launch_count",
    "ivit_block_forward_static", "STATIC_SCRATCH_BYTES", "EXPORTED_SYMBOLS",
    "ModelParams", "ivit_patch_embed_workspace_bytes", "ivit_patch_embed", "ivit_head_workspace_bytes", "ivit_head",
    "ivit_model_workspace_bytes", "ivit_model_forward", "ivit_selftest_wait_timeout", "ivit_selftest_int_rate",
    "ivit_shiftgelu_rowmax", "ivit_attention_lis", "ivit_layernorm_ptf", "ivit_selftest_withhold",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libivit_b200.so")
_lock = threading.Lock()
_lib = None

EXPORTED_SYMBOLS = (
    "ivit_status_string", "ivit_dyadic_from_double", "ivit_residual_from_double", "ivit_i0_from_scale",
    "ivit_linear_requant", "ivit_linear_shiftgelu", "ivit_attention", "ivit_shiftgelu", "ivit_layernorm",
    "ivit_block_workspace_bytes",
    "ivit_block_forward", "ivit_stream_status", "ivit_launch_count",
    "ivit_block_forward_static",
    "ivit_patch_embed_workspace_bytes", "ivit_patch_embed", "ivit_head_workspace_bytes", "ivit_head",
    "ivit_model_workspace_bytes", "ivit_model_forward",
    "ivit_selftest_wait_timeout", "ivit_selftest_int_rate",
    "ivit_shiftgelu_rowmax", "ivit_attention_lis", "ivit_layernorm_ptf", "ivit_selftest_withhold",
)

_STATUS = {0: "IVIT_OK", 1: "IVIT_ERR_INVALID_ARG", 2: "IVIT_ERR_UNSUPPORTED", 3: "IVIT_ERR_CUDA",
           4: "IVIT_ERR_TIMEOUT", 5: "IVIT_ERR_INTERNAL"}


class IvitError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)}")


class Dyadic(C.Structure):
    _fields_ = [("b", C.c_int32), ("c", C.c_int32)]


class Residual(C.Structure):
    _fields_ = [("b_skip", C.c_int32), ("b_branch", C.c_int32), ("c", C.c_int32)]


class BlockParams(C.Structure):
    """Mirror of ``ivit_block_params``."""
    _fields_ = [
        ("D", C.c_int32), ("H", C.c_int32), ("Dm", C.c_int32),
        ("ln1_gamma", C.c_void_p), ("ln1_beta", C.c_void_p), ("ln1_out", Dyadic),
        ("w_qkv", C.c_void_p), ("bias_qkv", C.c_void_p), ("b_qkv", C.c_void_p), ("c_qkv", C.c_void_p),
        ("logit", Dyadic), ("k_s", C.c_int32), ("attn_I0", C.c_int32), ("attn_M", C.c_int32),
        ("attn_k_out", C.c_int32), ("attn_out", Dyadic),
        ("w_o", C.c_void_p), ("bias_o", C.c_void_p), ("b_o", C.c_void_p), ("c_o", C.c_void_p),
        ("res1", Residual),
        ("ln2_gamma", C.c_void_p), ("ln2_beta", C.c_void_p), ("ln2_out", Dyadic),
        ("w1", C.c_void_p), ("bias1", C.c_void_p), ("b1", C.c_void_p), ("c1", C.c_void_p),
        ("gelu_I0", C.c_int32), ("gelu_M", C.c_int32), ("gelu_k_out", C.c_int32), ("gelu_out", Dyadic),
        ("w2", C.c_void_p), ("bias2", C.c_void_p), ("b2", C.c_void_p), ("c2", C.c_void_p),
        ("res2", Residual),
        ("ln_F", C.c_int32), ("ln_M", C.c_int32),
        ("linear_round", C.c_int32),
    ]


class ModelParams(C.Structure):
    """Mirror of ``ivit_model_params`` (``blocks`` points at a ctypes array of
    :class:`BlockParams` that the caller keeps alive)."""
    _fields_ = [
        ("C", C.c_int32), ("P", C.c_int32), ("D", C.c_int32), ("n_blocks", C.c_int32), ("Ncls", C.c_int32),
        ("w_pe", C.c_void_p), ("bias_pe", C.c_void_p), ("b_pe", C.c_void_p), ("c_pe", C.c_void_p),
        ("cls", C.c_void_p), ("pos", C.c_void_p), ("pos_add", Residual),
        ("blocks", C.POINTER(BlockParams)),
        ("head_gamma", C.c_void_p), ("head_beta", C.c_void_p), ("head_ln_F", C.c_int32), ("head_ln_M", C.c_int32),
        ("head_ln_out", Dyadic),
        ("w_head", C.c_void_p), ("bias_head", C.c_void_p), ("b_head", C.c_void_p), ("c_head", C.c_void_p),
        ("linear_round", C.c_int32),
    ]


def lib() -> C.CDLL:
    """Load the shared library (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise RuntimeError(f"{library_path} is missing: build it with "
                                   "`python -m integer_only_quantized_int8_b200.build`")
            L = C.CDLL(library_path)
            i32, i64, vp = C.c_int32, C.c_int64, C.c_void_p
            L.ivit_status_string.restype = C.c_char_p
            L.ivit_status_string.argtypes = [C.c_int]
            L.ivit_dyadic_from_double.restype = C.c_int
            L.ivit_dyadic_from_double.argtypes = [C.c_double, C.POINTER(Dyadic)]
            L.ivit_residual_from_double.restype = C.c_int
            L.ivit_residual_from_double.argtypes = [C.c_double, C.c_double, C.POINTER(Residual)]
            L.ivit_i0_from_scale.restype = C.c_int
            L.ivit_i0_from_scale.argtypes = [C.c_double, C.POINTER(C.c_int32)]
            L.ivit_linear_requant.restype = C.c_int
            L.ivit_linear_requant.argtypes = [vp, i64, i32, vp, i32, vp, vp, vp, i32, i32, vp, Residual, vp, vp]
            L.ivit_linear_shiftgelu.restype = C.c_int
            L.ivit_linear_shiftgelu.argtypes = [vp, i64, i32, vp, i32, vp, vp, vp, i32, i32, i32, i32, Dyadic, vp, vp]
            L.ivit_attention.restype = C.c_int
            L.ivit_attention.argtypes = [vp, i32, i32, i32, Dyadic, i32, i32, i32, i32, Dyadic, vp, vp]
            L.ivit_shiftgelu.restype = C.c_int
            L.ivit_shiftgelu.argtypes = [vp, i64, i32, i32, i32, Dyadic, vp, vp]
            L.ivit_layernorm.restype = C.c_int
            L.ivit_layernorm.argtypes = [vp, i64, i32, vp, vp, i32, i32, Dyadic, vp, vp]
            L.ivit_block_workspace_bytes.restype = C.c_size_t
            L.ivit_block_workspace_bytes.argtypes = [i32, i32, i32, i32]
            L.ivit_block_forward.restype = C.c_int
            L.ivit_block_forward.argtypes = [C.POINTER(BlockParams), vp, vp, vp, C.c_size_t, i32, i32, vp]
            L.ivit_block_forward_static.restype = C.c_int
            L.ivit_block_forward_static.argtypes = [C.POINTER(BlockParams), vp, vp, i32, i32, vp]
            L.ivit_patch_embed_workspace_bytes.restype = C.c_size_t
            L.ivit_patch_embed_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
            L.ivit_patch_embed.restype = C.c_int
            L.ivit_patch_embed.argtypes = [vp, i32, i32, i32, i32, i32, vp, i32, vp, vp, vp, i32, vp, vp, Residual,
                                           vp, C.c_size_t, vp, vp]
            L.ivit_head_workspace_bytes.restype = C.c_size_t
            L.ivit_head_workspace_bytes.argtypes = [i32, i32]
            L.ivit_head.restype = C.c_int
            L.ivit_head.argtypes = [vp, i32, i32, i32, vp, vp, i32, i32, Dyadic, vp, i32, vp, vp, vp, i32, vp,
                                    C.c_size_t, vp, vp]
            L.ivit_model_workspace_bytes.restype = C.c_size_t
            L.ivit_model_workspace_bytes.argtypes = [C.POINTER(ModelParams), i32, i32, i32]
            L.ivit_model_forward.restype = C.c_int
            L.ivit_model_forward.argtypes = [C.POINTER(ModelParams), vp, i32, i32, i32, vp, C.c_size_t, vp, vp]
            L.ivit_stream_status.restype = C.c_int
            L.ivit_stream_status.argtypes = [vp]
            L.ivit_launch_count.restype = C.c_uint64
            L.ivit_launch_count.argtypes = []
            L.ivit_selftest_wait_timeout.restype = C.c_int
            L.ivit_selftest_wait_timeout.argtypes = [vp]
            L.ivit_shiftgelu_rowmax.restype = C.c_int
            L.ivit_shiftgelu_rowmax.argtypes = [vp, i64, i32, i32, i32, i32, Dyadic, vp, vp]
            L.ivit_attention_lis.restype = C.c_int
            L.ivit_attention_lis.argtypes = [vp, i32, i32, i32, Dyadic, i32, i32, i32, Dyadic, vp, vp]
            L.ivit_layernorm_ptf.restype = C.c_int
            L.ivit_layernorm_ptf.argtypes = [vp, i64, i32, vp, vp, vp, i32, i32, Dyadic, vp, vp]
            L.ivit_selftest_withhold.restype = C.c_int
            L.ivit_selftest_withhold.argtypes = [i32, i32]
            L.ivit_selftest_int_rate.restype = C.c_int
            L.ivit_selftest_int_rate.argtypes = [i32, vp, i32, C.POINTER(C.c_int64), vp]
            _lib = L
    return _lib


def _check(fn: str, st: int):
    if st != 0:
        raise IvitError(fn, st)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t, dtype, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    return t.data_ptr()


def _holds(n: int, **tensors):
    """Each given tensor must hold at least n elements: the library reads or
    writes that many through its pointer."""
    for name, t in tensors.items():
        if t is not None and t.numel() < n:
            raise ValueError(f"{name} holds {t.numel()} elements, needs {n}")


def _dy(d) -> Dyadic:
    return d if isinstance(d, Dyadic) else Dyadic(int(d[0]), int(d[1]))


def _res(r) -> Residual:
    if r is None:
        return Residual(0, 0, 0)
    return r if isinstance(r, Residual) else Residual(int(r[0]), int(r[1]), int(r[2]))


# ---------------------------------------------------------------------------
# host-side parameter helpers
# ---------------------------------------------------------------------------

def ivit_status_string(status: int) -> str:
    return lib().ivit_status_string(int(status)).decode()


def ivit_dyadic_from_double(s: float):
    d = Dyadic()
    _check("ivit_dyadic_from_double", lib().ivit_dyadic_from_double(float(s), C.byref(d)))
    return int(d.b), int(d.c)


def ivit_residual_from_double(s_skip: float, s_branch: float):
    r = Residual()
    _check("ivit_residual_from_double", lib().ivit_residual_from_double(float(s_skip), float(s_branch), C.byref(r)))
    return int(r.b_skip), int(r.b_branch), int(r.c)


def ivit_i0_from_scale(S: float) -> int:
    v = C.c_int32()
    _check("ivit_i0_from_scale", lib().ivit_i0_from_scale(float(S), C.byref(v)))
    return int(v.value)


# ---------------------------------------------------------------------------
# operators
# ---------------------------------------------------------------------------

def ivit_linear_requant(X, W, bias, b, c, Y, out_bits: int = 8, skip=None, res=None, stream=None, rounding: int = 0):
    """Y = sat((b_j (X W^T + bias)_ij) >> c_j) [+ residual]; X [M,K], W [N,K], Y [M,N] int8
    (rounding 1: the requant rounds half up)."""
    M, K = X.shape
    N = W.shape[0]
    if W.shape[1] != K or tuple(Y.shape) != (M, N):
        raise ValueError("shape mismatch")
    if skip is not None and tuple(skip.shape) != (M, N):
        raise ValueError("skip shape mismatch")
    _holds(N, bias=bias, b=b, c=c)
    st = lib().ivit_linear_requant(_ptr(X, torch.int8, "X"), M, K, _ptr(W, torch.int8, "W"), N,
                                   _ptr(bias, torch.int32, "bias"), _ptr(b, torch.int32, "b"),
                                   _ptr(c, torch.int8, "c"), int(out_bits), int(rounding), _ptr(skip, torch.int8, "skip"),
                                   _res(res), _ptr(Y, torch.int8, "Y"), _stream(stream))
    _check("ivit_linear_requant", st)
    return Y


def ivit_linear_shiftgelu(X, W, bias, b, c, gelu_I0: int, gelu_M: int, gelu_k_out: int, gelu_out, Y,
                          stream=None, rounding: int = 0):
    """Y = ShiftGELU(sat_8((b_j (X W^T + bias)_ij) >> c_j)) in one kernel."""
    M, K = X.shape
    N = W.shape[0]
    if W.shape[1] != K or tuple(Y.shape) != (M, N):
        raise ValueError("shape mismatch")
    _holds(N, bias=bias, b=b, c=c)
    st = lib().ivit_linear_shiftgelu(_ptr(X, torch.int8, "X"), M, K, _ptr(W, torch.int8, "W"), N,
                                     _ptr(bias, torch.int32, "bias"), _ptr(b, torch.int32, "b"),
                                     _ptr(c, torch.int8, "c"), int(rounding), int(gelu_I0), int(gelu_M), int(gelu_k_out),
                                     _dy(gelu_out), _ptr(Y, torch.int8, "Y"), _stream(stream))
    _check("ivit_linear_shiftgelu", st)
    return Y


def ivit_attention(qkv, B: int, N: int, H: int, logit, k_s: int, I0: int, M: int, k_out: int, out, ctx,
                   stream=None):
    """ctx [B*N, H*64] from qkv [B*N, 3*H*64] (Shiftmax attention)."""
    if tuple(qkv.shape) != (B * N, 3 * H * 64) or tuple(ctx.shape) != (B * N, H * 64):
        raise ValueError("shape mismatch")
    st = lib().ivit_attention(_ptr(qkv, torch.int8, "qkv"), B, N, H, _dy(logit), int(k_s), int(I0), int(M),
                              int(k_out), _dy(out), _ptr(ctx, torch.int8, "ctx"), _stream(stream))
    _check("ivit_attention", st)
    return ctx


def ivit_shiftgelu(x, I0: int, M: int, k_out: int, out, y, stream=None):
    if x.numel() != y.numel():
        raise ValueError("shape mismatch")
    st = lib().ivit_shiftgelu(_ptr(x, torch.int8, "x"), x.numel(), int(I0), int(M), int(k_out), _dy(out),
                              _ptr(y, torch.int8, "y"), _stream(stream))
    _check("ivit_shiftgelu", st)
    return y


def ivit_layernorm(x, gamma, beta, F: int, M_ln: int, out, y, stream=None):
    rows, cols = x.shape
    if tuple(y.shape) != (rows, cols) or gamma.numel() != cols or beta.numel() != cols:
        raise ValueError("shape mismatch")
    st = lib().ivit_layernorm(_ptr(x, torch.int8, "x"), rows, cols, _ptr(gamma, torch.int8, "gamma"),
                              _ptr(beta, torch.int32, "beta"), int(F), int(M_ln), _dy(out),
                              _ptr(y, torch.int8, "y"), _stream(stream))
    _check("ivit_layernorm", st)
    return y


def ivit_shiftgelu_rowmax(x, I0: int, M: int, k_out: int, out, y, stream=None):
    """ShiftGELU of x [rows, cols] with I_max the row's largest exponent."""
    rows, cols = x.shape
    if tuple(y.shape) != (rows, cols):
        raise ValueError("shape mismatch")
    st = lib().ivit_shiftgelu_rowmax(_ptr(x, torch.int8, "x"), rows, cols, int(I0), int(M), int(k_out), _dy(out),
                                     _ptr(y, torch.int8, "y"), _stream(stream))
    _check("ivit_shiftgelu_rowmax", st)
    return y


def ivit_attention_lis(qkv, B: int, N: int, H: int, logit, k_s: int, I0: int, M: int, out, ctx, stream=None):
    """Attention with Log-Int-Softmax (4-bit log2 attention map, A V by bit shifts)."""
    _holds(int(B) * int(N) * 3 * int(H) * 64, qkv=qkv)
    _holds(int(B) * int(N) * int(H) * 64, ctx=ctx)
    st = lib().ivit_attention_lis(_ptr(qkv, torch.int8, "qkv"), int(B), int(N), int(H), _dy(logit), int(k_s),
                                  int(I0), int(M), _dy(out), _ptr(ctx, torch.int8, "ctx"), _stream(stream))
    _check("ivit_attention_lis", st)
    return ctx


def ivit_layernorm_ptf(x, alpha, gamma, beta, F: int, M_ln: int, out, y, stream=None):
    """I-LayerNorm of x [rows, cols] whose channel i carries the factor 2^alpha[i]."""
    rows, cols = x.shape
    if tuple(y.shape) != (rows, cols) or gamma.numel() != cols or beta.numel() != cols or alpha.numel() != cols:
        raise ValueError("shape mismatch")
    st = lib().ivit_layernorm_ptf(_ptr(x, torch.int8, "x"), rows, cols, _ptr(alpha, torch.uint8, "alpha"),
                                  _ptr(gamma, torch.int8, "gamma"), _ptr(beta, torch.int32, "beta"), int(F),
                                  int(M_ln), _dy(out), _ptr(y, torch.int8, "y"), _stream(stream))
    _check("ivit_layernorm_ptf", st)
    return y


def ivit_block_workspace_bytes(B: int, N: int, D: int, Dm: int) -> int:
    return int(lib().ivit_block_workspace_bytes(int(B), int(N), int(D), int(Dm)))


def ivit_block_forward(params, x, y, workspace, B: int, N: int, stream=None):
    """One encoder block; ``params`` is a :class:`BlockParams` (or an object with ``.c``)."""
    p = params.c if hasattr(params, "c") else params
    _holds(int(B) * int(N) * p.D, x=x, y=y)
    st = lib().ivit_block_forward(C.byref(p), _ptr(x, torch.int8, "x"), _ptr(y, torch.int8, "y"),
                                  _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), int(B), int(N),
                                  _stream(stream))
    _check("ivit_block_forward", st)
    return y


# Bytes of the library's fixed device array (IVIT_STATIC_SCRATCH_BYTES).
STATIC_SCRATCH_BYTES = 32 << 20


def ivit_block_forward_static(params, x, y, B: int, N: int, stream=None):
    """One encoder block without a workspace, for callers that cannot allocate
    device memory (plugins without an allocator, code inside a framework that
    has reserved the whole device, loops that cannot afford cudaMalloc).  The
    intermediates live in the library's own 32 MiB device array, shared by all
    calls on a device: calls that overlap on the GPU race.  Larger batches
    raise IvitError (IVIT_ERR_UNSUPPORTED) before any tensor is looked at."""
    p = params.c if hasattr(params, "c") else params
    if ivit_block_workspace_bytes(B, N, p.D, p.Dm) > STATIC_SCRATCH_BYTES:
        raise IvitError("ivit_block_forward_static", 2)
    _holds(int(B) * int(N) * p.D, x=x, y=y)
    st = lib().ivit_block_forward_static(C.byref(p), _ptr(x, torch.int8, "x"), _ptr(y, torch.int8, "y"), int(B),
                                         int(N), _stream(stream))
    _check("ivit_block_forward_static", st)
    return y


def ivit_stream_status(stream=None) -> int:
    return int(lib().ivit_stream_status(_stream(stream)))


def ivit_launch_count() -> int:
    return int(lib().ivit_launch_count())


def ivit_selftest_wait_timeout(stream=None):
    """Enqueue the diagnostic kernel whose bounded wait runs out (about one
    second); ivit_stream_status() then reports IVIT_ERR_TIMEOUT once."""
    _check("ivit_selftest_wait_timeout", lib().ivit_selftest_wait_timeout(_stream(stream)))


SELFTEST_GEMM = 1
SELFTEST_ATTENTION = 2


def ivit_selftest_withhold(kernel: int, index: int):
    """Make the next launch of a production kernel (SELFTEST_GEMM or
    SELFTEST_ATTENTION) have its first CTA's TMA producer stop before its
    index-th load, so a bounded wait in that kernel runs out (about one
    second): ivit_stream_status() then reports IVIT_ERR_TIMEOUT once."""
    _check("ivit_selftest_withhold", lib().ivit_selftest_withhold(int(kernel), int(index)))


def ivit_selftest_int_rate(iters: int, sink, stream=None) -> int:
    """Enqueue the integer-throughput probe; returns the integer operations
    the launch executes (time it on the stream to get a rate)."""
    ops = C.c_int64(0)
    _check("ivit_selftest_int_rate", lib().ivit_selftest_int_rate(int(iters), _ptr(sink, torch.int32, "sink"),
                                                                  sink.numel(), C.byref(ops), _stream(stream)))
    return int(ops.value)


def ivit_patch_embed_workspace_bytes(B: int, C_in: int, Hi: int, Wi: int, P: int, D: int) -> int:
    return int(lib().ivit_patch_embed_workspace_bytes(int(B), int(C_in), int(Hi), int(Wi), int(P), int(D)))


def ivit_patch_embed(img, P: int, W, bias, b, c, cls, pos, pos_add, workspace, x, stream=None, rounding: int = 0):
    """x [B*(Np+1), D] from img [B, C, Hi, Wi]: patches through W [D, C*P*P],
    the class token first, the position embedding joined by ``pos_add``."""
    B, C_in, Hi, Wi = img.shape
    D = W.shape[0]
    if W.numel() != D * C_in * P * P:
        raise ValueError(f"W must be [D, C*P*P] = [{D}, {C_in * P * P}]")
    Ntok = (Hi // P) * (Wi // P) + 1
    _holds(D, bias=bias, b=b, c=c, cls=cls)
    _holds(Ntok * D, pos=pos)
    _holds(B * Ntok * D, x=x)
    st = lib().ivit_patch_embed(_ptr(img, torch.int8, "img"), B, C_in, Hi, Wi, int(P), _ptr(W, torch.int8, "W"), D,
                                _ptr(bias, torch.int32, "bias"), _ptr(b, torch.int32, "b"), _ptr(c, torch.int8, "c"),
                                int(rounding), _ptr(cls, torch.int8, "cls"), _ptr(pos, torch.int8, "pos"), _res(pos_add),
                                _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _ptr(x, torch.int8, "x"),
                                _stream(stream))
    _check("ivit_patch_embed", st)
    return x


def ivit_head_workspace_bytes(B: int, D: int) -> int:
    return int(lib().ivit_head_workspace_bytes(int(B), int(D)))


def ivit_head(x, B: int, Ntok: int, gamma, beta, F: int, M_ln: int, ln_out, W, bias, b, c, workspace, logits,
              stream=None, rounding: int = 0):
    """logits [B, Ncls] from the class tokens of x [B*Ntok, D]."""
    D = x.shape[1]
    Ncls = W.shape[0]
    if W.shape[1] != D:
        raise ValueError(f"W must be [Ncls, D] with D = {D}")
    _holds(int(B) * int(Ntok) * D, x=x)
    _holds(D, gamma=gamma, beta=beta)
    _holds(Ncls, bias=bias, b=b, c=c)
    _holds(int(B) * Ncls, logits=logits)
    st = lib().ivit_head(_ptr(x, torch.int8, "x"), int(B), int(Ntok), D, _ptr(gamma, torch.int8, "gamma"),
                         _ptr(beta, torch.int32, "beta"), int(F), int(M_ln), _dy(ln_out), _ptr(W, torch.int8, "W"),
                         W.shape[0], _ptr(bias, torch.int32, "bias"), _ptr(b, torch.int32, "b"),
                         _ptr(c, torch.int8, "c"), int(rounding), _ptr(workspace, torch.uint8, "workspace"),
                         workspace.numel(),
                         _ptr(logits, torch.int8, "logits"), _stream(stream))
    _check("ivit_head", st)
    return logits


def ivit_model_workspace_bytes(params, B: int, Hi: int, Wi: int) -> int:
    p = params.c if hasattr(params, "c") else params
    return int(lib().ivit_model_workspace_bytes(C.byref(p), int(B), int(Hi), int(Wi)))


def ivit_model_forward(params, img, workspace, logits, stream=None):
    """logits [B, Ncls] from img [B, C, Hi, Wi]; ``params`` is a
    :class:`ModelParams` (or an object with ``.c``)."""
    p = params.c if hasattr(params, "c") else params
    B, C_in, Hi, Wi = img.shape
    if C_in != p.C:
        raise ValueError(f"img has {C_in} channels, the model {p.C}")
    _holds(B * p.Ncls, logits=logits)
    st = lib().ivit_model_forward(C.byref(p), _ptr(img, torch.int8, "img"), B, Hi, Wi,
                                  _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                  _ptr(logits, torch.int8, "logits"), _stream(stream))
    _check("ivit_model_forward", st)
    return logits
