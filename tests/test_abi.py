"""Host-side checks of the C ABI (no compute call needs a GPU here).

- the shared library loads and exports every entry point include/ivit.h declares;
- the host parameter helpers agree with the oracle's own implementations;
- argument validation rejects bad calls before anything is enqueued;
- the product parameter builder equals the oracle's, field by field.
"""
import math
import os
import re

import numpy as np
import pytest
import torch

import integer_only_quantized_int8_b200 as ivit
import oracle
import synthetic
from integer_only_quantized_int8_b200 import build as ivit_build
from integer_only_quantized_int8_b200 import params as ivit_params

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    ivit_build.build()


def _declared():
    src = "".join(open(os.path.join(ROOT, "include", h)).read()
                  for h in sorted(os.listdir(os.path.join(ROOT, "include"))) if h.endswith(".h"))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ivit_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    import ctypes
    L = ctypes.CDLL(ivit.library_path)
    decl = _declared()
    assert len(decl) >= 12
    for name in decl:
        assert hasattr(L, name), name
    assert sorted(decl) == sorted(ivit.EXPORTED_SYMBOLS)


def test_status_strings():
    assert ivit.ivit_status_string(0) == "IVIT_OK"
    assert ivit.ivit_status_string(4) == "IVIT_ERR_TIMEOUT"


def test_dyadic_helper_matches_oracle():
    r = np.random.default_rng(20)
    for s in np.exp(r.uniform(math.log(2.0 ** -24), math.log(2.0 ** 12), size=5000)):
        assert ivit.ivit_dyadic_from_double(s) == oracle.dyadic(s)
    for s in (0.0, 0.5, 1.0, 3.0, 2.0 ** 30):
        assert ivit.ivit_dyadic_from_double(s) == oracle.dyadic(s)
    for bad in (-1.0, float("nan"), float("inf"), 2.0 ** 31):
        with pytest.raises(ivit.IvitError):
            ivit.ivit_dyadic_from_double(bad)


def test_residual_and_i0_helpers_match_oracle():
    r = np.random.default_rng(21)
    for s1, s2 in np.exp(r.uniform(-8, 4, size=(2000, 2))):
        assert ivit.ivit_residual_from_double(s1, s2) == oracle.dyadic_pair(s1, s2)
    for S in np.exp(r.uniform(-12, 3, size=2000)):
        assert ivit.ivit_i0_from_scale(S) == oracle.recip_i0(S)
    with pytest.raises(ivit.IvitError):
        ivit.ivit_i0_from_scale(0.0)


def test_validation_rejects_before_launch():
    import ctypes as C
    L = ivit.lib()
    none = ivit.Residual(0, 0, 0)
    # null pointers
    assert L.ivit_linear_requant(None, 16, 16, None, 16, None, None, None, 8, 0, None, none, None, None) == 1
    # misaligned pointer (odd address) and bad shapes; no device pointer is touched
    p = 0x1000
    assert L.ivit_linear_requant(p + 1, 16, 16, p, 16, None, p, p, 8, 0, None, none, p, None) == 1
    assert L.ivit_linear_requant(p, 16, 24, p, 16, None, p, p, 8, 0, None, none, p, None) == 1   # K % 16
    assert L.ivit_linear_requant(p, 16, 16, p, 16, None, p, p, 9, 0, None, none, p, None) == 1   # out_bits
    assert L.ivit_linear_requant(p, 16, 16, p, 16, None, p, p, 8, 2, None, none, p, None) == 1   # rounding mode
    d = ivit.Dyadic(1, 0)
    assert L.ivit_attention(p, 1, 8, 1, d, 17, 4, 30, 8, d, p, None) == 1     # k_s > 16
    # patch embedding: null image, patch size not dividing the image, C P P not a multiple of 16
    assert L.ivit_patch_embed(None, 1, 3, 32, 32, 16, p, 64, None, p, p, 0, p, p, none, p, 1 << 20, p, None) == 1
    assert L.ivit_patch_embed(p, 1, 3, 40, 32, 16, p, 64, None, p, p, 0, p, p, none, p, 1 << 20, p, None) == 1
    assert L.ivit_patch_embed(p, 1, 3, 28, 28, 14, p, 64, None, p, p, 0, p, p, none, p, 1 << 20, p, None) == 1
    assert L.ivit_patch_embed(p, 1, 3, 32, 32, 16, p, 64, None, p, p, 0, p, p, none, p, 16, p, None) == 1  # workspace
    # head: class count not a multiple of 16, width past 2048
    assert L.ivit_head(p, 1, 3, 64, p, p, 7, 23, d, p, 1000, None, p, p, 0, p, 1 << 20, p, None) == 1
    assert L.ivit_head(p, 1, 3, 4096, p, p, 7, 23, d, p, 1008, None, p, p, 0, p, 1 << 20, p, None) == 1
    assert L.ivit_attention(p, 1, 300, 1, d, 12, 4, 30, 8, d, p, None) == 2   # wide logits past 256 keys
    assert L.ivit_attention(p, 1, 8, 1, d, 16, 50000, 30, 8, d, p, None) == 2  # n_max * I0 >= 2^32
    assert L.ivit_attention(p, 1, 8, 1, d, 8, 0, 30, 8, d, p, None) == 1      # I0 < 1
    assert L.ivit_attention(p, 1, 8, 1, d, 8, 4, 31, 8, d, p, None) == 1      # M > 30
    assert L.ivit_attention(p, 1, 641, 1, d, 8, 4, 30, 8, d, p, None) == 2    # too many keys
    assert L.ivit_attention(p, 1, 8, 1, ivit.Dyadic(1, 32), 8, 4, 30, 8, d, p, None) == 1
    assert L.ivit_layernorm(p, 4, 24, p, p, 7, 23, d, p, None) == 1          # cols % 16
    assert L.ivit_layernorm(p, 4, 32, p, p, 7, 24, d, p, None) == 1          # M_ln > 23
    assert L.ivit_shiftgelu(p, 16, 0, 30, 8, d, p, None) == 1
    # empty inputs are a successful no-op that touches nothing
    assert L.ivit_shiftgelu(None, 0, 4, 30, 8, d, None, None) == 0
    assert L.ivit_layernorm(None, 0, 32, None, None, 7, 23, d, None, None) == 0


def test_product_model_params_equal_oracle_model_params():
    """Patch embedding, position add, head and every block: the library's host
    helpers and the oracle derive the same integers (no GPU involved)."""
    mc = synthetic.model_case(B=2, Hi=32, Wi=48, P=16, D=192, H=3, Dm=768, blocks=2, Ncls=100, seed=4)
    a = ivit_params.model_integer_params(mc)
    b = oracle.model_params(mc)
    for k in ("b_pe", "c_pe", "b_head", "c_head"):
        np.testing.assert_array_equal(np.asarray(a[k], np.int64), np.asarray(b[k], np.int64), err_msg=k)
    assert tuple(a["pos_add"]) == tuple(b["pos_add"])
    assert tuple(a["head_ln_out"]) == tuple(b["head_ln_out"])
    assert (a["ln_F"], a["ln_M"], a["P"]) == (b["ln_F"], b["ln_M"], b["P"])
    assert len(a["blocks"]) == len(b["blocks"]) == 2
    for qa, qb in zip(a["blocks"], b["blocks"]):
        for k, v in qb.items():
            if isinstance(v, np.ndarray):
                np.testing.assert_array_equal(np.asarray(qa[k]).astype(np.int64), v.astype(np.int64), err_msg=k)
            else:
                assert tuple(np.atleast_1d(qa[k])) == tuple(np.atleast_1d(v)), k


def _read(ptr, like):
    """The bytes at a host address, as an array shaped like `like`."""
    import ctypes as C
    a = np.asarray(like)
    raw = (C.c_char * a.nbytes).from_address(ptr)
    return np.frombuffer(bytes(raw), dtype=a.dtype).reshape(a.shape)


def test_parameter_structs_point_at_the_right_tables():
    """params.to_device / model_to_device on host memory: every pointer of the
    C structs reads back its own table, and every scalar is the dict's."""
    mc = synthetic.model_case(B=2, Hi=32, Wi=32, P=16, D=128, H=2, Dm=256, blocks=2, Ncls=40, seed=6)
    m = ivit_params.model_integer_params(mc)
    m["linear_round"] = 1
    for blk in m["blocks"]:
        blk["linear_round"] = 1
    dm = ivit_params.model_to_device(m, "cpu")
    s = dm.c
    assert (s.C, s.P, s.D, s.n_blocks, s.Ncls) == (m["C"], m["P"], m["D"], 2, m["Ncls_pad"])
    assert (s.pos_add.b_skip, s.pos_add.b_branch, s.pos_add.c) == tuple(m["pos_add"])
    assert (s.head_ln_out.b, s.head_ln_out.c) == tuple(m["head_ln_out"])
    assert (s.head_ln_F, s.head_ln_M, s.linear_round) == (m["ln_F"], m["ln_M"], 1)
    for name, dt in (("w_pe", np.int8), ("bias_pe", np.int32), ("b_pe", np.int32), ("c_pe", np.int8),
                     ("cls", np.int8), ("pos", np.int8), ("head_gamma", np.int8), ("head_beta", np.int32),
                     ("w_head", np.int8), ("bias_head", np.int32), ("b_head", np.int32), ("c_head", np.int8)):
        want = np.asarray(m[name]).astype(dt)
        np.testing.assert_array_equal(_read(getattr(s, name), want), want, err_msg=name)
    for i, p in enumerate(m["blocks"]):
        bs = s.blocks[i]
        assert (bs.D, bs.H, bs.Dm) == (p["D"], p["H"], p["Dm"])
        for f in ("ln1_out", "ln2_out", "logit", "attn_out", "gelu_out"):
            assert (getattr(bs, f).b, getattr(bs, f).c) == tuple(p[f]), f
        for f in ("res1", "res2"):
            r = getattr(bs, f)
            assert (r.b_skip, r.b_branch, r.c) == tuple(p[f]), f
        for f in ("k_s", "attn_I0", "attn_M", "attn_k_out", "gelu_I0", "gelu_M", "gelu_k_out", "ln_F", "ln_M",
                  "linear_round"):
            assert getattr(bs, f) == p[f], f
        for name, dt in ivit_params._TENSORS.items():
            want = np.asarray(p[name]).astype({torch.int8: np.int8, torch.int32: np.int32}[dt])
            np.testing.assert_array_equal(_read(getattr(bs, name), want), want, err_msg=f"block {i} {name}")


def test_block_checks_every_pointer_before_launch():
    """ivit_block_forward refuses a misaligned activation or parameter pointer
    with nothing enqueued.  The baseline call is valid except that it asks for
    12-bit logits over 300 keys, which the host refuses as unsupported after
    every pointer check, so no call here reaches a launch on any machine."""
    import ctypes as C
    L = ivit.lib()
    ptr_fields = [name for name, t in ivit.BlockParams._fields_ if t is C.c_void_p]
    base = 0x100000

    def params(**over):
        p = ivit.BlockParams()
        p.D, p.H, p.Dm = 64, 1, 256
        for i, f in enumerate(ptr_fields):
            setattr(p, f, base + 0x1000 * (i + 1))
        p.ln1_out = p.ln2_out = p.logit = p.attn_out = p.gelu_out = ivit.Dyadic(1, 0)
        p.k_s, p.attn_I0, p.attn_M, p.attn_k_out = 12, 4, 30, 8
        p.gelu_I0, p.gelu_M, p.gelu_k_out = 4, 30, 8
        p.res1 = p.res2 = ivit.Residual(1, 1, 1)
        p.ln_F, p.ln_M, p.linear_round = 7, 23, 0
        for k, v in over.items():
            setattr(p, k, v)
        return p

    B, N = 1, 300
    x, y, ws = 0x1000000, 0x2000000, 0x3000000
    ws_bytes = ivit.ivit_block_workspace_bytes(B, N, 64, 256)

    def call(p, xx=x, yy=y):
        return L.ivit_block_forward(C.byref(p), xx, yy, ws, ws_bytes, B, N, None)

    assert call(params()) == 2                      # every pointer passes; the attention shape does not
    assert call(params(), xx=x + 8) == 1            # misaligned input
    assert call(params(), yy=y + 4) == 1            # misaligned output
    for f in ptr_fields:
        good = getattr(params(), f)
        assert call(params(**{f: good + 1})) == 1, f  # misaligned parameter
        if f.startswith("bias"):
            assert call(params(**{f: None})) == 2, f  # the biases are optional
        else:
            assert call(params(**{f: None})) == 1, f  # the rest are not


def test_empty_batches_are_no_ops_on_every_entry_point():
    """B = 0 (or N = 0) returns IVIT_OK after the argument checks, touches no
    memory and needs no device, for the block, attention, patch embedding
    and head as for the elementwise operators."""
    import ctypes as C
    L = ivit.lib()
    p = 0x100000
    d = ivit.Dyadic(1, 0)
    none = ivit.Residual(0, 0, 0)
    blk = ivit.BlockParams()
    blk.D, blk.H, blk.Dm = 64, 1, 256
    assert L.ivit_block_forward(C.byref(blk), p, p + 0x1000, p + 0x2000, 0, 0, 197, None) == 0
    assert L.ivit_block_forward(C.byref(blk), p, p + 0x1000, p + 0x2000, 0, 4, 0, None) == 0
    assert L.ivit_attention(p, 0, 197, 12, d, 8, 4, 30, 8, d, p, None) == 0
    assert L.ivit_attention(p, 3, 0, 12, d, 8, 4, 30, 8, d, p, None) == 0
    assert L.ivit_patch_embed(p, 0, 3, 32, 32, 16, p, 64, None, p, p, 0, p, p, none, p, 1 << 20, p, None) == 0
    assert L.ivit_head(p, 0, 5, 64, p, p, 7, 23, d, p, 32, None, p, p, 0, p, 1 << 20, p, None) == 0
    # an empty batch still gets its arguments checked
    assert L.ivit_block_forward(C.byref(blk), p, p, p + 0x2000, 0, 0, 197, None) == 1     # x aliases y
    assert L.ivit_attention(p, 0, 197, 12, d, 17, 4, 30, 8, d, p, None) == 1              # k_s > 16


def test_workspace_bytes():
    assert ivit.ivit_block_workspace_bytes(0, 197, 768, 3072) == 0
    T, D, Dm = 64 * 197, 768, 3072
    up = lambda v: (v + 255) // 256 * 256
    assert ivit.ivit_block_workspace_bytes(64, 197, D, Dm) == up(T * D) * 3 + up(T * 3 * D) + up(T * Dm)


def test_product_params_equal_oracle_params():
    wl = synthetic.make_workload(B=2, N=9, D=192, H=3, Dm=768, blocks=2, seed=2, n_cal=2,
                                 tails="laplace")
    for q in wl.blocks:
        a = ivit_params.integer_params(q)
        b = oracle.block_params(q)
        assert set(b) <= set(a)
        for k, v in b.items():
            if isinstance(v, np.ndarray):
                np.testing.assert_array_equal(np.asarray(a[k]).astype(np.int64), v.astype(np.int64), err_msg=k)
            else:
                assert tuple(np.atleast_1d(a[k])) == tuple(np.atleast_1d(v)), k
