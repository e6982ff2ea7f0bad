"""Integer parameters of an encoder block, built from real-valued scales.

Off-line host step (not part of the hot path): every multiplier is a dyadic
number DN(ratio of scales) ("I-ViT: Integer-only Quantization for Efficient
Vision Transformer Inference", section 3.2) and every I_0 is round(1 / S)
(section 3.3), both computed by the library's own host helpers
(``ivit_dyadic_from_double``, ``ivit_residual_from_double``,
``ivit_i0_from_scale``).  The result is uploaded once to device memory.
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import numpy as np
import torch

from . import (BlockParams, Dyadic, ModelParams, Residual, ivit_dyadic_from_double, ivit_i0_from_scale,
               ivit_residual_from_double)

# method constants (readings of the pages: M = 30 for IntDiv, 8-bit Shiftmax /
# ShiftGELU outputs, 8-bit logits, F = 7 fractional bits and M_ln = 23 in
# I-LayerNorm)
DEFAULTS = dict(attn_M=30, attn_k_out=8, k_s=8, gelu_M=30, gelu_k_out=8, ln_F=7, ln_M=23)


def _per_channel(s_in: float, s_w: np.ndarray, s_out: np.ndarray):
    bs, cs = [], []
    for sw, so in zip(s_w, s_out):
        b, c = ivit_dyadic_from_double(float(s_in) * float(sw) / float(so))
        bs.append(b)
        cs.append(c)
    return np.asarray(bs, np.int32), np.asarray(cs, np.int8)


def integer_params(q, **consts) -> Dict:
    """Integer parameters (host numpy / ints) of one block from a quantised
    block description with fields D, H, Dm, int8/int32 tensors, per-channel
    weight scales and the activation scales dict ``scales``."""
    k = dict(DEFAULTS)
    k.update(consts)
    S = q.scales
    D, Dm = q.D, q.Dm
    p = dict(D=D, H=q.H, Dm=Dm, **k)
    p["ln1_gamma"], p["ln1_beta"] = q.ln1_gamma, q.ln1_beta
    p["ln1_out"] = ivit_dyadic_from_double(S["gamma1"] * 2.0 ** -k["ln_F"] / S["ln1"])
    qkv_out = np.concatenate([np.full(D, S["q"]), np.full(D, S["k"]), np.full(D, S["v"])])
    p["w_qkv"], p["bias_qkv"] = q.w_qkv, q.bias_qkv
    p["b_qkv"], p["c_qkv"] = _per_channel(S["ln1"], q.s_w_qkv, qkv_out)
    p["logit"] = ivit_dyadic_from_double(S["q"] * S["k"] / (8.0 * S["logit"]))
    p["attn_I0"] = ivit_i0_from_scale(S["logit"])
    p["attn_out"] = ivit_dyadic_from_double(S["v"] * 2.0 ** -(k["attn_k_out"] - 1) / S["ctx"])
    p["w_o"], p["bias_o"] = q.w_o, q.bias_o
    p["b_o"], p["c_o"] = _per_channel(S["ctx"], q.s_w_o, np.full(D, S["o"]))
    p["res1"] = ivit_residual_from_double(S["x"] / S["xh"], S["o"] / S["xh"])
    p["ln2_gamma"], p["ln2_beta"] = q.ln2_gamma, q.ln2_beta
    p["ln2_out"] = ivit_dyadic_from_double(S["gamma2"] * 2.0 ** -k["ln_F"] / S["ln2"])
    p["w1"], p["bias1"] = q.w1, q.bias1
    p["b1"], p["c1"] = _per_channel(S["ln2"], q.s_w1, np.full(Dm, S["h"]))
    p["gelu_I0"] = ivit_i0_from_scale(S["h"])
    p["gelu_out"] = ivit_dyadic_from_double(S["h"] * 2.0 ** -(k["gelu_k_out"] - 1) / S["g"])
    p["w2"], p["bias2"] = q.w2, q.bias2
    p["b2"], p["c2"] = _per_channel(S["g"], q.s_w2, np.full(D, S["f"]))
    p["res2"] = ivit_residual_from_double(S["xh"] / S["y"], S["f"] / S["y"])
    return p


_TENSORS = {
    "ln1_gamma": torch.int8, "ln1_beta": torch.int32, "w_qkv": torch.int8, "bias_qkv": torch.int32,
    "b_qkv": torch.int32, "c_qkv": torch.int8, "w_o": torch.int8, "bias_o": torch.int32, "b_o": torch.int32,
    "c_o": torch.int8, "ln2_gamma": torch.int8, "ln2_beta": torch.int32, "w1": torch.int8, "bias1": torch.int32,
    "b1": torch.int32, "c1": torch.int8, "w2": torch.int8, "bias2": torch.int32, "b2": torch.int32,
    "c2": torch.int8,
}


@dataclasses.dataclass
class DeviceBlockParams:
    """Device copies of one block's tensors plus the ``ivit_block_params`` struct."""
    tensors: Dict[str, torch.Tensor]
    c: BlockParams
    host: Dict


def to_device(p: Dict, device="cuda") -> DeviceBlockParams:
    t = {}
    for name, dt in _TENSORS.items():
        a = np.ascontiguousarray(p[name])
        t[name] = torch.from_numpy(a).to(device=device, dtype=dt).contiguous()
    s = BlockParams()
    s.D, s.H, s.Dm = p["D"], p["H"], p["Dm"]
    for name in _TENSORS:
        setattr(s, name, t[name].data_ptr())
    s.ln1_out = Dyadic(*p["ln1_out"])
    s.ln2_out = Dyadic(*p["ln2_out"])
    s.logit = Dyadic(*p["logit"])
    s.attn_out = Dyadic(*p["attn_out"])
    s.gelu_out = Dyadic(*p["gelu_out"])
    s.k_s, s.attn_I0, s.attn_M, s.attn_k_out = p["k_s"], p["attn_I0"], p["attn_M"], p["attn_k_out"]
    s.gelu_I0, s.gelu_M, s.gelu_k_out = p["gelu_I0"], p["gelu_M"], p["gelu_k_out"]
    s.res1 = Residual(*p["res1"])
    s.res2 = Residual(*p["res2"])
    s.ln_F, s.ln_M = p["ln_F"], p["ln_M"]
    s.linear_round = int(p.get("linear_round", 0))
    return DeviceBlockParams(tensors=t, c=s, host=p)



# ---------------------------------------------------------------------------
# a whole model: patch embedding, blocks, classifier head
# ---------------------------------------------------------------------------

def model_integer_params(mc, **consts) -> Dict:
    """Integer parameters of a whole model from a ``synthetic.ModelCase``-like
    description: the patch projection and the classifier are int8 linear
    layers (per-channel DN of S_in S_w / S_out), the position embedding joins
    the tokens with the DN pair (S_e / S_x, S_pos / S_x), and the head's
    I-LayerNorm output multiplier is DN(S_gamma 2^-F / S_ln)."""
    k = dict(DEFAULTS)
    k.update(consts)
    S = mc.scales
    D = mc.w_pe.shape[0]
    m = dict(P=mc.P, C=mc.img.shape[1], D=D, Ncls_pad=mc.w_head.shape[0], ln_F=k["ln_F"], ln_M=k["ln_M"])
    m["w_pe"], m["bias_pe"] = mc.w_pe, mc.bias_pe
    m["b_pe"], m["c_pe"] = _per_channel(S["img"], mc.s_w_pe, np.full(D, S["e"]))
    m["cls"], m["pos"] = mc.cls, mc.pos
    m["pos_add"] = ivit_residual_from_double(S["e"] / S["x"], S["pos"] / S["x"])
    m["head_gamma"], m["head_beta"] = mc.head_gamma, mc.head_beta
    m["head_ln_out"] = ivit_dyadic_from_double(S["head_gamma"] * 2.0 ** -k["ln_F"] / S["head_ln"])
    m["w_head"], m["bias_head"] = mc.w_head, mc.bias_head
    m["b_head"], m["c_head"] = _per_channel(S["head_ln"], mc.s_w_head, np.full(mc.w_head.shape[0], S["logits"]))
    m["blocks"] = [integer_params(q, **consts) for q in mc.wl.blocks]
    return m


_MODEL_TENSORS = {
    "w_pe": torch.int8, "bias_pe": torch.int32, "b_pe": torch.int32, "c_pe": torch.int8, "cls": torch.int8,
    "pos": torch.int8, "head_gamma": torch.int8, "head_beta": torch.int32, "w_head": torch.int8,
    "bias_head": torch.int32, "b_head": torch.int32, "c_head": torch.int8,
}


@dataclasses.dataclass
class DeviceModelParams:
    """Device copies of a model's tensors, its blocks and the ``ivit_model_params`` struct."""
    tensors: Dict[str, torch.Tensor]
    blocks: list
    block_array: object
    c: ModelParams
    host: Dict


def model_to_device(m: Dict, device="cuda") -> DeviceModelParams:
    t = {}
    for name, dt in _MODEL_TENSORS.items():
        a = np.ascontiguousarray(m[name])
        t[name] = torch.from_numpy(a).to(device=device, dtype=dt).contiguous()
    blocks = [to_device(p, device) for p in m["blocks"]]
    arr = (BlockParams * max(1, len(blocks)))(*[b.c for b in blocks])
    s = ModelParams()
    s.C, s.P, s.D, s.n_blocks, s.Ncls = m["C"], m["P"], m["D"], len(blocks), m["Ncls_pad"]
    for name in ("w_pe", "bias_pe", "b_pe", "c_pe", "cls", "pos", "head_gamma", "head_beta", "w_head", "bias_head",
                 "b_head", "c_head"):
        setattr(s, name, t[name].data_ptr())
    s.pos_add = Residual(*m["pos_add"])
    s.blocks = arr
    s.head_ln_F, s.head_ln_M = m["ln_F"], m["ln_M"]
    s.head_ln_out = Dyadic(*m["head_ln_out"])
    s.linear_round = int(m.get("linear_round", 0))
    return DeviceModelParams(tensors=t, blocks=blocks, block_array=arr, c=s, host=m)
