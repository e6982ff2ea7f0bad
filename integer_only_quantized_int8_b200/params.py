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

from . import (BlockParams, Dyadic, Residual, ivit_dyadic_from_double, ivit_i0_from_scale,
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
    return DeviceBlockParams(tensors=t, c=s, host=p)
