"""Seeded synthetic inputs for the integer-only ViT block.

This module is shared by the oracle side (tests) and the product side (tests,
bench).  It holds none of the integer method's arithmetic: it draws real-valued
tensors with the shapes and distributions of the ViT workloads, rounds them to
int8/int32 with a plain symmetric rounding, and measures real-valued
calibration statistics (max |value| per tensor) with an ordinary floating-point
ViT block.  Turning those real scales into integer parameters (dyadic
multipliers, I_0) is done separately by each side with its own code.

No dataset or trained weights exist here; ImageNet-shaped inputs are replaced
by Gaussian activations with log-uniform per-channel spread (the inter-channel
variation that FQ-ViT and Trio-ViT describe), and weights by N(0, 0.02^2)
random initialisation.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

try:  # exact GELU for the floating-point calibration model
    from scipy.special import erf as _erf
except Exception:  # pragma: no cover
    _erf = np.vectorize(math.erf)

HEAD_DIM = 64

# The five workloads: (B, N, D, H, Dm, blocks, per-channel std range, logit tails)
CONFIGS: Dict[str, dict] = {
    "deit_t_b1": dict(B=1, N=197, D=192, H=3, Dm=768, blocks=1, chan_std=(0.1, 10.0), tails="normal"),
    "deit_s_b64": dict(B=64, N=197, D=384, H=6, Dm=1536, blocks=1, chan_std=(0.1, 10.0), tails="normal"),
    "vit_b_b64": dict(B=64, N=197, D=768, H=12, Dm=3072, blocks=1, chan_std=(0.1, 20.0), tails="normal"),
    "vit_l_b32_x12": dict(B=32, N=197, D=1024, H=16, Dm=4096, blocks=12, chan_std=(0.1, 10.0), tails="normal"),
    "vit_b384_b16": dict(B=16, N=577, D=768, H=12, Dm=3072, blocks=1, chan_std=(0.1, 10.0), tails="laplace"),
}
CONFIG_ORDER = ["deit_t_b1", "deit_s_b64", "vit_b_b64", "vit_l_b32_x12", "vit_b384_b16"]

# tensor ids for independent sub-streams
_TID = dict(x=1, chan=2, wqkv=3, bqkv=4, wo=5, bo=6, w1=7, b1=8, w2=9, b2=10, g1=11, be1=12, g2=13,
            be2=14, rank1=15, op=16, img=17, wpe=18, bpe=19, cls=20, pos=21, hg=22, hbe=23, whead=24, bhead=25)


def rng(seed: int, tensor: str, block: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), _TID[tensor], int(block)]))


def round_sym(v: np.ndarray, S, lim: int = 127) -> np.ndarray:
    """Round-half-away-from-zero of v / S, clipped to +-lim (symmetric)."""
    t = np.asarray(v, dtype=np.float64) / S
    r = np.copysign(np.floor(np.abs(t) + 0.5), t)
    return np.clip(r, -lim, lim)


def scale_of(v: np.ndarray, bits: int = 8) -> float:
    """Symmetric scale S = 2m / (2^bits - 1) with m = max |v|."""
    m = float(np.max(np.abs(v))) if np.size(v) else 0.0
    m = max(m, 1e-8)
    return 2.0 * m / float((1 << bits) - 1)


def quant_i8(v: np.ndarray, S) -> np.ndarray:
    return round_sym(v, S).astype(np.int8)


def quant_i32(v: np.ndarray, S) -> np.ndarray:
    return round_sym(v, S, lim=2**31 - 1).astype(np.int32)


# ---------------------------------------------------------------------------
# floating-point ViT block used only for calibration statistics
# ---------------------------------------------------------------------------

def _layernorm_f(x, g, b):
    mu = x.mean(-1, keepdims=True)
    var = x.var(-1, keepdims=True)
    return (x - mu) / np.sqrt(var + 1e-6) * g + b


def _gelu_f(x):
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def _attention_f(qkv, B, N, H):
    D = H * HEAD_DIM
    q = qkv[:, :D].reshape(B, N, H, HEAD_DIM).transpose(0, 2, 1, 3)
    k = qkv[:, D:2 * D].reshape(B, N, H, HEAD_DIM).transpose(0, 2, 1, 3)
    v = qkv[:, 2 * D:].reshape(B, N, H, HEAD_DIM).transpose(0, 2, 1, 3)
    logits = q @ k.transpose(0, 1, 3, 2) / math.sqrt(HEAD_DIM)
    p = np.exp(logits - logits.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    ctx = (p @ v).transpose(0, 2, 1, 3).reshape(B * N, D)
    return logits, ctx


# ---------------------------------------------------------------------------
# one quantised block
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class QuantBlock:
    D: int
    H: int
    Dm: int
    ln1_gamma: np.ndarray
    ln1_beta: np.ndarray
    w_qkv: np.ndarray
    bias_qkv: np.ndarray
    s_w_qkv: np.ndarray
    w_o: np.ndarray
    bias_o: np.ndarray
    s_w_o: np.ndarray
    ln2_gamma: np.ndarray
    ln2_beta: np.ndarray
    w1: np.ndarray
    bias1: np.ndarray
    s_w1: np.ndarray
    w2: np.ndarray
    bias2: np.ndarray
    s_w2: np.ndarray
    scales: Dict[str, float]


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    N: int
    D: int
    H: int
    Dm: int
    x: np.ndarray                 # [B*N x D] int8 input of block 0
    blocks: list                  # QuantBlock per block
    ln_F: int = 7
    k_s: int = 8


def _per_channel_weights(w):
    s = np.array([scale_of(row) for row in w])
    return quant_i8(w, s[:, None]), s


def make_workload(name: str = "custom", B: int = 1, N: int = 197, D: int = 192, H: int = 3, Dm: int = 768,
                  blocks: int = 1, chan_std=(0.1, 10.0), tails: str = "normal", seed: int = 0,
                  n_cal: Optional[int] = None, ln_F: int = 7, k_s: int = 8) -> Workload:
    """Seeded synthetic workload: int8 input plus quantised weights of ``blocks`` blocks.

    Real scales of every activation come from a floating-point forward pass of
    the same (dequantised) block on the first ``n_cal`` images.
    """
    assert D == H * HEAD_DIM
    T = B * N
    n_cal = min(B, 8) if n_cal is None else min(B, n_cal)
    lo, hi = chan_std
    sig = np.exp(rng(seed, "chan").uniform(math.log(lo), math.log(hi), size=D))
    x_f = rng(seed, "x").standard_normal((T, D)) * sig[None, :]
    S_x = scale_of(x_f)
    x_i8 = quant_i8(x_f, S_x)
    xin_cal = x_i8[: n_cal * N].astype(np.float64) * S_x       # what block 0 really sees
    S_in = S_x
    out = []
    for blk in range(blocks):
        g = lambda t: rng(seed, t, blk)
        w_qkv = g("wqkv").standard_normal((3 * D, D)) * 0.02
        if tails == "laplace":
            # heavy-tailed logits: Q and K of every head share a rank-1 direction,
            # so q_i . k_j / 8 ~ u_i v_j with u, v ~ N(0, 1) (product-normal tails)
            r = g("rank1")
            for h in range(H):
                a = r.standard_normal(HEAD_DIM)
                a *= math.sqrt(8.0) / np.linalg.norm(a)
                p1 = r.standard_normal(D); p1 /= np.linalg.norm(p1)
                p2 = r.standard_normal(D); p2 /= np.linalg.norm(p2)
                w_qkv[h * HEAD_DIM:(h + 1) * HEAD_DIM] += np.outer(a, p1)
                w_qkv[D + h * HEAD_DIM:D + (h + 1) * HEAD_DIM] += np.outer(a, p2)
        b_qkv = g("bqkv").standard_normal(3 * D) * 0.02
        w_o = g("wo").standard_normal((D, D)) * 0.02
        b_o = g("bo").standard_normal(D) * 0.02
        w1 = g("w1").standard_normal((Dm, D)) * 0.02
        b1 = g("b1").standard_normal(Dm) * 0.02
        w2 = g("w2").standard_normal((D, Dm)) * 0.02
        b2 = g("b2").standard_normal(D) * 0.02
        g1 = 1.0 + 0.1 * g("g1").standard_normal(D)
        be1 = 0.02 * g("be1").standard_normal(D)
        g2 = 1.0 + 0.1 * g("g2").standard_normal(D)
        be2 = 0.02 * g("be2").standard_normal(D)

        wq_qkv, s_qkv = _per_channel_weights(w_qkv)
        wq_o, s_o = _per_channel_weights(w_o)
        wq_1, s_1 = _per_channel_weights(w1)
        wq_2, s_2 = _per_channel_weights(w2)
        S_g1, S_g2 = scale_of(g1), scale_of(g2)
        g1q, g2q = quant_i8(g1, S_g1), quant_i8(g2, S_g2)
        g1d, g2d = g1q * S_g1, g2q * S_g2

        # floating-point forward on the calibration images, dequantised weights
        S = {"x": S_in, "gamma1": S_g1, "gamma2": S_g2}
        xf = xin_cal
        ln1 = _layernorm_f(xf, g1d, be1)
        S["ln1"] = scale_of(ln1)
        qkv = ln1 @ (wq_qkv * s_qkv[:, None]).T + b_qkv
        S["q"], S["k"], S["v"] = scale_of(qkv[:, :D]), scale_of(qkv[:, D:2 * D]), scale_of(qkv[:, 2 * D:])
        logits, ctx = _attention_f(qkv, n_cal, N, H)
        S["logit"] = scale_of(logits, bits=k_s)
        S["ctx"] = scale_of(ctx)
        o = ctx @ (wq_o * s_o[:, None]).T + b_o
        S["o"] = scale_of(o)
        xh = xf + o
        S["xh"] = scale_of(xh)
        ln2 = _layernorm_f(xh, g2d, be2)
        S["ln2"] = scale_of(ln2)
        h = ln2 @ (wq_1 * s_1[:, None]).T + b1
        S["h"] = scale_of(h)
        gg = _gelu_f(h)
        S["g"] = scale_of(gg)
        f = gg @ (wq_2 * s_2[:, None]).T + b2
        S["f"] = scale_of(f)
        y = xh + f
        S["y"] = scale_of(y)

        qb = QuantBlock(
            D=D, H=H, Dm=Dm,
            ln1_gamma=g1q, ln1_beta=quant_i32(be1, S_g1 * 2.0 ** -ln_F),
            w_qkv=wq_qkv, bias_qkv=quant_i32(b_qkv, S["ln1"] * s_qkv), s_w_qkv=s_qkv,
            w_o=wq_o, bias_o=quant_i32(b_o, S["ctx"] * s_o), s_w_o=s_o,
            ln2_gamma=g2q, ln2_beta=quant_i32(be2, S_g2 * 2.0 ** -ln_F),
            w1=wq_1, bias1=quant_i32(b1, S["ln2"] * s_1), s_w1=s_1,
            w2=wq_2, bias2=quant_i32(b2, S["g"] * s_2), s_w2=s_2,
            scales=S)
        out.append(qb)
        # next block sees this block's output at scale S_y
        S_in = S["y"]
        xin_cal = quant_i8(y, S_in).astype(np.float64) * S_in
    return Workload(name=name, B=B, N=N, D=D, H=H, Dm=Dm, x=x_i8, blocks=out, ln_F=ln_F, k_s=k_s)


def workload(name: str, seed: int = 0, **overrides) -> Workload:
    """One of the five named workloads (``CONFIGS``), optionally with overrides (e.g. B)."""
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    return make_workload(name=name, seed=seed, **cfg)


# ---------------------------------------------------------------------------
# standalone operator inputs
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class LinearCase:
    X: np.ndarray
    W: np.ndarray
    bias: np.ndarray
    ratio: np.ndarray            # per output channel: S_in * S_w[j] / S_out
    skip: Optional[np.ndarray] = None
    res_ratio: tuple = (0.0, 0.0)   # (S_skip / S_y, S_branch / S_y)


def linear_case(M: int, K: int, N: int, seed: int = 0, with_skip: bool = False) -> LinearCase:
    r = rng(seed, "op", 1)
    xf = r.standard_normal((M, K))
    S_in = scale_of(xf)
    X = quant_i8(xf, S_in)
    w = r.standard_normal((N, K)) * 0.02
    W, s_w = _per_channel_weights(w)
    bf = r.standard_normal(N) * 0.02
    cal = min(M, 256)
    yf = (X[:cal] * S_in) @ (W * s_w[:, None]).T + bf
    S_out = scale_of(yf)
    case = LinearCase(X=X, W=W, bias=quant_i32(bf, S_in * s_w), ratio=S_in * s_w / S_out)
    if with_skip:
        sk_f = r.standard_normal((M, N)) * 2.0
        S_sk = scale_of(sk_f)
        case.skip = quant_i8(sk_f, S_sk)
        S_y = scale_of(sk_f[:cal] + yf)
        case.res_ratio = (S_sk / S_y, S_out / S_y)
    return case


@dataclasses.dataclass
class AttentionCase:
    qkv: np.ndarray              # [B*N x 3*H*64] int8
    B: int
    N: int
    H: int
    logit_ratio: float           # S_q S_k / (8 S_logit)
    S_logit: float
    out_ratio: float             # S_v 2^-(k_out-1) / S_ctx
    k_s: int = 8
    k_out: int = 8


def attention_case(B: int, N: int, H: int, seed: int = 0, tails: str = "normal", k_s: int = 8,
                   k_out: int = 8, strength: float = 2.0) -> AttentionCase:
    """QKV with a per-head shared rank-1 direction so logits are varied.

    tails="laplace": logits ~ u_i v_j (product of two unit normals, heavy tails);
    tails="normal": a weaker shared direction plus noise.
    """
    r = rng(seed, "op", 2)
    D = H * HEAD_DIM
    T = B * N
    q = r.standard_normal((T, D)) * 0.5
    k = r.standard_normal((T, D)) * 0.5
    v = r.standard_normal((T, D))
    amp = math.sqrt(8.0) if tails == "laplace" else math.sqrt(8.0 * strength) / 2.0
    for h in range(H):
        a = r.standard_normal(HEAD_DIM)
        a *= amp / np.linalg.norm(a)
        u = r.standard_normal(T)
        w = r.standard_normal(T)
        sl = slice(h * HEAD_DIM, (h + 1) * HEAD_DIM)
        q[:, sl] += np.outer(u, a)
        k[:, sl] += np.outer(w, a)
    S_q, S_k, S_v = scale_of(q), scale_of(k), scale_of(v)
    qkv = np.concatenate([quant_i8(q, S_q), quant_i8(k, S_k), quant_i8(v, S_v)], axis=1)
    cal = min(B, 4)
    deq = np.concatenate([qkv[:, :D] * S_q, qkv[:, D:2 * D] * S_k, qkv[:, 2 * D:] * S_v], axis=1)
    logits, ctx = _attention_f(deq[: cal * N], cal, N, H)
    S_logit = scale_of(logits, bits=k_s)
    S_ctx = scale_of(ctx)
    return AttentionCase(qkv=qkv, B=B, N=N, H=H, logit_ratio=S_q * S_k / (8.0 * S_logit),
                         S_logit=S_logit, out_ratio=S_v * 2.0 ** -(k_out - 1) / S_ctx, k_s=k_s, k_out=k_out)


@dataclasses.dataclass
class GeluCase:
    x: np.ndarray
    S_h: float
    out_ratio: float             # S_h 2^-(k_out-1) / S_g


def gelu_case(n: int, seed: int = 0, spread: float = 3.0, k_out: int = 8) -> GeluCase:
    r = rng(seed, "op", 3)
    hf = r.standard_normal(n) * spread
    S_h = scale_of(hf)
    x = quant_i8(hf, S_h)
    S_g = scale_of(_gelu_f(x[: min(n, 1 << 20)] * S_h))
    return GeluCase(x=x, S_h=S_h, out_ratio=S_h * 2.0 ** -(k_out - 1) / S_g)


@dataclasses.dataclass
class LayerNormCase:
    x: np.ndarray
    gamma: np.ndarray
    beta: np.ndarray
    out_ratio: float             # S_gamma 2^-F / S_out
    F: int = 7


def layernorm_case(rows: int, cols: int, seed: int = 0, chan_std=(0.1, 10.0), F: int = 7) -> LayerNormCase:
    r = rng(seed, "op", 4)
    sig = np.exp(r.uniform(math.log(chan_std[0]), math.log(chan_std[1]), size=cols))
    xf = r.standard_normal((rows, cols)) * sig[None, :]
    S_x = scale_of(xf)
    x = quant_i8(xf, S_x)
    g = 1.0 + 0.1 * r.standard_normal(cols)
    be = 0.02 * r.standard_normal(cols)
    S_g = scale_of(g)
    gq = quant_i8(g, S_g)
    cal = min(rows, 4096)
    yf = _layernorm_f(x[:cal] * S_x, gq * S_g, be)
    S_out = scale_of(yf)
    return LayerNormCase(x=x, gamma=gq, beta=quant_i32(be, S_g * 2.0 ** -F), out_ratio=S_g * 2.0 ** -F / S_out, F=F)


@dataclasses.dataclass
class PtfCase:
    x_ptf: np.ndarray            # int8, channel i at scale s 2^alpha_i
    alpha: np.ndarray            # uint8 power-of-two factors in [0, 3]
    x_tensor: np.ndarray         # int8, one per-tensor scale (= s 2^3)
    gamma: np.ndarray
    beta: np.ndarray
    out_ratio: float             # S_gamma 2^-F / S_out
    S_out: float
    ln_float: np.ndarray         # floating-point LayerNorm of the unquantised rows
    F: int = 7


def ptf_case(rows: int, cols: int, seed: int = 0, chan_std=(0.1, 20.0), K: int = 3, F: int = 7) -> PtfCase:
    """LayerNorm inputs with inter-channel variation (per-channel std
    log-uniform on chan_std, as the ViT-B workload), quantised two ways: one
    per-tensor scale S, and power-of-two factors on a layer-wise s = S / 2^K,
    where channel i takes the smallest alpha_i in [0, K] whose range
    s 2^alpha_i 127.5 covers the channel (off-line calibration)."""
    r = rng(seed, "op", 5)
    sig = np.exp(r.uniform(math.log(chan_std[0]), math.log(chan_std[1]), size=cols))
    xf = r.standard_normal((rows, cols)) * sig[None, :]
    S = scale_of(xf)
    s = S / 2.0 ** K
    m = np.max(np.abs(xf), axis=0)
    alpha = np.clip(np.ceil(np.log2(np.maximum(m / (127.5 * s), 1e-30))), 0, K).astype(np.uint8)
    x_ptf = quant_i8(xf, s * 2.0 ** alpha.astype(np.float64)[None, :])
    x_tensor = quant_i8(xf, S)
    g = 1.0 + 0.1 * r.standard_normal(cols)
    be = 0.02 * r.standard_normal(cols)
    S_g = scale_of(g)
    gq = quant_i8(g, S_g)
    ln_f = _layernorm_f(xf, gq * S_g, be)
    S_out = scale_of(ln_f)
    return PtfCase(x_ptf=x_ptf, alpha=alpha, x_tensor=x_tensor, gamma=gq, beta=quant_i32(be, S_g * 2.0 ** -F),
                   out_ratio=S_g * 2.0 ** -F / S_out, S_out=S_out, ln_float=ln_f, F=F)


# ---------------------------------------------------------------------------
# a whole model: patch embedding, blocks, classifier head
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class ModelCase:
    img: np.ndarray              # [B x C x Hi x Wi] int8
    P: int
    w_pe: np.ndarray             # [D x C*P*P] int8, per output channel
    s_w_pe: np.ndarray
    bias_pe: np.ndarray          # int32 at S_img * s_w_pe
    cls: np.ndarray              # [D] int8 at the embedding scale
    pos: np.ndarray              # [(Np+1) x D] int8
    head_gamma: np.ndarray       # int8
    head_beta: np.ndarray        # int32 at S_head_gamma 2^-ln_F
    w_head: np.ndarray           # [Ncls_pad x D] int8 (rows past Ncls are zero)
    s_w_head: np.ndarray
    bias_head: np.ndarray        # int32 at S_head_ln * s_w_head
    Ncls: int                    # real classes; w_head has a multiple of 16 rows
    wl: Workload                 # the blocks (their block-0 input scale is the token scale)
    scales: Dict[str, float]     # img, e (embeddings), pos, x (tokens), head_gamma, head_ln, logits


def _patches_f(img, P):
    B, Cin, Hi, Wi = img.shape
    t = img.reshape(B, Cin, Hi // P, P, Wi // P, P).transpose(0, 2, 4, 1, 3, 5)
    return t.reshape(B * (Hi // P) * (Wi // P), Cin * P * P)


def model_case(B: int = 2, Hi: int = 224, Wi: int = 224, P: int = 16, C: int = 3, D: int = 192, H: int = 3,
               Dm: int = 768, blocks: int = 2, Ncls: int = 1000, seed: int = 0, n_cal: int = 2,
               ln_F: int = 7) -> ModelCase:
    """Seeded synthetic ViT: an int8 image batch, patch projection, class and
    position embeddings, ``blocks`` encoder blocks (``make_workload``) and a
    classifier head padded to a multiple of 16 classes.  Real scales come from
    a floating-point pass on the first ``n_cal`` images."""
    Np = (Hi // P) * (Wi // P)
    wl = make_workload(name="model", B=B, N=Np + 1, D=D, H=H, Dm=Dm, blocks=blocks, seed=seed, ln_F=ln_F)
    S = {}
    img_f = rng(seed, "img").standard_normal((B, C, Hi, Wi))
    S["img"] = scale_of(img_f)
    img = quant_i8(img_f, S["img"])
    w = rng(seed, "wpe").standard_normal((D, C * P * P)) * 0.02
    w_pe, s_w_pe = _per_channel_weights(w)
    b_f = rng(seed, "bpe").standard_normal(D) * 0.02
    cal = min(B, n_cal)
    e_f = _patches_f(img[:cal].astype(np.float64) * S["img"], P) @ (w_pe * s_w_pe[:, None]).T + b_f
    S["e"] = scale_of(e_f)
    cls_f = rng(seed, "cls").standard_normal(D) * 0.02
    pos_f = rng(seed, "pos").standard_normal((Np + 1, D)) * 0.02
    S["pos"] = scale_of(pos_f)
    S["x"] = wl.blocks[0].scales["x"]
    # head: I-LayerNorm on the class token, then the classifier
    hg = 1.0 + 0.1 * rng(seed, "hg").standard_normal(D)
    hbe = 0.02 * rng(seed, "hbe").standard_normal(D)
    S["head_gamma"] = scale_of(hg)
    hgq = quant_i8(hg, S["head_gamma"])
    y_last = wl.blocks[-1].scales["y"]
    t_f = rng(seed, "hg", 1).standard_normal((max(cal, 8), D)) * 40.0 * y_last
    ln_f = _layernorm_f(t_f, hgq * S["head_gamma"], hbe)
    S["head_ln"] = scale_of(ln_f)
    wh = rng(seed, "whead").standard_normal((Ncls, D)) * 0.02
    w_head, s_w_head = _per_channel_weights(wh)
    bh = rng(seed, "bhead").standard_normal(Ncls) * 0.02
    S["logits"] = scale_of(ln_f @ (w_head * s_w_head[:, None]).T + bh)
    pad = (-Ncls) % 16
    bias_head = quant_i32(bh, S["head_ln"] * s_w_head)
    if pad:
        w_head = np.concatenate([w_head, np.zeros((pad, D), np.int8)])
        s_w_head = np.concatenate([s_w_head, np.full(pad, s_w_head[0])])
        bias_head = np.concatenate([bias_head, np.zeros(pad, np.int32)])
    return ModelCase(img=img, P=P, w_pe=w_pe, s_w_pe=s_w_pe, bias_pe=quant_i32(b_f, S["img"] * s_w_pe),
                     cls=quant_i8(cls_f, S["e"]), pos=quant_i8(pos_f, S["pos"]), head_gamma=hgq,
                     head_beta=quant_i32(hbe, S["head_gamma"] * 2.0 ** -ln_F), w_head=w_head, s_w_head=s_w_head,
                     bias_head=bias_head, Ncls=Ncls, wl=wl, scales=S)
