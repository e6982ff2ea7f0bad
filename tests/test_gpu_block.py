"""GPU parity of the encoder block against the CPU oracle, bit for bit.

Small blocks are compared in full.  The five named workloads run at full size
in the launch configuration the benchmark times (the whole batch, every block
back to back) and every image is compared: the oracle runs one image per task
on every host core (images never interact inside a block, so this is the same
result as one call over the batch).  One small block is also compared stage by
stage, from the intermediates the block leaves in its workspace, so that a
mismatch names the step it starts at.
"""
import time

import numpy as np
import pytest
import torch

import integer_only_quantized_int8_b200 as ivit
import oracle
import synthetic
from integer_only_quantized_int8_b200 import build as ivit_build
from integer_only_quantized_int8_b200 import params as ivit_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    ivit_build.build()
    yield
    assert ivit.ivit_stream_status() == 0


def run_blocks_gpu(wl):
    T = wl.B * wl.N
    dps = [ivit_params.to_device(ivit_params.integer_params(q)) for q in wl.blocks]
    ws = torch.empty(ivit.ivit_block_workspace_bytes(wl.B, wl.N, wl.D, wl.Dm), dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(wl.x).cuda()
    bufs = [x, torch.empty((T, wl.D), dtype=torch.int8, device="cuda"),
            torch.empty((T, wl.D), dtype=torch.int8, device="cuda")]
    cur = 0
    for i, dp in enumerate(dps):
        nxt = 1 + (i % 2)
        ivit.ivit_block_forward(dp, bufs[cur], bufs[nxt], ws, wl.B, wl.N)
        cur = nxt
    torch.cuda.synchronize()
    return bufs[cur].cpu().numpy()


def run_blocks_oracle(wl, images):
    N, D = wl.N, wl.D
    ps = [oracle.block_params(q) for q in wl.blocks]
    out = {}
    for b in images:
        x = wl.x[b * N:(b + 1) * N]
        for p in ps:
            x = oracle.block_forward(p, x, 1, N)
        out[b] = x
    return out


def run_blocks_oracle_all(wl):
    """Every image of the batch through every block, one image per host thread."""
    x = wl.x
    threads = 1
    for q in wl.blocks:
        x, threads = oracle.block_forward_images(oracle.block_params(q), x, wl.B, wl.N)
    return x, threads


SMALL = [
    dict(B=2, N=13, D=128, H=2, Dm=256, tails="normal"),
    dict(B=1, N=197, D=192, H=3, Dm=768, tails="laplace"),
    dict(B=3, N=130, D=256, H=4, Dm=512, tails="normal"),
    dict(B=2, N=1, D=64, H=1, Dm=128, tails="normal"),
    dict(B=2, N=40, D=128, H=2, Dm=256, blocks=3, tails="laplace"),
]


@pytest.mark.parametrize("cfg", SMALL)
def test_block_parity_small(cfg):
    cfg = dict(cfg)
    blocks = cfg.pop("blocks", 1)
    wl = synthetic.make_workload(seed=7, n_cal=2, blocks=blocks, **cfg)
    got = run_blocks_gpu(wl)
    want = run_blocks_oracle(wl, range(wl.B))
    for b in range(wl.B):
        np.testing.assert_array_equal(got[b * wl.N:(b + 1) * wl.N], want[b], err_msg=f"image {b}")


@pytest.mark.parametrize("name", synthetic.CONFIG_ORDER)
def test_block_parity_full_size(name):
    wl = synthetic.workload(name, seed=0)
    got = run_blocks_gpu(wl)
    t0 = time.perf_counter()
    want, threads = run_blocks_oracle_all(wl)
    print(f"[oracle] {name}: {wl.B} images x {len(wl.blocks)} block(s) on {threads} host threads, "
          f"{time.perf_counter() - t0:.1f} s")
    for b in range(wl.B):
        sl = slice(b * wl.N, (b + 1) * wl.N)
        np.testing.assert_array_equal(got[sl], want[sl], err_msg=f"{name} image {b}")
    # the block is not degenerate at this size: the output uses the int8 range
    assert np.unique(got).size > 100


def test_block_stages_match_oracle():
    """Every intermediate of one block against the oracle's operators, each fed
    the oracle's own previous stage, so the first differing stage is named."""
    wl = synthetic.make_workload(seed=13, n_cal=2, B=3, N=197, D=192, H=3, Dm=768, tails="laplace")
    B, N, D, Dm, H = wl.B, wl.N, wl.D, wl.Dm, wl.H
    T = B * N
    dp = ivit_params.to_device(ivit_params.integer_params(wl.blocks[0]))
    ws = torch.empty(ivit.ivit_block_workspace_bytes(B, N, D, Dm), dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(wl.x).cuda()
    y = torch.empty_like(x)
    ivit.ivit_block_forward(dp, x, y, ws, B, N)
    torch.cuda.synchronize()
    # workspace sub-buffers, 256-byte aligned: ln | qkv | ctx | xh | g (ln holds LN2 at the end)
    up = lambda v: (v + 255) // 256 * 256
    w8 = ws.view(torch.int8).cpu().numpy()
    o_qkv = up(T * D)
    o_ctx = o_qkv + up(T * 3 * D)
    o_xh = o_ctx + up(T * D)
    o_g = o_xh + up(T * D)
    got = {"qkv": w8[o_qkv:o_qkv + T * 3 * D].reshape(T, 3 * D), "ctx": w8[o_ctx:o_ctx + T * D].reshape(T, D),
           "xh": w8[o_xh:o_xh + T * D].reshape(T, D), "ln2": w8[:T * D].reshape(T, D),
           "g": w8[o_g:o_g + T * Dm].reshape(T, Dm), "y": y.cpu().numpy()}
    p = oracle.block_params(wl.blocks[0])
    want = {}
    ln1 = oracle.layernorm(wl.x, p["ln1_gamma"], p["ln1_beta"], p["ln_F"], p["ln_M"], p["ln1_out"])
    want["qkv"] = oracle.linear_requant(ln1, p["w_qkv"], p["bias_qkv"], p["b_qkv"], p["c_qkv"])
    want["ctx"] = oracle.attention(want["qkv"], B, N, H, p["logit"], p["k_s"], p["attn_I0"], p["attn_M"],
                                   p["attn_k_out"], p["attn_out"])
    want["xh"] = oracle.linear_requant(want["ctx"], p["w_o"], p["bias_o"], p["b_o"], p["c_o"], skip=wl.x,
                                       res=p["res1"])
    want["ln2"] = oracle.layernorm(want["xh"], p["ln2_gamma"], p["ln2_beta"], p["ln_F"], p["ln_M"], p["ln2_out"])
    h = oracle.linear_requant(want["ln2"], p["w1"], p["bias1"], p["b1"], p["c1"])
    want["g"] = oracle.shiftgelu(h, p["gelu_I0"], p["gelu_M"], p["gelu_k_out"], p["gelu_out"])
    want["y"] = oracle.linear_requant(want["g"], p["w2"], p["bias2"], p["b2"], p["c2"], skip=want["xh"],
                                      res=p["res2"])
    for stage in ("qkv", "ctx", "xh", "ln2", "g", "y"):
        bad = int(np.sum(got[stage] != want[stage]))
        assert bad == 0, f"stage {stage}: {bad} of {want[stage].size} values differ from the oracle"
    # the composed operators are the oracle's block
    np.testing.assert_array_equal(want["y"], oracle.block_forward(p, wl.x, B, N))


def test_block_parity_linear_round_half_up():
    """A block whose four linear layers round half up, against the oracle's
    block with the same reading."""
    wl = synthetic.make_workload(seed=11, n_cal=2, B=2, N=61, D=192, H=3, Dm=768)
    ip = ivit_params.integer_params(wl.blocks[0])
    ip["linear_round"] = 1
    dp = ivit_params.to_device(ip)
    ws = torch.empty(ivit.ivit_block_workspace_bytes(wl.B, wl.N, wl.D, wl.Dm), dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(wl.x).cuda()
    y = torch.empty_like(x)
    ivit.ivit_block_forward(dp, x, y, ws, wl.B, wl.N)
    op = oracle.block_params(wl.blocks[0])
    op["linear_round"] = 1
    want = oracle.block_forward(op, wl.x, wl.B, wl.N)
    np.testing.assert_array_equal(y.cpu().numpy(), want)
    op["linear_round"] = 0
    assert not np.array_equal(want, oracle.block_forward(op, wl.x, wl.B, wl.N))
