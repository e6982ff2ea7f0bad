"""GPU parity of the encoder block against the CPU oracle, bit for bit.

Small blocks are compared in full.  The five named workloads run at full size
in the launch configuration the benchmark times (the whole batch, every block
back to back); the oracle then recomputes sampled images, which is exact
because images never interact inside a block.
"""
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
    B = wl.B
    images = sorted({0, B - 1} | ({B // 2} if wl.blocks.__len__() == 1 else set()))
    want = run_blocks_oracle(wl, images)
    for b in images:
        np.testing.assert_array_equal(got[b * wl.N:(b + 1) * wl.N], want[b], err_msg=f"{name} image {b}")
    # the block is not degenerate at this size: the output uses the int8 range
    assert np.unique(got).size > 100


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
