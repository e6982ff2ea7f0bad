"""Host-side checks of the seeded input generator (no method arithmetic)."""
import numpy as np

import synthetic


def test_seeded_and_deterministic():
    a = synthetic.make_workload(B=2, N=7, D=128, H=2, Dm=256, seed=5, n_cal=2)
    b = synthetic.make_workload(B=2, N=7, D=128, H=2, Dm=256, seed=5, n_cal=2)
    c = synthetic.make_workload(B=2, N=7, D=128, H=2, Dm=256, seed=6, n_cal=2)
    np.testing.assert_array_equal(a.x, b.x)
    np.testing.assert_array_equal(a.blocks[0].w1, b.blocks[0].w1)
    assert a.blocks[0].scales == b.blocks[0].scales
    assert not np.array_equal(a.x, c.x)


def test_shapes_dtypes_and_ranges():
    wl = synthetic.make_workload(B=3, N=11, D=192, H=3, Dm=768, blocks=2, seed=1, n_cal=2)
    assert wl.x.shape == (33, 192) and wl.x.dtype == np.int8
    assert len(wl.blocks) == 2
    q = wl.blocks[1]
    assert q.w_qkv.shape == (576, 192) and q.w_qkv.dtype == np.int8
    assert q.w2.shape == (192, 768) and q.bias2.dtype == np.int32
    assert q.s_w1.shape == (768,)
    assert np.abs(wl.x.astype(int)).max() == 127          # per-tensor max maps to 127
    for k, v in q.scales.items():
        assert v > 0, k
    # chained blocks: block 1 input scale is block 0 output scale
    assert q.scales["x"] == wl.blocks[0].scales["y"]


def test_named_configs():
    assert synthetic.CONFIG_ORDER == list(synthetic.CONFIGS)
    for name, cfg in synthetic.CONFIGS.items():
        assert cfg["D"] == cfg["H"] * 64 and cfg["Dm"] == 4 * cfg["D"]


def test_op_cases():
    lc = synthetic.linear_case(40, 64, 48, seed=1, with_skip=True)
    assert lc.X.shape == (40, 64) and lc.W.shape == (48, 64) and lc.skip.shape == (40, 48)
    ac = synthetic.attention_case(2, 13, 2, seed=1, tails="laplace")
    assert ac.qkv.shape == (26, 384) and ac.S_logit > 0
    gc = synthetic.gelu_case(1000, seed=1)
    assert gc.x.dtype == np.int8 and gc.S_h > 0
    nc = synthetic.layernorm_case(10, 192, seed=1)
    assert nc.x.shape == (10, 192) and nc.beta.dtype == np.int32
