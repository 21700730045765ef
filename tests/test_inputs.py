"""The seeded input generator: bf16 rounding, determinism and the configs' shapes."""
import numpy as np
import pytest

import pba_inputs as pi


def test_bf16_round_to_nearest_even_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, -0.0, 65504.0, 1e-30],
                                 np.float32)])
    ours = pi.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = pi.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_seeded_and_distinct_streams():
    cfg = pi.custom("t", B=2, H=2, N=8, c=8)
    a = pi.make_inputs(cfg, seed=0)
    b = pi.make_inputs(cfg, seed=0)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    assert not np.array_equal(a["q"], a["k"])
    c = pi.make_inputs(cfg, seed=1)
    assert not np.array_equal(a["q"], c["q"])


@pytest.mark.parametrize("name,masked_count", [("C1", 6), ("C2", 13), ("C3", 38), ("C4", 0),
                                               ("C5", 115)])
def test_config_masks(name, masked_count):
    cfg = pi.CONFIGS[name]
    keep = cfg.keep()
    assert keep.shape == (cfg.N,)
    assert int((keep == 0).sum()) == masked_count


def test_bias_std():
    cfg = pi.CONFIGS["C4"]
    d = pi.make_inputs(cfg, seed=0, with_dout=False, B=1)
    s = pi.bf16_bits_to_f32(d["bias"]).std()
    assert abs(s - 0.5) < 0.01
