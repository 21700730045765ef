"""GPU forward pass against the fp64 oracle, element by element on the same seeded bf16
inputs: small shapes that span several tiles and a ragged tail (full comparison), edge
cases, and the five workload configurations at full size (sampled (b, h) slices, each
compared in full)."""
import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import (assert_lse_close, assert_out_close, bf16_to_f64_tensor, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as p
    return p


def _inputs(B, H, Nq, Nk, C, masked=(), gate=True, bias=True, seed=0, bias_std=1.0,
            per_row_mask=False):
    d = {"q": pi.normal_bf16(seed, 1, (B, Nq, H, C)),
         "k": pi.normal_bf16(seed, 2, (B, Nk, H, C)),
         "v": pi.normal_bf16(seed, 3, (B, Nk, H, C))}
    if gate:
        d["g"] = pi.normal_bf16(seed, 4, (B, Nq, H, C))
    if bias:
        d["bias"] = pi.normal_bf16(seed, 5, (H, Nq, Nk), bias_std)
    keep = np.ones(Nk, np.uint8)
    for lo, hi in masked:
        keep[lo:hi] = 0
    if per_row_mask:
        rng = np.random.default_rng(seed + 7)
        keep = np.stack([keep] * B)
        keep &= (rng.random((B, Nk)) > 0.2).astype(np.uint8)
    d["keep"] = keep
    return d


def _run_and_check(pba, d, scale=None, use_mask=True):
    import torch
    t = to_dev(d)
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t.get("bias"),
                                 t["keep"] if use_mask else None, t.get("g"),
                                 scale=scale or 0.0)
    pba.pba_device_status()
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    ref_out, ref_lse = oracle.fwd(f["q"], f["k"], f["v"], f.get("bias"),
                                  f["keep"] if use_mask else None, f.get("g"), scale=scale)
    assert_out_close(bf16_to_f64_tensor(out), ref_out)
    assert_lse_close(lse.cpu().numpy().astype(np.float64), ref_lse)
    return out, lse


CASES = {
    # name: (B, H, Nq, Nk, C, masked, gate, bias)
    "tiny_triangle_config": (64, 4, 64, 64, 32, ((58, 64),), True, True),
    "ragged_two_tiles": (5, 2, 200, 200, 32, ((190, 200),), True, True),
    "c24_padded": (6, 3, 136, 136, 24, (), True, True),
    "c64": (3, 2, 136, 136, 64, ((0, 3),), True, True),
    "c16": (4, 2, 72, 72, 16, (), True, True),
    "c8": (3, 1, 40, 40, 8, (), True, True),
    "c40": (3, 2, 96, 96, 40, ((90, 96),), True, True),
    "nq_ne_nk": (4, 2, 72, 200, 32, ((100, 130),), True, True),
    "odd_B_chunk": (7, 2, 128, 256, 32, (), True, True),
    "single_row_head": (1, 1, 256, 256, 32, ((250, 256),), True, True),
    "no_bias_no_gate": (9, 2, 128, 128, 32, (), False, False),
    "small_N": (3, 2, 8, 8, 32, (), True, True),
    "three_key_tiles": (10, 2, 384, 384, 32, ((100, 140), (300, 384)), True, True),
    "many_rows_one_tile": (40, 1, 128, 128, 32, ((120, 128),), True, True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_fwd_matches_oracle(pba, name):
    B, H, Nq, Nk, C, masked, gate, bias = CASES[name]
    _run_and_check(pba, _inputs(B, H, Nq, Nk, C, masked, gate, bias))


def test_fwd_explicit_scale(pba):
    _run_and_check(pba, _inputs(4, 2, 128, 128, 32, ((10, 20),)), scale=0.3)


def test_fwd_no_mask_pointer(pba):
    _run_and_check(pba, _inputs(4, 2, 136, 136, 32), use_mask=False)


def test_fwd_per_row_mask(pba):
    _run_and_check(pba, _inputs(6, 2, 136, 136, 32, ((130, 136),), per_row_mask=True))


def test_fwd_fully_masked_rows(pba):
    import torch
    d = _inputs(3, 2, 64, 64, 32, ((0, 64),))
    out, lse = _run_and_check(pba, d)
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_fwd_strided_packed_qkv(pba):
    """q, k, v as channel slices of one packed [B, N, H, 3C] tensor, gate and out strided."""
    import torch
    B, H, N, C = 5, 2, 136, 32
    d = _inputs(B, H, N, N, C, ((120, 136),))
    t = to_dev(d)
    packed = torch.cat([t["q"], t["k"], t["v"]], dim=-1).contiguous()
    q, k, v = packed[..., :C], packed[..., C:2 * C], packed[..., 2 * C:]
    gbig = torch.zeros(B, N, H, 2 * C, dtype=torch.bfloat16, device="cuda")
    gbig[..., C:] = t["g"]
    g = gbig[..., C:]
    obig = torch.zeros(B, N, H, 2 * C, dtype=torch.bfloat16, device="cuda")
    out = obig[..., :C]
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    pba.pba_fwd(q, k, v, t["bias"], t["keep"], g, out, lse)
    pba.pba_device_status()
    assert torch.all(obig[..., C:] == 0)
    f = {k2: (pi.bf16_bits_to_f64(v2) if k2 != "keep" else v2) for k2, v2 in d.items()}
    ref_out, ref_lse = oracle.fwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f["g"])
    assert_out_close(bf16_to_f64_tensor(out), ref_out)
    assert_lse_close(lse.cpu().numpy().astype(np.float64), ref_lse)


def test_fwd_is_deterministic(pba):
    import torch
    t = to_dev(_inputs(16, 2, 256, 256, 32, ((250, 256),)))
    o1, l1 = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    o2, l2 = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _sample_slices(B, H, n=4, seed=0):
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (B - 1, H - 1)}
    while len(picks) < min(n, B * H):
        picks.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(picks)


@pytest.mark.parametrize("cfg_name", ["C1", "C2", "C3", "C4", "C5"])
def test_fwd_full_config_sampled(pba, cfg_name):
    """The workload configurations at full size, in the launch configuration the benchmark
    times; whole (b, h) slices compared against the oracle."""
    cfg = pi.CONFIGS[cfg_name]
    d = pi.make_inputs(cfg, seed=0, with_dout=False)
    t = to_dev(d)
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    pba.pba_device_status()
    keep = d["keep"]
    for b, h in _sample_slices(cfg.B, cfg.H):
        sl = lambda a: pi.bf16_bits_to_f64(a[b, :, h])
        ref_o, ref_l = oracle.fwd_slice(sl(d["q"]), sl(d["k"]), sl(d["v"]),
                                        pi.bf16_bits_to_f64(d["bias"][h]), keep, sl(d["g"]))
        got_o = out[b, :, h].float().cpu().numpy().astype(np.float64)
        assert_out_close(got_o, ref_o, "out[%d,:,%d]" % (b, h))
        assert_lse_close(lse[b, h].cpu().numpy().astype(np.float64), ref_l)
    # properties that hold at any size: finite outputs, |out| <= max|v| (softmax convexity)
    assert torch_all_finite(out) and torch_all_finite(lse)
    vmax = float(t["v"].abs().max())
    assert float(out.abs().max()) <= vmax * 1.01


def torch_all_finite(x):
    import torch
    return bool(torch.isfinite(x.float()).all())
