"""Block-sparse local attention (pba_fwd_local / pba_bwd_local through the C ABI): query tile
t attends only key tiles [t - window, t + window].  The kernels never read the other tiles, so
they must equal the fp64 oracle of the dense operator with those (query, key) pairs masked:
the oracle receives the bias with -inf at every pair outside the window, the GPU the plain
bias (whose out-of-window values would change the result if they were read)."""
import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import (assert_grad_close, assert_lse_close, assert_out_close, bf16_to_f64_tensor,
                         to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as m
    return m


def _ref(d, window, Nq, Nk):
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    f["bias"] = np.where(pi.window_pair_mask(Nq, Nk, window)[None], f["bias"], -np.inf)
    return f


def _check(pba, B, H, N, C, window, masked=(), gate=True, seed=0, Nq=None):
    cfg = pi.custom("local", B=B, H=H, N=N, c=C, masked=masked, gate=gate)
    d = pi.make_inputs(cfg, seed=seed)
    if Nq is not None:   # fewer queries than keys: the first Nq rows of q, g, dout, bias
        for k in ("q", "g", "dout"):
            if k in d:
                d[k] = np.ascontiguousarray(d[k][:, :Nq])
        d["bias"] = np.ascontiguousarray(d["bias"][:, :Nq])
    nq = N if Nq is None else Nq
    t = to_dev(d)
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t.get("g"), window=window)
    dq, dk, dv, dg, db = pba.attention_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t.get("g"), out, lse,
                                           t["dout"], window=window)
    pba.pba_device_status()
    f = _ref(d, window, nq, N)
    r_out, r_lse = oracle.fwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f.get("g"))
    assert_out_close(bf16_to_f64_tensor(out), r_out)
    assert_lse_close(lse.cpu().numpy().astype(np.float64), r_lse)
    r_dq, r_dk, r_dv, r_dg, r_db = oracle.bwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f.get("g"), f["dout"])
    assert_grad_close(bf16_to_f64_tensor(dq), r_dq, "dq")
    assert_grad_close(bf16_to_f64_tensor(dk), r_dk, "dk")
    assert_grad_close(bf16_to_f64_tensor(dv), r_dv, "dv")
    got_db = db.cpu().numpy().astype(np.float64)
    assert_grad_close(got_db, r_db, "dbias")
    outside = ~pi.window_pair_mask(nq, N, window)
    assert np.all(got_db[:, outside] == 0.0), "dbias outside the window must be exactly zero"
    if gate:
        assert_grad_close(bf16_to_f64_tensor(dg), r_dg, "dgate")


CASES = {
    # name: (B, H, N, C, window, masked)
    "w1_c32_five_tiles": (4, 2, 640, 32, 1, ((620, 640),)),
    "w0_diagonal_tiles": (3, 2, 384, 32, 0, ()),
    "w2_c16_ragged": (3, 2, 712, 16, 2, ((0, 7),)),
    "w1_c64": (2, 2, 512, 64, 1, ((500, 512),)),
    "w1_c24_padded": (3, 3, 520, 24, 1, ()),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_local_attention_matches_masked_dense_oracle(pba, name):
    B, H, N, C, window, masked = CASES[name]
    _check(pba, B, H, N, C, window, masked)


def test_local_attention_no_gate(pba):
    _check(pba, 3, 2, 512, 32, 1, ((400, 410),), gate=False)


def test_local_attention_fewer_queries_than_keys(pba):
    _check(pba, 3, 2, 640, 32, 1, ((630, 640),), Nq=512)


def test_wide_window_is_the_dense_operator(pba):
    """A window covering every tile visits exactly the dense kernel's steps: bit-identical."""
    import torch
    cfg = pi.custom("wide", B=4, H=2, N=400, c=32, masked=((390, 400),))
    t = to_dev(pi.make_inputs(cfg, seed=3))
    dense = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    wide = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], window=8)
    assert torch.equal(dense[0], wide[0]) and torch.equal(dense[1], wide[1])
    gd = pba.attention_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], dense[0], dense[1], t["dout"])
    gw = pba.attention_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], dense[0], dense[1], t["dout"],
                           window=8)
    pba.pba_device_status()
    for name, a, b in zip(("dk", "dv", "dgate", "dbias"), gd[1:], gw[1:]):
        assert torch.equal(a, b), name


def test_local_dbias_bit_stable(pba):
    import torch
    cfg = pi.custom("lstab", B=24, H=2, N=640, c=32, masked=((600, 640),))
    t = to_dev(pi.make_inputs(cfg, seed=4))
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], window=1)
    ref = None
    for _ in range(3):
        db = pba.attention_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], out, lse, t["dout"],
                               window=1)[4]
        pba.pba_device_status()
        if ref is None:
            ref = db.clone()
        else:
            assert torch.equal(ref, db)


def test_atom_attention_size_sampled(pba):
    """The sequence-local atom attention workload's size (48 copies x 3072 atoms, window 1):
    rows of a few (b, h) problems compared with the oracle row by row."""
    cfg = pi.CONFIGS["C6"]
    d = pi.make_inputs(cfg, seed=0)
    t = to_dev(d)
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], window=cfg.window)
    pba.pba_device_status()
    f = _ref(d, cfg.window, cfg.N, cfg.N)
    got = bf16_to_f64_tensor(out)
    gl = lse.cpu().numpy().astype(np.float64)
    for b in (0, 47):
        for h in (0, 3):
            rows = np.r_[0:40, 1500:1540, 3000:3072]
            bias_bh = f["bias"][h][rows]
            r_out, r_lse = oracle.fwd_slice(f["q"][b, rows, h], f["k"][b, :, h], f["v"][b, :, h], bias_bh,
                                            f["keep"], f["g"][b, rows, h])
            assert_out_close(got[b, rows, h], r_out)
            assert_lse_close(gl[b, h, rows], r_lse)


def test_local_attention_per_row_key_mask(pba):
    """A key mask with one row per b (its words travel with each row's K/V tiles) under a window."""
    B, H, N, C, window = 4, 2, 512, 32, 1
    cfg = pi.custom("lrow", B=B, H=H, N=N, c=C)
    d = pi.make_inputs(cfg, seed=7)
    keep = np.ones((B, N), dtype=np.uint8)
    for b in range(B):
        keep[b, 480 - 37 * b:] = 0          # a different padding tail per row
        keep[b, 100 + 50 * b: 110 + 50 * b] = 0
    d["keep"] = keep
    t = to_dev(d)
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], window=window)
    dq, dk, dv, dg, db = pba.attention_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], out, lse,
                                           t["dout"], window=window)
    pba.pba_device_status()
    f = _ref(d, window, N, N)
    r_out, r_lse = oracle.fwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f["g"])
    assert_out_close(bf16_to_f64_tensor(out), r_out)
    assert_lse_close(lse.cpu().numpy().astype(np.float64), r_lse)
    r_dq, r_dk, r_dv, r_dg, r_db = oracle.bwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f["g"], f["dout"])
    for name, got, ref in (("dq", dq, r_dq), ("dk", dk, r_dk), ("dv", dv, r_dv), ("dgate", dg, r_dg)):
        assert_grad_close(bf16_to_f64_tensor(got), ref, name)
    assert_grad_close(db.cpu().numpy().astype(np.float64), r_db, "dbias")
