"""MSA pair-weighted averaging on the GPU (pba_pwa_fwd / pba_pwa_bwd through the C ABI)
against the fp64 oracle (oracle.pwa_fwd / oracle.pwa_bwd) on the same seeded bf16 inputs:
small shapes compared in full, edge cases, bit-stability of dbias, and the MSA row workload's
size (128 rows x 256 tokens, 8 heads, c=32)."""
import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import GRAD_REL_L2, LSE_MAX_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, assert_grad_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pba():
    import pair_biased_attention_gated_b200 as m
    return m


def _inputs(B, H, N, C, masked, gate, bias, seed=0):
    cfg = pi.custom("pwa", B=B, H=H, N=N, c=C, masked=masked, gate=gate)
    d = pi.make_inputs(cfg, seed=seed)
    if not bias:
        d.pop("bias")
    d.pop("q"), d.pop("k")
    return d


def _run(pba, t, want_dbias=True):
    keep = t.get("keep")
    out, lse = pba.pwa_fwd(t["v"], t.get("bias"), keep, t.get("g"))
    dv, dg, db = pba.pwa_bwd(t["v"], t.get("bias"), keep, t.get("g"), out, t["dout"], want_dbias)
    pba.pba_device_status()
    return out, lse, dv, dg, db


def _check_full(pba, d):
    f64 = pi.bf16_bits_to_f64
    t = to_dev(d)
    out, lse, dv, dg, db = _run(pba, t)
    v, bias, g, dout = f64(d["v"]), (f64(d["bias"]) if "bias" in d else None), \
        (f64(d["g"]) if "g" in d else None), f64(d["dout"])
    keep = d.get("keep")
    r_out, r_lse = oracle.pwa_fwd(v, bias, keep, g)
    got = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - r_out)
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (err.max(), err.mean())
    gl = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(r_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - r_lse[fin]).max(initial=0.0) <= LSE_MAX_ABS
    # the backward from the oracle's own forward output, as the GPU uses its own
    r_dv, r_dg, r_db = oracle.pwa_bwd(v, bias, keep, g, dout)
    assert_grad_close(dv.float().cpu().numpy().astype(np.float64), r_dv, "dv")
    assert_grad_close(db.cpu().numpy().astype(np.float64), r_db, "dbias")
    if g is not None:
        assert_grad_close(dg.float().cpu().numpy().astype(np.float64), r_dg, "dgate")


CASES = {
    # name: (B, H, N, C, masked, gate, bias)
    "ragged_c32": (4, 2, 136, 32, ((130, 136),), True, True),
    "c16": (3, 2, 72, 16, (), True, True),
    "c24_padded": (5, 3, 128, 24, (), True, True),
    "c64": (2, 2, 200, 64, ((0, 5),), True, True),
    "no_gate": (6, 2, 96, 32, ((90, 96),), False, True),
    "no_bias": (3, 2, 80, 32, ((10, 20),), True, False),
    "rows_over_one_chunk": (20, 1, 256, 32, ((250, 256),), True, True),
    "small_N": (3, 2, 8, 32, (), True, True),
    "three_tiles": (6, 2, 300, 32, ((100, 140),), True, True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_pwa_matches_oracle(pba, name):
    B, H, N, C, masked, gate, bias = CASES[name]
    _check_full(pba, _inputs(B, H, N, C, masked, gate, bias))


def test_pwa_all_keys_masked(pba):
    d = _inputs(3, 2, 40, 32, ((0, 40),), True, True)
    t = to_dev(d)
    out, lse, dv, dg, db = _run(pba, t)
    assert float(out.float().abs().max()) == 0.0
    assert bool(np.isneginf(lse.cpu().numpy()).all())
    assert float(dv.float().abs().max()) == 0.0 and float(db.abs().max()) == 0.0


def test_pwa_dbias_bit_stable(pba):
    import torch
    t = to_dev(_inputs(24, 2, 200, 32, ((190, 200),), True, True))
    ref = None
    for _ in range(3):
        db = _run(pba, t)[4]
        if ref is None:
            ref = db.clone()
        else:
            assert torch.equal(ref, db)


def test_pwa_without_dbias(pba):
    t = to_dev(_inputs(4, 2, 136, 32, (), True, True))
    out, lse, dv, dg, db = _run(pba, t)
    dv2, dg2, db2 = pba.pwa_bwd(t["v"], t["bias"], t["keep"], t["g"], out, t["dout"], want_dbias=False)
    assert db2 is None
    import torch
    assert torch.equal(dv, dv2) and torch.equal(dg, dg2)


def test_pwa_rejects_per_row_mask_and_rectangular(pba):
    import ctypes
    d = pba.dims_dense(4, 2, 64, 64, 32)
    d.smask_b = 64
    st = pba.lib.pba_pwa_fwd(*([16] * 7), 1 << 30, ctypes.byref(d), None)
    assert st == 2 and "shared" in pba.lib.pba_last_error().decode()
    d2 = pba.dims_dense(4, 2, 64, 96, 32)
    st = pba.lib.pba_pwa_fwd(*([16] * 7), 1 << 30, ctypes.byref(d2), None)
    assert st == 2 and "Nq == Nk" in pba.lib.pba_last_error().decode()


def test_pwa_msa_row_size(pba):
    """The MSA row workload's size in the benchmark's launch configuration, compared in full."""
    cfg = pi.CONFIGS["C2"]
    _check_full(pba, _inputs(cfg.B, cfg.H, cfg.N, cfg.c, cfg.masked, True, True))
