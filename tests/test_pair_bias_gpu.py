"""Pair-bias projection on the GPU (pba_pair_bias_fwd / pba_pair_bias_bwd through the C ABI)
against the fp64 oracle (oracle.pair_bias_fwd / pair_bias_bwd) on the same seeded inputs.

Tolerances: the bias and dz are bf16 outputs, so each element may differ from the oracle
by its bf16 rounding (2^-8 relative) plus the fp32 arithmetic before it (bounded here by
1e-3 absolute, a margin over 256-term fp32 sums of unit-size terms); dz, dw, dgamma and
dbeta also meet the gradients' relative L2 bound of 1e-2."""
import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import GRAD_REL_L2, OUT_MAX_ABS, OUT_MEAN_ABS, assert_grad_close, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-5
BF16_REL = 2.0 ** -8
ABS = 1e-3


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as m
    return m


def _dev(d, transpose=False):
    import torch
    z = torch.from_numpy(d["z"].view(np.int16)).view(torch.bfloat16).cuda()
    if transpose:
        z = z.transpose(0, 1)   # element (i, j) = stored (j, i): the ending-node bias
    f = {k: torch.from_numpy(d[k]).cuda() for k in ("gamma", "beta", "w", "dbias")}
    return z, f


def _ref_inputs(d, transpose=False):
    z = pi.bf16_bits_to_f64(d["z"])
    if transpose:
        z = np.ascontiguousarray(z.transpose(1, 0, 2))
    return z, d["gamma"].astype(np.float64), d["beta"].astype(np.float64), d["w"].astype(np.float64), \
        d["dbias"].astype(np.float64)


def _assert_elementwise(got, ref, what):
    err = np.abs(got - ref)
    bound = BF16_REL * np.abs(ref) + ABS
    worst = np.max(err - bound)
    assert worst <= 0, "%s: max excess over the bound %.3g (max err %.3g)" % (what, worst, err.max())


def _check(pba, Ni, Nj, Cz, H, seed=0, transpose=False, dbias_shape=None):
    d = pi.make_pair_bias_inputs(Nj if transpose else Ni, Ni if transpose else Nj, Cz, H, seed)
    if transpose:
        d["dbias"] = np.ascontiguousarray(d["dbias"].transpose(0, 2, 1))
    z, f = _dev(d, transpose)
    bias = pba.pair_bias_fwd(z, f["gamma"], f["beta"], f["w"], EPS)
    dz, dw, dgamma, dbeta = pba.pair_bias_bwd(z, f["gamma"], f["beta"], f["w"], f["dbias"], EPS)
    pba.pba_device_status()
    rz, rg, rb, rw, rdb = _ref_inputs(d, transpose)
    r_bias = oracle.pair_bias_fwd(rz, rg, rb, rw, EPS)
    _assert_elementwise(bias.float().cpu().numpy().astype(np.float64), r_bias, "bias")
    r_dz, r_dw, r_dg, r_db = oracle.pair_bias_bwd(rz, rg, rb, rw, rdb, EPS)
    got_dz = dz.float().cpu().numpy().astype(np.float64)
    _assert_elementwise(got_dz, r_dz, "dz")
    assert_grad_close(got_dz, r_dz, "dz")
    assert_grad_close(dw.cpu().numpy().astype(np.float64), r_dw, "dw")
    assert_grad_close(dgamma.cpu().numpy().astype(np.float64), r_dg, "dgamma")
    assert_grad_close(dbeta.cpu().numpy().astype(np.float64), r_db, "dbeta")


CASES = {
    # name: (Ni, Nj, Cz, H)
    "tiny_ragged_c64_h1": (3, 5, 64, 1),
    "three_tiles_c128_h8": (4, 300, 128, 8),
    "c192_h16": (2, 128, 192, 16),
    "c256_h4_ragged": (3, 200, 256, 4),
    "h3_padded": (5, 130, 128, 3),
    "msa_row_pair_256": (256, 256, 128, 8),
    # Cz = 128 runs the backward whose parameter sums are tensor-core products: every padded
    # head count (4, 8, 16), one head, and a ragged row end
    "c128_h16_ragged": (3, 200, 128, 16),
    "c128_h1_ragged": (4, 77, 128, 1),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_pair_bias_matches_oracle(pba, name):
    _check(pba, *CASES[name])


def test_pair_bias_transposed_view(pba):
    """bias[h, i, j] from z[j, i, :] (the ending-node triangle attention): the same call
    with the two z strides exchanged."""
    _check(pba, 136, 72, 128, 4, seed=3, transpose=True)


def test_pair_bias_large_triangle_size(pba):
    """The large triangle workload's pair representation (768 x 768, Cz = 128, 4 heads)."""
    _check(pba, 768, 768, 128, 4, seed=1)


def test_pair_bias_bwd_bit_stable(pba):
    import torch
    d = pi.make_pair_bias_inputs(96, 384, 128, 16, seed=4)
    z, f = _dev(d)
    ref = None
    for _ in range(3):
        out = pba.pair_bias_bwd(z, f["gamma"], f["beta"], f["w"], f["dbias"], EPS)
        pba.pba_device_status()
        if ref is None:
            ref = [t.clone() for t in out]
        else:
            assert all(torch.equal(a, b) for a, b in zip(ref, out))


def test_pair_bias_empty_problem(pba):
    import torch
    z = torch.empty((0, 16, 128), dtype=torch.bfloat16, device="cuda")
    gamma = torch.ones(128, device="cuda")
    beta = torch.zeros(128, device="cuda")
    w = torch.ones(128, 4, device="cuda")
    dbias = torch.empty((4, 0, 16), device="cuda")
    dz, dw, dgamma, dbeta = pba.pair_bias_bwd(z, gamma, beta, w, dbias, EPS)
    pba.pba_device_status()
    assert float(dw.abs().max()) == 0.0 and float(dgamma.abs().max()) == 0.0 and float(dbeta.abs().max()) == 0.0


def test_pair_bias_feeds_the_attention(pba):
    """LayerNorm -> projection -> attention: the GPU chain against the oracle chain (the
    oracle's own fp64 bias into the attention oracle), at the attention's tolerances."""
    B, N, H, c, Cz = 8, 200, 4, 32, 128
    d = pi.make_pair_bias_inputs(N, N, Cz, H, seed=5)
    z, f = _dev(d)
    bias = pba.pair_bias_fwd(z, f["gamma"], f["beta"], f["w"], EPS)
    cfg = pi.custom("chain", B=B, H=H, N=N, c=c, masked=((190, 200),))
    a = pi.make_inputs(cfg, seed=5, with_dout=False)
    t = to_dev(a)
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], bias, t["keep"], t["g"])
    pba.pba_device_status()
    rz, rg, rb, rw, _ = _ref_inputs(d)
    r_bias = oracle.pair_bias_fwd(rz, rg, rb, rw, EPS)
    fa = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in a.items()}
    r_out, _ = oracle.fwd(fa["q"], fa["k"], fa["v"], r_bias, fa["keep"], fa["g"])
    err = np.abs(out.float().cpu().numpy().astype(np.float64) - r_out)
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (err.max(), err.mean())
