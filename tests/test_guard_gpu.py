"""Guard bands around every output and workspace (in place of a memory checker): each buffer
the library writes is a view into a larger allocation whose bytes before and after it hold a
NaN pattern.  After the call the guards must be untouched (no write out of bounds), the
outputs must hold no pattern (written in full, never left partly unset or accumulated into),
and the results must equal those of the same call on fresh allocations.  Covers the
attention forward and backward (dense, head dims 24 and 64, local attention), MSA
pair-weighted averaging and the pair-bias prologue."""
import math

import numpy as np
import pytest

import pba_inputs as pi
from pba_testlib import rel_l2, to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096   # elements on each side (keeps every view 16-byte and 256-byte aligned)


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as m
    return m


class Guarded:
    """A tensor of `shape` inside an allocation with GUARD elements on either side; every
    element starts as a NaN bit pattern."""

    def __init__(self, shape, dtype):
        import torch
        self.idt, self.pat = {torch.bfloat16: (torch.int16, 0x7FC1),
                              torch.float32: (torch.int32, 0x7FC00001),
                              torch.uint8: (torch.uint8, 0xA5)}[dtype]
        self.n = math.prod(shape)
        self.buf = torch.empty(self.n + 2 * GUARD, dtype=dtype, device="cuda")
        self.buf.view(self.idt).fill_(self.pat)
        self.t = self.buf[GUARD:GUARD + self.n].view(shape)

    def check(self, name, written=True):
        raw = self.buf.view(self.idt)
        assert bool((raw[:GUARD] == self.pat).all()), "%s: guard before it overwritten" % name
        assert bool((raw[GUARD + self.n:] == self.pat).all()), "%s: guard after it overwritten" % name
        if written:
            assert not bool((raw[GUARD:GUARD + self.n] == self.pat).any()), "%s: not written in full" % name


def _close(got, ref, name, tol=2e-3):
    import torch
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), "%s: finiteness differs" % name
    assert np.array_equal(g[~fin], r[~fin]), "%s: non-finite values differ" % name
    if fin.any():
        assert rel_l2(g[fin], r[fin]) <= tol, "%s: differs from the call on fresh buffers" % name


def _attention_inputs(B, H, N, C, masked):
    d = {"q": pi.normal_bf16(0, 1, (B, N, H, C)), "k": pi.normal_bf16(0, 2, (B, N, H, C)),
         "v": pi.normal_bf16(0, 3, (B, N, H, C)), "g": pi.normal_bf16(0, 4, (B, N, H, C)),
         "bias": pi.normal_bf16(0, 5, (H, N, N)), "dout": pi.normal_bf16(0, 6, (B, N, H, C))}
    keep = np.ones(N, np.uint8)
    for lo, hi in masked:
        keep[lo:hi] = 0
    d["keep"] = keep
    return to_dev(d)


ATTENTION_CASES = {
    # name: (B, H, N, C, masked key ranges, window)
    "c24_ragged": (3, 2, 200, 24, ((190, 200),), -1),
    "c64_two_tiles": (2, 2, 136, 64, ((0, 9),), -1),
    "c32_local_window1": (2, 2, 392, 32, ((384, 392),), 1),
}


@pytest.mark.parametrize("name", sorted(ATTENTION_CASES))
def test_attention_writes_only_its_outputs(pba, name):
    import torch
    B, H, N, C, masked, window = ATTENTION_CASES[name]
    t = _attention_inputs(B, H, N, C, masked)
    q, k, v, g, bias, keep, dout = (t[x] for x in ("q", "k", "v", "g", "bias", "keep", "dout"))
    r_out, r_lse = pba.attention_fwd(q, k, v, bias, keep, g, window=window)
    r_grads = pba.attention_bwd(q, k, v, bias, keep, g, r_out, r_lse, dout, window=window)

    out, lse = Guarded((B, N, H, C), torch.bfloat16), Guarded((B, H, N), torch.float32)
    pba.pba_fwd(q, k, v, bias, keep, g, out.t, lse.t, window=window)
    grads = [Guarded((B, N, H, C), torch.bfloat16) for _ in range(4)]   # dq, dk, dv, dgate
    dbias = Guarded((H, N, N), torch.float32)
    dims = pba.make_dims(q, k, v, g, out.t, bias, keep, 0.0, dout=dout)
    ws = Guarded((pba.pba_bwd_workspace_size(dims),), torch.uint8)
    dq, dk, dv, dg = (x.t for x in grads)
    pba.pba_bwd(q, k, v, bias, keep, g, out.t, lse.t, dout, dq, dk, dv, dbias.t, dg, ws.t,
                window=window)
    pba.pba_device_status()

    out.check("out"), lse.check("lse"), dbias.check("dbias"), ws.check("workspace", written=False)
    for x, nm in zip(grads, ("dq", "dk", "dv", "dgate")):
        x.check(nm)
    assert torch.equal(out.t, r_out) and torch.equal(lse.t, r_lse)
    rq, rk, rv, rg, rb = r_grads
    for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv"), (dg, rg, "dgate"),
                         (dbias.t, rb, "dbias")):
        _close(got, ref, nm)


def test_pwa_writes_only_its_outputs(pba):
    import ctypes
    import torch
    B, H, N, C = 6, 2, 200, 32
    t = _attention_inputs(B, H, N, C, ((190, 200),))
    v, g, bias, keep, dout = (t[x] for x in ("v", "g", "bias", "keep", "dout"))
    r_out, r_lse = pba.pwa_fwd(v, bias, keep, g)
    r_dv, r_dg, r_db = pba.pwa_bwd(v, bias, keep, g, r_out, dout)

    out, lse = Guarded((B, N, H, C), torch.bfloat16), Guarded((H, N), torch.float32)
    d = pba.pwa_dims(v, g, out.t, bias, keep)
    ws_f = Guarded((int(pba.lib.pba_pwa_fwd_workspace_size(ctypes.byref(d))),), torch.uint8)
    pba.pba_pwa_fwd(v, bias, keep, g, out.t, lse.t, ws_f.t)
    dv, dg = Guarded((B, N, H, C), torch.bfloat16), Guarded((B, N, H, C), torch.bfloat16)
    db = Guarded((H, N, N), torch.float32)
    d = pba.pwa_dims(v, g, out.t, bias, keep, dout=dout)
    ws_b = Guarded((int(pba.lib.pba_pwa_bwd_workspace_size(ctypes.byref(d))),), torch.uint8)
    pba.pba_pwa_bwd(v, bias, keep, g, out.t, dout, dv.t, db.t, dg.t, ws_b.t)
    pba.pba_device_status()

    out.check("out"), lse.check("lse_w"), dv.check("dv"), dg.check("dgate"), db.check("dbias")
    ws_f.check("forward workspace", written=False), ws_b.check("backward workspace", written=False)
    for got, ref, nm in ((out.t, r_out, "out"), (lse.t, r_lse, "lse_w"), (dv.t, r_dv, "dv"),
                         (dg.t, r_dg, "dgate"), (db.t, r_db, "dbias")):
        _close(got, ref, nm)


def test_pair_bias_writes_only_its_outputs(pba):
    import ctypes
    import torch
    Ni, Nj, Cz, H = 40, 72, 128, 4
    d = pi.make_pair_bias_inputs(Ni, Nj, Cz, H, seed=0)
    z = torch.from_numpy(d["z"].view(np.int16)).view(torch.bfloat16).cuda()
    gamma, beta, w, dbias = (torch.from_numpy(d[x]).cuda() for x in ("gamma", "beta", "w", "dbias"))
    r_bias = pba.pair_bias_fwd(z, gamma, beta, w)
    r_dz, r_dw, r_dgamma, r_dbeta = pba.pair_bias_bwd(z, gamma, beta, w, dbias)

    bias = Guarded((H, Ni, Nj), torch.bfloat16)
    pba.pba_pair_bias_fwd(z, gamma, beta, w, bias.t)
    dz = Guarded((Ni, Nj, Cz), torch.bfloat16)
    dw = Guarded((Cz, H), torch.float32)
    dgamma, dbeta = Guarded((Cz,), torch.float32), Guarded((Cz,), torch.float32)
    dims = pba.pair_bias_dims(z, dbias=dbias)
    ws = Guarded((max(int(pba.lib.pba_pair_bias_bwd_workspace_size(ctypes.byref(dims))), 256),),
                 torch.uint8)
    pba.pba_pair_bias_bwd(z, gamma, beta, w, dbias, dz.t, dw.t, dgamma.t, dbeta.t, ws.t)
    pba.pba_device_status()

    bias.check("bias"), dz.check("dz"), dw.check("dw"), dgamma.check("dgamma"), dbeta.check("dbeta")
    ws.check("workspace", written=False)
    for got, ref, nm in ((bias.t, r_bias, "bias"), (dz.t, r_dz, "dz"), (dw.t, r_dw, "dw"),
                         (dgamma.t, r_dgamma, "dgamma"), (dbeta.t, r_dbeta, "dbeta")):
        _close(got, ref, nm)
