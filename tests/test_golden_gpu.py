"""The hand-worked two-token example of tests/golden/two_token.json on the GPU.

Pair-biased attention as stated on the "AlphaFold3 open-source implementation" page,
Model Efficiency section: the pair bias is added after the key-query dot product, and its
gradient is the gradient of the scaled logits summed over the broadcast axis.  The example
(B = 1, H = 1, N = 2, c = 1, scale = 1) is embedded at head dimension 32: channel 0 carries
the example's values, channels 1..31 are zero, and the scale is passed explicitly as 1.
The kernels must reproduce the hand-derived outputs and gradients within the bf16
tolerances, give exact zeros in the padding channels, and agree with the oracle run on the
same bf16 inputs (the example's ln 3 - 2 is not a bf16 number, so the GPU sees it rounded).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from pba_testlib import (GRAD_REL_L2, LSE_MAX_ABS, OUT_MAX_ABS, assert_grad_close, rel_l2)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_token.json")
C = 32


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as p
    return p


def _num(x):
    return {"ln3-2": math.log(3.0) - 2.0, "ln2": math.log(2.0), "ln4": math.log(4.0)}.get(x, x) \
        if isinstance(x, str) else float(x)


def _embed(vals):
    """[N] values -> a [1, N, 1, C] bf16 tensor with the values in channel 0."""
    import torch
    t = torch.zeros(1, len(vals), 1, C, dtype=torch.float32)
    t[0, :, 0, 0] = torch.tensor([_num(x) for x in vals], dtype=torch.float32)
    return t.to(torch.bfloat16).cuda()


def test_two_token_example_on_gpu(pba):
    import torch
    with open(GOLDEN) as f:
        gold = json.load(f)
    inp, exp = gold["inputs"], gold["expected"]
    assert inp["scale"] == 1.0 and inp["N"] == 2
    q, k, v, g, dout = (_embed(inp[n]) for n in ("q", "k", "v", "g", "dout"))
    # bias [1, 2, 2] inside rows of 8 keys (the row stride must be a multiple of 8)
    bias_buf = torch.zeros(1, 2, 8, dtype=torch.float32)
    bias_buf[0, :, :2] = torch.tensor([[_num(x) for x in r] for r in inp["bias"]])
    bias = bias_buf.to(torch.bfloat16).cuda()[:, :, :2]
    out, lse = pba.attention_fwd(q, k, v, bias, None, g, scale=1.0)
    dq, dk, dv, dg, db = pba.attention_bwd(q, k, v, bias, None, g, out, lse, dout, scale=1.0)
    pba.pba_device_status()

    ch0 = lambda t: t[0, :, 0, 0].double().cpu().numpy()
    # against the hand-derived values (exact inputs)
    want_out = np.array([_num(x) for x in exp["out"]])
    assert np.abs(ch0(out) - want_out).max() <= OUT_MAX_ABS
    want_lse = np.array([_num(x) for x in exp["lse"]])
    assert np.abs(lse[0, 0].double().cpu().numpy() - want_lse).max() <= LSE_MAX_ABS
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv), ("dg", dg)):
        want = np.array([_num(x) for x in exp[name]])
        assert rel_l2(ch0(got), want) <= GRAD_REL_L2, (name, ch0(got), want)
    want_db = np.array([[_num(x) for x in r] for r in exp["dbias"]])
    assert rel_l2(db[0].double().cpu().numpy(), want_db) <= GRAD_REL_L2
    # the padding channels carry nothing
    for name, t in (("out", out), ("dq", dq), ("dk", dk), ("dv", dv), ("dg", dg)):
        assert bool((t[..., 1:] == 0).all()), name
    # against the oracle on the same (bf16-rounded) inputs
    f = lambda t: t.double().cpu().numpy()
    fb = f(bias)
    ro, rl = oracle.fwd(f(q), f(k), f(v), fb, None, f(g), scale=1.0)
    assert np.abs(f(out) - ro).max() <= OUT_MAX_ABS
    assert np.abs(f(lse) - rl).max() <= LSE_MAX_ABS
    rq, rk, rv, rg, rb = oracle.bwd(f(q), f(k), f(v), fb, None, f(g), f(dout), scale=1.0)
    assert_grad_close(f(dq), rq, "dq")
    assert_grad_close(f(dk), rk, "dk")
    assert_grad_close(f(dv), rv, "dv")
    assert_grad_close(f(dg), rg, "dgate")
    assert_grad_close(f(db), rb, "dbias")
