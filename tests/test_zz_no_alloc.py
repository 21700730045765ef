"""pba_bwd_noalloc: the backward pass for callers that cannot allocate device memory
(for instance a plugin inside another framework's executor that owns all device memory,
or a language binding without a device allocator).  It uses the library's built-in
64 MiB scratch array instead of a caller workspace.

The tests call the entry point through the C ABI twice in a row and check each result
against the workspace-taking pba_bwd and against the fp64 oracle, with the tolerance of
the other gradient tests; once with gate and bias, once without either (dgate and dbias
not requested).  They also check that a call leaves the device's free memory unchanged.
The file is collected last."""
import ctypes

import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import GRAD_REL_L2, rel_l2, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as p
    return p


def _call_noalloc(pba, t, out, lse, grads):
    dq, dk, dv, dg, db = grads
    d = pba.make_dims(t["q"], t["k"], t["v"], t.get("g"), out, t.get("bias"), t["keep"], dout=t["dout"])
    ptr = lambda x: None if x is None else x.data_ptr()
    import torch
    st = pba.lib.pba_bwd_noalloc(ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(t.get("bias")),
                                 ptr(t["keep"]), ptr(t.get("g")), ptr(out), ptr(lse), ptr(t["dout"]),
                                 ptr(dq), ptr(dk), ptr(dv), ptr(db), ptr(dg), ctypes.byref(d),
                                 torch.cuda.current_stream().cuda_stream)
    assert st == 0, pba.lib.pba_last_error().decode()
    pba.pba_device_status()


def _run(pba, d, with_gate_bias):
    import torch
    t = to_dev(d)
    g, bias = t.get("g"), t.get("bias")
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], bias, t["keep"], g)
    ref = pba.attention_bwd(t["q"], t["k"], t["v"], bias, t["keep"], g, out, lse, t["dout"],
                            want_dbias=with_gate_bias)
    pba.pba_device_status()
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    orc = oracle.bwd(f["q"], f["k"], f["v"], f.get("bias"), f["keep"], f.get("g"), f["dout"])
    names = ("dq", "dk", "dv", "dgate", "dbias")
    for call in range(2):
        grads = [torch.full_like(t["q"], 3.0), torch.full_like(t["k"], 3.0),
                 torch.full_like(t["v"], 3.0), None, None]
        if with_gate_bias:
            grads[3] = torch.full_like(g, 3.0)
            grads[4] = torch.full_like(ref[4], 3.0)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _call_noalloc(pba, t, out, lse, grads)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        assert free_after >= free_before, "call %d took %d bytes of device memory" % (
            call, free_before - free_after)
        for i, name in enumerate(names):
            if grads[i] is None:
                continue
            got = grads[i].double().cpu().numpy()
            r = rel_l2(got, ref[i].double().cpu().numpy())
            assert r <= GRAD_REL_L2, "call %d: %s relative L2 %.3g against pba_bwd" % (call, name, r)
            r = rel_l2(got, orc[i])
            assert r <= GRAD_REL_L2, "call %d: %s relative L2 %.3g against the oracle" % (call, name, r)


def test_noalloc_matches_pba_bwd_and_oracle_twice(pba):
    cfg = pi.custom("noalloc", B=24, H=2, N=200, c=32, masked=((190, 200),))
    _run(pba, pi.make_inputs(cfg, seed=3), with_gate_bias=True)


def test_noalloc_without_gate_and_bias_twice(pba):
    cfg = pi.custom("noalloc_plain", B=12, H=2, N=136, c=32, masked=((130, 136),), gate=False)
    d = pi.make_inputs(cfg, seed=4)
    d.pop("bias")
    assert "g" not in d
    _run(pba, d, with_gate_bias=False)


def test_noalloc_rejects_sizes_beyond_its_scratch(pba):
    # the triangle attention workload (384 rows of 384 tokens, 4 heads) needs more than
    # 64 MiB of scratch: refused on the host, before any launch (the dummy pointers pass
    # the argument checks, which come first)
    d = pba.dims_dense(384, 4, 384, 384, 32)
    assert pba.pba_bwd_workspace_size(d) > (64 << 20)
    st = pba.lib.pba_bwd_noalloc(*([16] * 14), ctypes.byref(d), None)
    assert st == 2
    assert "scratch" in pba.lib.pba_last_error().decode()


def test_noalloc_checks_arguments_before_scratch_size(pba):
    # a null required pointer is an argument error even when the sizes are too large
    d = pba.dims_dense(384, 4, 384, 384, 32)
    args = [16] * 14
    args[0] = None   # q
    st = pba.lib.pba_bwd_noalloc(*args, ctypes.byref(d), None)
    assert st == 1
