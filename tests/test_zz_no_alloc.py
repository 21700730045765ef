"""pba_bwd_noalloc: the backward pass for callers that cannot allocate device memory
(for instance a plugin inside another framework's executor that owns all device memory,
or a language binding without a device allocator).  It uses the library's built-in
64 MiB scratch array instead of a caller workspace.

The test calls the entry point through the C ABI twice in a row and checks each result
against the workspace-taking pba_bwd, with the tolerance of the other gradient tests.
It lives in a file of its own, collected last."""
import ctypes

import numpy as np
import pytest

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
    d = pba.make_dims(t["q"], t["k"], t["v"], t["g"], out, t["bias"], t["keep"], dout=t["dout"])
    ptr = lambda x: None if x is None else x.data_ptr()
    import torch
    st = pba.lib.pba_bwd_noalloc(ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(t["bias"]),
                                 ptr(t["keep"]), ptr(t["g"]), ptr(out), ptr(lse), ptr(t["dout"]),
                                 ptr(dq), ptr(dk), ptr(dv), ptr(db), ptr(dg), ctypes.byref(d),
                                 torch.cuda.current_stream().cuda_stream)
    assert st == 0, pba.lib.pba_last_error().decode()
    pba.pba_device_status()


def test_noalloc_matches_workspace_entry_point_twice(pba):
    import torch
    cfg = pi.custom("noalloc", B=24, H=2, N=200, c=32, masked=((190, 200),))
    t = to_dev(pi.make_inputs(cfg, seed=3))
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    ref = pba.attention_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], out, lse,
                            t["dout"])
    pba.pba_device_status()
    for _ in range(2):
        grads = (torch.full_like(t["q"], 3.0), torch.full_like(t["k"], 3.0),
                 torch.full_like(t["v"], 3.0), torch.full_like(t["g"], 3.0),
                 torch.full_like(ref[4], 3.0))
        _call_noalloc(pba, t, out, lse, grads)
        for name, got, want in zip(("dq", "dk", "dv", "dgate", "dbias"), grads, ref):
            r = rel_l2(got.double().cpu().numpy(), want.double().cpu().numpy())
            assert r <= GRAD_REL_L2, "%s relative L2 %.3g" % (name, r)


def test_noalloc_rejects_sizes_beyond_its_scratch(pba):
    # the triangle attention workload (384 rows of 384 tokens, 4 heads) needs more than
    # 64 MiB of scratch: refused on the host, before any launch
    d = pba.dims_dense(384, 4, 384, 384, 32)
    assert pba.pba_bwd_workspace_size(d) > (64 << 20)
    st = pba.lib.pba_bwd_noalloc(*([16] * 14), ctypes.byref(d), None)
    assert st == 2
    assert "scratch" in pba.lib.pba_last_error().decode()
