"""The backward pass runs its dbias kernel on a second stream of the library's and makes the
caller's stream wait for it, so everything stays ordered on the caller's stream.  Two
problems launched back to back on two different streams (sharing that second stream), with
no host synchronisation in between, give the same results as each problem run alone; and a
caller that reads dbias right after the call on its own stream sees the finished values."""
import numpy as np
import pytest

import pba_inputs as pi
from pba_testlib import assert_grad_close, to_dev

pytestmark = pytest.mark.gpu


def _problem(seed, N):
    import torch
    import pair_biased_attention_gated_b200 as pba
    cfg = pi.custom("streams%d" % seed, B=5, H=2, N=N, c=32, masked=((N - 9, N),))
    t = to_dev(pi.make_inputs(cfg, seed=seed))
    q, k, v, g, bias, keep, dout = t["q"], t["k"], t["v"], t["g"], t["bias"], t["keep"], t["dout"]
    B, N, H, C = q.shape
    out, lse = torch.empty_like(q), torch.empty(B, H, N, device="cuda")
    pba.pba_fwd(q, k, v, bias, keep, g, out, lse)
    res = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=torch.empty_like(g), db=torch.empty(H, N, N, device="cuda"))
    ws = torch.empty(pba.pba_bwd_workspace_size(pba.make_dims(q, k, v, g, out, bias, keep)),
                     dtype=torch.uint8, device="cuda")

    def bwd():
        pba.pba_bwd(q, k, v, bias, keep, g, out, lse, dout, res["dq"], res["dk"], res["dv"], res["db"],
                    res["dg"], ws)
    return bwd, res


def test_two_streams_back_to_back_match_each_alone():
    import torch
    import pair_biased_attention_gated_b200 as pba
    bwd_a, res_a = _problem(21, 200)
    bwd_b, res_b = _problem(22, 264)
    torch.cuda.synchronize()
    # each alone
    bwd_a()
    torch.cuda.synchronize()
    ref_a = {k: x.clone() for k, x in res_a.items()}
    bwd_b()
    torch.cuda.synchronize()
    ref_b = {k: x.clone() for k, x in res_b.items()}
    for x in list(res_a.values()) + list(res_b.values()):
        x.zero_()
    torch.cuda.synchronize()
    # back to back on two streams; each stream then copies its dbias right away
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(sa):
        bwd_a()
        copy_a = res_a["db"].clone()
    with torch.cuda.stream(sb):
        bwd_b()
        copy_b = res_b["db"].clone()
    torch.cuda.synchronize()
    pba.pba_device_status()
    for ref, res, copy in ((ref_a, res_a, copy_a), (ref_b, res_b, copy_b)):
        assert torch.equal(ref["db"], res["db"]) and torch.equal(ref["db"], copy), "dbias"
        for name in ("dk", "dv", "dg"):
            assert torch.equal(ref[name], res[name]), name
        assert_grad_close(res["dq"].float().cpu().numpy().astype(np.float64),
                          ref["dq"].float().cpu().numpy().astype(np.float64), "dq")
