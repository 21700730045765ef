"""The library's calls allocate nothing and are stream-ordered, so a whole fwd+bwd step can be
captured once in a CUDA graph and replayed: the replay gives the eager call's results (bit for
bit where no floating-point atomics are involved; dq, accumulated with reductions in any
order, within the gradient tolerance)."""
import numpy as np
import pytest

import pba_inputs as pi
from pba_testlib import assert_grad_close, to_dev

pytestmark = pytest.mark.gpu


def test_fwd_bwd_step_replays_in_a_cuda_graph():
    import torch
    import pair_biased_attention_gated_b200 as pba
    cfg = pi.custom("graph", B=6, H=2, N=200, c=32, masked=((190, 200),))
    t = to_dev(pi.make_inputs(cfg, seed=9))
    q, k, v, g, bias, keep, dout = t["q"], t["k"], t["v"], t["g"], t["bias"], t["keep"], t["dout"]
    B, N, H, C = q.shape
    out, lse = torch.empty_like(q), torch.empty(B, H, N, device="cuda")
    dq, dk, dv, dg = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g)
    db = torch.empty(H, N, N, device="cuda")
    ws = torch.empty(pba.pba_bwd_workspace_size(pba.make_dims(q, k, v, g, out, bias, keep)),
                     dtype=torch.uint8, device="cuda")

    def step():
        pba.pba_fwd(q, k, v, bias, keep, g, out, lse)
        pba.pba_bwd(q, k, v, bias, keep, g, out, lse, dout, dq, dk, dv, db, dg, ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    pba.pba_device_status()
    ref = [x.clone() for x in (out, lse, dq, dk, dv, db, dg)]

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for x in (out, lse, dq, dk, dv, db, dg):
        x.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    pba.pba_device_status()
    for name, a, b in zip(("out", "lse", "dk", "dv", "dbias", "dgate"), (ref[0], ref[1], ref[3], ref[4], ref[5], ref[6]),
                          (out, lse, dk, dv, db, dg)):
        assert torch.equal(a, b), name
    assert_grad_close(dq.float().cpu().numpy().astype(np.float64), ref[2].float().cpu().numpy().astype(np.float64), "dq")
    del graph
