"""Row-sharded backward pass on the GPU (pair_biased_attention_gated_b200/sharded.py): the
library computes each row group's bias-gradient partial and pba_dbias_sum adds them in
group order.  Two ranks are emulated on the one GPU one after the other (their partials
concatenated in rank order, which is the order the all-gather delivers; no kernel of one
waits on the other): the bias gradient is bit-identical to one rank holding every group,
and matches the oracle on the whole batch within the gradient tolerance.

Row sharding as on the Design-CP page ("Context Parallelism for Design of Protein
Nanoparticles", Method); the bias gradient is the sum over the broadcast rows
("AlphaFold3 open-source implementation" page, Model Efficiency section)."""
import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import assert_grad_close, bf16_to_f64_tensor, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as p
    return p


def test_two_emulated_ranks_match_one_bit_for_bit(pba):
    import torch
    from pair_biased_attention_gated_b200 import sharded as sh
    B, GROUPS = 22, 4
    cfg = pi.custom("shard_gpu", B=B, H=2, N=200, c=32, masked=((190, 200),))
    d = pi.make_inputs(cfg, seed=9)
    t = to_dev(d)
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    rows = lambda x, lo, hi: x[lo:hi]
    args = ("q", "k", "v")

    def rank_part(world, rank):
        lo, hi = sh.rank_rows(B, GROUPS, world, rank)
        r = lambda x: rows(x, lo, hi)
        ws = sh.workspace_for(r(t["q"]), r(t["k"]), r(t["v"]), r(t["g"]), r(out), t["bias"], t["keep"],
                              B, GROUPS, world, rank)
        return sh.local_backward(r(t["q"]), r(t["k"]), r(t["v"]), t["bias"], t["keep"], r(t["g"]),
                                 r(out), r(lse), r(t["dout"]), B_total=B, groups=GROUPS,
                                 world=world, rank=rank, workspace=ws)

    one = rank_part(1, 0)
    db1 = sh.sum_partials(one[4])
    two = [rank_part(2, r) for r in range(2)]
    db2 = sh.sum_partials(torch.cat([two[0][4], two[1][4]], dim=0))
    pba.pba_device_status()
    assert torch.equal(db1, db2)
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    rq, rk, rv, rg, rb = oracle.bwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f["g"], f["dout"])
    assert_grad_close(db2.cpu().numpy().astype(np.float64), rb, "dbias")
    dq = torch.cat([two[0][0], two[1][0]], dim=0)
    dv = torch.cat([two[0][2], two[1][2]], dim=0)
    assert_grad_close(bf16_to_f64_tensor(dq), rq, "dq")
    assert_grad_close(bf16_to_f64_tensor(dv), rv, "dv")


def test_dbias_sum_adds_in_order(pba):
    import torch
    g = torch.Generator().manual_seed(0)
    parts = (torch.randn(5, 3, 7, 9, generator=g) * torch.tensor([1e6, 1.0, -1e6, 1e-3, 3.0]).view(5, 1, 1, 1)).float()
    want = parts[0].clone()
    for p in range(1, 5):
        want += parts[p]
    from pair_biased_attention_gated_b200 import sharded as sh
    for n_last in (9, 8):   # odd length: the element-wise path; multiple of four: the vector path
        pp = parts[..., :n_last].contiguous().cuda()
        got = sh.sum_partials(pp).cpu()
        w = want[..., :n_last]
        assert torch.equal(got, w.contiguous())
