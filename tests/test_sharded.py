"""Row-sharded backward pass across ranks (pair_biased_attention_gated_b200/sharded.py) on
CPU: the row groups and their assignment to ranks, and two gloo ranks that each compute
their rows, all-gather the bias-gradient partials and add them in group order.  The
per-group backward is the fp64 oracle here (the sharding and the exchange are what is
tested); the bias gradient must come out bit-identical on both ranks and to one rank
holding every group, and equal to the oracle on the whole batch.

The row sharding follows the Design-CP page ("Context Parallelism for Design of Protein
Nanoparticles", Method); the bias gradient is the sum over the broadcast rows ("AlphaFold3
open-source implementation" page, Model Efficiency section)."""
import importlib.util
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _sharded():
    spec = importlib.util.spec_from_file_location(
        "pba_sharded", os.path.join(ROOT, "pair_biased_attention_gated_b200", "sharded.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


B, H, N, C, GROUPS = 7, 2, 24, 8, 4


def _inputs():
    import pba_inputs as pi
    cfg = pi.custom("shard", B=B, H=H, N=N, c=C, masked=((20, 24),))
    d = pi.make_inputs(cfg, seed=5)
    f = {k: (torch.from_numpy(pi.bf16_bits_to_f64(v)) if k != "keep" else torch.from_numpy(v))
         for k, v in d.items()}
    import oracle
    out, lse = oracle.fwd(f["q"].numpy(), f["k"].numpy(), f["v"].numpy(), f["bias"].numpy(),
                          f["keep"].numpy(), f["g"].numpy())
    f["out"], f["lse"] = torch.from_numpy(out), torch.from_numpy(lse)
    return f


def _oracle_bwd_group(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dgate, dbias, ws):
    import oracle
    n = lambda t: None if t is None else t.numpy()
    rq, rk, rv, rg, rb = oracle.bwd(n(q), n(k), n(v), n(bias), n(key_mask), n(gate), n(dout))
    dq.copy_(torch.from_numpy(rq))
    dk.copy_(torch.from_numpy(rk))
    dv.copy_(torch.from_numpy(rv))
    if dgate is not None:
        dgate.copy_(torch.from_numpy(rg))
    dbias.copy_(torch.from_numpy(rb).float())


def _ordered_sum(parts, out):
    acc = parts[0].clone()
    for p in range(1, parts.shape[0]):
        acc += parts[p]
    out.copy_(acc)


def _run(sh, f, world, rank, pg=None):
    lo, hi = sh.rank_rows(B, GROUPS, world, rank)
    r = lambda t: t[lo:hi]
    return sh.sharded_backward(r(f["q"]), r(f["k"]), r(f["v"]), f["bias"], f["keep"], r(f["g"]),
                               r(f["out"]), r(f["lse"]), r(f["dout"]), B_total=B, groups=GROUPS,
                               pg=pg, world=world, rank=rank, bwd_group=_oracle_bwd_group,
                               sum_parts=_ordered_sum)


def test_row_groups_cover_the_rows_in_order():
    sh = _sharded()
    gs = sh.row_groups(7, 4)
    assert gs == [(0, 2), (2, 4), (4, 6), (6, 7)]
    assert sh.row_groups(3, 4) == [(0, 1), (1, 2), (2, 3), (3, 3)]
    assert list(sh.rank_groups(4, 2, 1)) == [2, 3]
    assert sh.rank_rows(7, 4, 2, 0) == (0, 4) and sh.rank_rows(7, 4, 2, 1) == (4, 7)
    with pytest.raises(ValueError):
        sh.rank_groups(6, 4, 0)


def test_one_rank_matches_the_oracle_on_the_whole_batch():
    sh = _sharded()
    f = _inputs()
    dq, dk, dv, dg, db = _run(sh, f, 1, 0)
    import oracle
    rq, rk, rv, rg, rb = oracle.bwd(*(f[k].numpy() for k in ("q", "k", "v", "bias", "keep", "g", "dout")))
    np.testing.assert_allclose(dq.numpy(), rq, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv.numpy(), rv, rtol=0, atol=1e-12)
    # the ordered fp32 sum of the groups' fp32 partials against the fp64 whole-batch sum
    np.testing.assert_allclose(db.numpy(), rb, rtol=1e-5, atol=1e-6)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sh = _sharded()
        f = _inputs()
        dq, dk, dv, dg, db = _run(sh, f, world, rank, pg=dist)
        out[rank] = (dq.numpy().tobytes(), dv.numpy().tobytes(), db.numpy().tobytes())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_give_bit_identical_dbias():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    sh = _sharded()
    f = _inputs()
    dq1, _, dv1, _, db1 = _run(sh, f, 1, 0)
    for r in range(world):
        assert out[r][2] == db1.numpy().tobytes(), "rank %d dbias differs" % r
        lo, hi = sh.rank_rows(B, GROUPS, world, r)
        assert out[r][0] == dq1[lo:hi].numpy().tobytes()
        assert out[r][1] == dv1[lo:hi].numpy().tobytes()
