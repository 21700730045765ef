"""GPU backward pass (dq, dk, dv, dgate, dbias) against the fp64 oracle on the same seeded
bf16 inputs: small shapes (full comparison), edge cases, bit-stability of dbias, and the
five workload configurations at full size (whole (b, h) slices and dbias rows sampled).

The bias gradient is the logits' gradient summed over the broadcast rows ("AlphaFold3
open-source implementation" page, Model Efficiency section)."""
import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import (GRAD_REL_L2, assert_grad_close, bf16_to_f64_tensor, rel_l2, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as p
    return p


def _inputs(B, H, Nq, Nk, C, masked=(), gate=True, bias=True, seed=0, per_row_mask=False):
    d = {"q": pi.normal_bf16(seed, 1, (B, Nq, H, C)),
         "k": pi.normal_bf16(seed, 2, (B, Nk, H, C)),
         "v": pi.normal_bf16(seed, 3, (B, Nk, H, C)),
         "dout": pi.normal_bf16(seed, 6, (B, Nq, H, C))}
    if gate:
        d["g"] = pi.normal_bf16(seed, 4, (B, Nq, H, C))
    if bias:
        d["bias"] = pi.normal_bf16(seed, 5, (H, Nq, Nk))
    keep = np.ones(Nk, np.uint8)
    for lo, hi in masked:
        keep[lo:hi] = 0
    if per_row_mask:
        rng = np.random.default_rng(seed + 7)
        keep = np.stack([keep] * B)
        keep &= (rng.random((B, Nk)) > 0.2).astype(np.uint8)
    d["keep"] = keep
    return d


def _gpu_fwd_bwd(pba, t, want_dbias=True):
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t.get("bias"), t.get("keep"), t.get("g"))
    grads = pba.attention_bwd(t["q"], t["k"], t["v"], t.get("bias"), t.get("keep"), t.get("g"),
                              out, lse, t["dout"], want_dbias=want_dbias)
    pba.pba_device_status()
    return out, lse, grads


def _check_full(pba, d):
    t = to_dev(d)
    _, _, (dq, dk, dv, dg, db) = _gpu_fwd_bwd(pba, t)
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    rq, rk, rv, rg, rb = oracle.bwd(f["q"], f["k"], f["v"], f.get("bias"), f["keep"], f.get("g"),
                                    f["dout"])
    assert_grad_close(bf16_to_f64_tensor(dq), rq, "dq")
    assert_grad_close(bf16_to_f64_tensor(dk), rk, "dk")
    assert_grad_close(bf16_to_f64_tensor(dv), rv, "dv")
    if dg is not None:
        assert_grad_close(bf16_to_f64_tensor(dg), rg, "dgate")
    assert_grad_close(db.cpu().numpy().astype(np.float64), rb, "dbias")
    return (dq, dk, dv, dg, db), (rq, rk, rv, rg, rb)


CASES = {
    # name: (B, H, Nq, Nk, C, masked, gate, bias)
    "tiny_triangle_config": (64, 4, 64, 64, 32, ((58, 64),), True, True),
    "ragged_two_tiles": (5, 2, 200, 200, 32, ((190, 200),), True, True),
    "c24_padded": (6, 3, 136, 136, 24, (), True, True),
    "c64": (3, 2, 136, 136, 64, ((0, 3),), True, True),
    "c16": (4, 2, 72, 72, 16, (), True, True),
    "c8": (3, 1, 40, 40, 8, (), True, True),
    "nq_ne_nk": (4, 2, 72, 200, 32, ((100, 130),), True, True),
    "nq_gt_nk": (3, 2, 264, 40, 32, (), True, True),
    "no_bias_no_gate": (9, 2, 128, 128, 32, (), False, False),
    "no_gate": (5, 2, 136, 136, 32, ((130, 136),), False, True),
    "single_row_head": (1, 1, 256, 256, 32, ((250, 256),), True, True),
    "three_key_tiles": (10, 2, 384, 384, 32, ((100, 140), (300, 384)), True, True),
    "many_rows_split": (70, 1, 128, 128, 32, ((120, 128),), True, True),
    # more (b, h, key tile) items than SMs: CTAs of the dq/dk/dv kernel run several items,
    # crossing K/V stages and dK/dV buffers (one of each at c = 64)
    "multi_item_c32": (40, 4, 136, 136, 32, ((130, 136),), True, True),
    "multi_item_c24": (30, 4, 200, 200, 24, ((190, 200),), True, True),
    "multi_item_c16": (40, 4, 72, 72, 16, (), True, True),
    "multi_item_c64": (24, 4, 136, 136, 64, ((0, 3),), True, True),
    # the dbias kernel's element-wise warpgroups own keys 0-47, 48-95 and 96-127 of a key
    # tile and skip the mask test when their whole range is attended: masked keys on and
    # around those edges, in both key tiles, and ranges left wholly attended beside them
    "mask_on_dbias_group_edges": (6, 2, 256, 256, 32,
                                  ((40, 50), (94, 97), (120, 121), (176, 180), (200, 208)), True, True),
    "mask_single_edge_keys": (5, 2, 256, 256, 32, ((47, 49), (95, 97), (223, 225)), True, True),
    "mask_on_dbias_group_edges_c16": (6, 2, 256, 256, 16, ((40, 50), (94, 97), (176, 180)), True, True),
    "mask_on_dbias_group_edges_c64": (4, 2, 256, 256, 64, ((47, 49), (95, 97), (200, 208)), True, True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_bwd_matches_oracle(pba, name):
    B, H, Nq, Nk, C, masked, gate, bias = CASES[name]
    _check_full(pba, _inputs(B, H, Nq, Nk, C, masked, gate, bias))


def test_bwd_per_row_mask(pba):
    _check_full(pba, _inputs(6, 2, 136, 136, 32, ((130, 136),), per_row_mask=True))


def test_bwd_per_row_mask_on_dbias_group_edges(pba):
    # per-row masks (about 20 % of keys dropped per row b) on top of masked group edges
    _check_full(pba, _inputs(6, 2, 256, 256, 32, ((46, 50), (94, 98)), per_row_mask=True, seed=3))


def test_bwd_fully_masked_rows_give_zero(pba):
    import torch
    d = _inputs(3, 2, 64, 64, 32, ((0, 64),))
    t = to_dev(d)
    _, _, (dq, dk, dv, dg, db) = _gpu_fwd_bwd(pba, t)
    for g in (dq, dk, dv, dg, db):
        assert torch.all(g == 0)


def test_dbias_bit_stable_over_runs(pba):
    import torch
    t = to_dev(_inputs(48, 2, 200, 200, 32, ((190, 200),)))
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    dbs = []
    for _ in range(3):
        *_, db = pba.attention_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], out, lse,
                                   t["dout"])
        dbs.append(db.clone())
    torch.cuda.synchronize()
    assert torch.equal(dbs[0], dbs[1]) and torch.equal(dbs[0], dbs[2])


def test_bwd_without_dbias_output(pba):
    d = _inputs(4, 2, 136, 136, 32, ((130, 136),))
    t = to_dev(d)
    _, _, (dq, dk, dv, dg, db) = _gpu_fwd_bwd(pba, t, want_dbias=False)
    assert db is None
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    rq, rk, rv, rg, _ = oracle.bwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f["g"], f["dout"])
    assert_grad_close(bf16_to_f64_tensor(dq), rq, "dq")
    assert_grad_close(bf16_to_f64_tensor(dv), rv, "dv")


def test_bwd_no_queries_zeroes_key_grads(pba):
    import torch
    B, H, Nk, C = 2, 2, 64, 32
    q = torch.empty(B, 0, H, C, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(B, Nk, H, C, device="cuda").bfloat16()
    v = torch.randn(B, Nk, H, C, device="cuda").bfloat16()
    lse = torch.empty(B, H, 0, device="cuda")
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(v, 7.0)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    pba.pba_bwd(q, k, v, None, None, None, q, lse, q, q, dk, dv, None, None, ws)
    pba.pba_device_status()
    assert torch.all(dk == 0) and torch.all(dv == 0)


def test_workspace_too_small_is_rejected(pba):
    import torch
    t = to_dev(_inputs(2, 2, 64, 64, 32))
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    dq, dk, dv, dg = (torch.empty_like(t["q"]) for _ in range(4))
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(pba.PbaError) as ei:
        pba.pba_bwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"], out, lse, t["dout"],
                    dq, dk, dv, None, dg, ws)
    assert ei.value.status == 5


def _sample_slices(B, H, n=3, seed=1):
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (B - 1, H - 1)}
    while len(picks) < min(n, B * H):
        picks.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(picks)


@pytest.mark.parametrize("cfg_name", ["C1", "C2", "C3", "C4", "C5"])
def test_bwd_full_config_sampled(pba, cfg_name):
    """Full-size workloads in the benchmark's launch configuration: whole (b, h) slices of
    dq, dk, dv, dgate and whole rows of dbias compared against the oracle."""
    import torch
    cfg = pi.CONFIGS[cfg_name]
    d = pi.make_inputs(cfg, seed=0)
    t = to_dev(d)
    out, lse, (dq, dk, dv, dg, db) = _gpu_fwd_bwd(pba, t)
    keep = d["keep"]
    for b, h in _sample_slices(cfg.B, cfg.H):
        sl = lambda a: pi.bf16_bits_to_f64(a[b, :, h])
        rq, rk, rv, rg, _ = oracle.bwd_slice(sl(d["q"]), sl(d["k"]), sl(d["v"]),
                                             pi.bf16_bits_to_f64(d["bias"][h]), keep, sl(d["g"]),
                                             sl(d["dout"]))
        for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv), ("dgate", dg, rg)):
            assert_grad_close(got[b, :, h].float().cpu().numpy().astype(np.float64), ref,
                              "%s[%d,:,%d]" % (name, b, h))
    # dbias rows: the sum over all B rows, for a few (h, i)
    rng = np.random.default_rng(2)
    for h in sorted({0, cfg.H - 1}):
        hs = lambda a: pi.bf16_bits_to_f64(a[:, :, h:h + 1])
        args = (hs(d["q"]), hs(d["k"]), hs(d["v"]), pi.bf16_bits_to_f64(d["bias"][h:h + 1]), keep,
                hs(d["g"]), hs(d["dout"]))
        for i in sorted({0, cfg.N - 1, int(rng.integers(cfg.N))}):
            ref = oracle.dbias_row(*args, 0, i)
            got = db[h, i].cpu().numpy().astype(np.float64)
            r = rel_l2(got, ref)
            assert r <= GRAD_REL_L2, "dbias[%d,%d] rel L2 %.3g" % (h, i, r)
    # properties at any size: all finite, and dbias rows sum to zero (softmax shift
    # invariance) up to the rounding of D = sum_c dout * out, which uses the bf16 `out`
    # (relative error <= 2^-8 per product): |sum_j dbias[h,i,j]| <= 2^-8 sum_b,c |dout out|
    assert bool(torch.isfinite(db).all())
    row_sums = db.double().sum(-1).abs()
    bound = (t["dout"].double() * out.double()).abs().sum(dim=(0, 3)).transpose(0, 1) * 2.0 ** -8
    assert bool((row_sums <= bound + 1e-6).all()), float((row_sums - bound).max())


def test_dbias_whole_head_large_triangle(pba):
    """Large triangle attention (768 rows x 768 keys, 4 heads, c = 32), the benchmark's
    launch configuration: every one of the 768 dbias rows of head 0 (each the sum of dS over
    all 768 broadcast rows) compared against the oracle, row by row and as a whole."""
    from concurrent.futures import ThreadPoolExecutor
    cfg = pi.CONFIGS["C5"]
    d = pi.make_inputs(cfg, seed=0)
    t = to_dev(d)
    _, _, (_, _, _, _, db) = _gpu_fwd_bwd(pba, t)
    h = 0
    hs = lambda a: pi.bf16_bits_to_f64(a[:, :, h:h + 1])
    args = (hs(d["q"]), hs(d["k"]), hs(d["v"]), pi.bf16_bits_to_f64(d["bias"][h:h + 1]), d["keep"],
            hs(d["g"]), hs(d["dout"]))
    # the oracle's C entry point runs without the GIL: one row per task
    with ThreadPoolExecutor(max_workers=max(1, min(32, oracle.threads()))) as ex:
        rows = list(ex.map(lambda i: oracle.dbias_row(*args, 0, i), range(cfg.N)))
    ref = np.stack(rows)
    got = db[h].cpu().numpy().astype(np.float64)
    assert rel_l2(got, ref) <= GRAD_REL_L2, "dbias head 0 rel L2 %.3g" % rel_l2(got, ref)
    worst = max(range(cfg.N), key=lambda i: rel_l2(got[i], ref[i]))
    assert rel_l2(got[worst], ref[worst]) <= GRAD_REL_L2, \
        "dbias[0,%d] rel L2 %.3g" % (worst, rel_l2(got[worst], ref[worst]))
