"""Pins of the oracle for MSA pair-weighted averaging (oracle.pwa_fwd / oracle.pwa_bwd):
the hand-worked example of tests/golden/pwa_two_token.json, the identity with the pinned
attention oracle at q = 0 (the pair-weighted average is pair-biased attention without its
key-query term), central finite differences of the forward for every gradient, and
closed-form invariants."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pwa_two_token.json")


def _val(x):
    if isinstance(x, str):
        return {"ln3": math.log(3.0), "ln4": math.log(4.0), "ln2": math.log(2.0)}[x]
    return float(x)


def _rand(B, H, N, C, masked, gate, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((B, N, H, C))
    bias = rng.standard_normal((H, N, N))
    g = rng.standard_normal((B, N, H, C)) if gate else None
    dout = rng.standard_normal((B, N, H, C))
    keep = np.ones(N, dtype=np.uint8)
    for lo, hi in masked:
        keep[lo:hi] = 0
    return v, bias, keep, g, dout


def test_two_token_golden():
    d = json.load(open(GOLDEN))
    inp, exp = d["inputs"], d["expected"]
    v = np.array(inp["v"]).reshape(1, 2, 1, 1)
    bias = np.array([[_val(x) for x in r] for r in inp["bias"]]).reshape(1, 2, 2)
    g = np.array(inp["g"]).reshape(1, 2, 1, 1)
    dout = np.array(inp["dout"]).reshape(1, 2, 1, 1)
    out, lse = oracle.pwa_fwd(v, bias, None, g)
    np.testing.assert_allclose(out.ravel(), exp["out"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse.ravel(), [_val(x) for x in exp["lse_w"]], rtol=0, atol=1e-14)
    dv, dg, db = oracle.pwa_bwd(v, bias, None, g, dout)
    np.testing.assert_allclose(dv.ravel(), exp["dv"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dg.ravel(), exp["dg"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(db.reshape(2, 2), exp["dbias"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("B,H,N,C,masked,gate,with_bias", [
    (3, 2, 7, 4, ((5, 7),), True, True),
    (2, 3, 9, 3, (), False, True),
    (4, 1, 6, 5, ((0, 2),), True, False),
])
def test_equals_attention_oracle_at_zero_query(B, H, N, C, masked, gate, with_bias):
    v, bias, keep, g, dout = _rand(B, H, N, C, masked, gate, 11)
    if not with_bias:
        bias = None
    rng = np.random.default_rng(5)
    q = np.zeros((B, N, H, C))
    k = rng.standard_normal((B, N, H, C))   # irrelevant once q = 0
    out_a, lse_a = oracle.fwd(q, k, v, bias, keep, g)
    out_p, lse_p = oracle.pwa_fwd(v, bias, keep, g)
    np.testing.assert_allclose(out_p, out_a, rtol=1e-12, atol=1e-12)
    for b in range(B):
        np.testing.assert_allclose(lse_p, lse_a[b], rtol=1e-12, atol=1e-12)
    dq_a, dk_a, dv_a, dg_a, db_a = oracle.bwd(q, k, v, bias if bias is not None else np.zeros((H, N, N)),
                                              keep, g, dout)
    dv_p, dg_p, db_p = oracle.pwa_bwd(v, bias, keep, g, dout)
    np.testing.assert_allclose(dv_p, dv_a, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(db_p, db_a, rtol=1e-10, atol=1e-12)
    if gate:
        np.testing.assert_allclose(dg_p, dg_a, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("masked,gate", [(((4, 6),), True), ((), False)])
def test_finite_differences(masked, gate):
    B, H, N, C = 2, 2, 6, 3
    v, bias, keep, g, dout = _rand(B, H, N, C, masked, gate, 3)
    loss = lambda v_, b_, g_: float((oracle.pwa_fwd(v_, b_, keep, g_)[0] * dout).sum())
    dv, dg, db = oracle.pwa_bwd(v, bias, keep, g, dout)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, arr, grad in (("v", v, dv), ("bias", bias, db)) + ((("g", g, dg),) if gate else ()):
        for _ in range(12):
            idx = tuple(int(rng.integers(s)) for s in arr.shape)
            a_p, a_m = arr.copy(), arr.copy()
            a_p[idx] += eps
            a_m[idx] -= eps
            args_p = {"v": v, "bias": bias, "g": g}
            args_m = dict(args_p)
            args_p[name], args_m[name] = a_p, a_m
            fd = (loss(args_p["v"], args_p["bias"], args_p["g"]) - loss(args_m["v"], args_m["bias"], args_m["g"])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * (1 + abs(fd)), (name, idx, fd, grad[idx])


def test_constant_v_gives_gated_v_and_zero_dbias():
    B, H, N, C = 2, 2, 5, 3
    _, bias, keep, g, dout = _rand(B, H, N, C, ((3, 4),), True, 7)
    v = np.broadcast_to(np.arange(1.0, C + 1.0), (B, N, H, C)).copy()
    out, _ = oracle.pwa_fwd(v, bias, keep, g)
    np.testing.assert_allclose(out, v / (1.0 + np.exp(-g)), rtol=1e-12, atol=1e-12)
    _, _, db = oracle.pwa_bwd(v, bias, keep, g, dout)
    np.testing.assert_allclose(db, 0.0, atol=1e-12)


def test_dbias_rows_sum_to_zero_and_masked_keys_get_nothing():
    B, H, N, C = 3, 2, 8, 4
    v, bias, keep, g, dout = _rand(B, H, N, C, ((2, 4),), True, 9)
    out, _ = oracle.pwa_fwd(v, bias, keep, g)
    v2 = v.copy()
    v2[:, 2:4] = 123.0          # values of masked keys cannot reach the output
    out2, _ = oracle.pwa_fwd(v2, bias, keep, g)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)
    _, _, db = oracle.pwa_bwd(v, bias, keep, g, dout)
    np.testing.assert_allclose(db.sum(-1), 0.0, atol=1e-12)
    np.testing.assert_allclose(db[:, :, 2:4], 0.0, atol=0)


def test_fully_masked_keys_give_zero():
    B, H, N, C = 2, 1, 4, 2
    v, bias, _, g, dout = _rand(B, H, N, C, (), True, 1)
    keep = np.zeros(N, dtype=np.uint8)
    out, lse = oracle.pwa_fwd(v, bias, keep, g)
    assert np.all(out == 0.0) and np.all(np.isneginf(lse))
    dv, dg, db = oracle.pwa_bwd(v, bias, keep, g, dout)
    assert np.all(dv == 0.0) and np.all(dg == 0.0) and np.all(db == 0.0)
