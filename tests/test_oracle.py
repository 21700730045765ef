"""Pins for the fp64 CPU oracle: it is checked against things other than itself.

- a hand-worked 2-token example (tests/golden/two_token.json);
- central finite differences of the oracle's own forward for every gradient;
- an independent library routine (torch's scaled_dot_product_attention in fp64 with a
  float attention mask broadcast over the batch, autograd for every gradient, the bias
  gradient arriving through the broadcast as a sum);
- closed-form invariants of softmax attention.

The operator is pair-biased gated attention as described on the "AlphaFold3 open-source
implementation" page, Model Efficiency section (bias added after the key-query dot
product; bias gradient = gradient of the scaled logits; broadcast in the forward pass
becomes a reduction in the backward pass; replicas folded into the batch axis).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _val(x):
    if isinstance(x, str):
        return {"ln2": math.log(2.0), "ln4": math.log(4.0), "ln3-2": math.log(3.0) - 2.0}[x]
    if isinstance(x, list):
        return [_val(y) for y in x]
    return float(x)


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ------------------------------------------------------------------------------------
# hand-worked example
# ------------------------------------------------------------------------------------

def test_two_token_golden():
    with open(os.path.join(GOLDEN, "two_token.json")) as f:
        gold = json.load(f)
    inp, exp = gold["inputs"], gold["expected"]
    sh = (1, 2, 1, 1)
    q = np.array(_val(inp["q"])).reshape(sh)
    k = np.array(_val(inp["k"])).reshape(sh)
    v = np.array(_val(inp["v"])).reshape(sh)
    g = np.array(_val(inp["g"])).reshape(sh)
    dout = np.array(_val(inp["dout"])).reshape(sh)
    bias = np.array(_val(inp["bias"])).reshape(1, 2, 2)
    out, lse = oracle.fwd(q, k, v, bias, None, g, scale=inp["scale"])
    np.testing.assert_allclose(out.ravel(), _val(exp["out"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse.ravel(), _val(exp["lse"]), rtol=0, atol=1e-14)
    dq, dk, dv, dg, db = oracle.bwd(q, k, v, bias, None, g, dout, scale=inp["scale"])
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv), ("dg", dg), ("dbias", db)):
        np.testing.assert_allclose(got.ravel(), np.ravel(_val(exp[name])), rtol=0, atol=1e-14,
                                   err_msg=name)


# ------------------------------------------------------------------------------------
# finite differences of the forward pass
# ------------------------------------------------------------------------------------

def _loss(q, k, v, bias, keep, g, dout, scale):
    out, _ = oracle.fwd(q, k, v, bias, keep, g, scale=scale)
    return float(np.sum(out * dout))


@pytest.mark.parametrize("B,H,Nq,Nk,C,masked,gate", [
    (2, 2, 3, 3, 2, (), True),
    (2, 2, 5, 5, 3, (1, 4), True),
    (2, 1, 3, 5, 3, (0,), False),
    (3, 2, 4, 2, 2, (), True),
])
def test_finite_differences(B, H, Nq, Nk, C, masked, gate):
    rng = np.random.default_rng(1234 + B * 100 + Nq * 10 + Nk)
    q, k, v = _rand(rng, B, Nq, H, C), _rand(rng, B, Nk, H, C), _rand(rng, B, Nk, H, C)
    bias = _rand(rng, H, Nq, Nk)
    g = _rand(rng, B, Nq, H, C) if gate else None
    dout = _rand(rng, B, Nq, H, C)
    keep = np.ones(Nk, np.uint8)
    for j in masked:
        keep[j] = 0
    scale = 0.7
    dq, dk, dv, dg, db = oracle.bwd(q, k, v, bias, keep, g, dout, scale=scale)
    grads = {"q": dq, "k": dk, "v": dv, "bias": db}
    if gate:
        grads["g"] = dg
    eps = 1e-6
    for name, grad in grads.items():
        arrs = {"q": q, "k": k, "v": v, "bias": bias, "g": g}
        x = arrs[name]
        num = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            x0 = x[idx]
            x[idx] = x0 + eps
            lp = _loss(q, k, v, bias, keep, g, dout, scale)
            x[idx] = x0 - eps
            lm = _loss(q, k, v, bias, keep, g, dout, scale)
            x[idx] = x0
            num[idx] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(num - grad)) / max(1.0, np.max(np.abs(grad)))
        assert err < 1e-7, (name, err)


# ------------------------------------------------------------------------------------
# independent library routine: torch SDPA in fp64 with autograd
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,Nq,Nk,C,masked,gate,scale", [
    (3, 2, 7, 7, 4, (), False, None),
    (4, 3, 9, 9, 8, (6, 7, 8), True, None),
    (2, 2, 5, 11, 6, (0, 3), True, 0.3),
    (5, 1, 16, 16, 3, (15,), True, None),
])
def test_against_torch_sdpa_autograd(B, H, Nq, Nk, C, masked, gate, scale):
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    rng = np.random.default_rng(99 + B + Nq + Nk)
    q, k, v = _rand(rng, B, Nq, H, C), _rand(rng, B, Nk, H, C), _rand(rng, B, Nk, H, C)
    bias = _rand(rng, H, Nq, Nk)
    g = _rand(rng, B, Nq, H, C) if gate else None
    dout = _rand(rng, B, Nq, H, C)
    keep = np.ones(Nk, np.uint8)
    for j in masked:
        keep[j] = 0
    out, lse = oracle.fwd(q, k, v, bias, keep, g, scale=scale)
    dq, dk, dv, dg, db = oracle.bwd(q, k, v, bias, keep, g, dout, scale=scale)

    T = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    tq, tk, tv, tb = T(q), T(k), T(v), T(bias)
    # library layout [B, N, H, C] -> SDPA layout [B, H, N, C]
    addmask = torch.tensor(np.where(keep > 0, 0.0, -np.inf))
    attn_mask = tb.unsqueeze(0).expand(B, H, Nq, Nk) + addmask
    o = F.scaled_dot_product_attention(tq.transpose(1, 2), tk.transpose(1, 2),
                                       tv.transpose(1, 2), attn_mask=attn_mask,
                                       scale=scale).transpose(1, 2)
    if gate:
        tg = T(g)
        o = torch.sigmoid(tg) * o
    o.backward(torch.tensor(dout))
    np.testing.assert_allclose(out, o.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(db, tb.grad.numpy(), rtol=1e-10, atol=1e-11)
    if gate:
        np.testing.assert_allclose(dg, tg.grad.numpy(), rtol=1e-10, atol=1e-11)
    # logsumexp from the library's own reduction
    sc = (1.0 / math.sqrt(C)) if scale is None else scale
    logits = torch.einsum("bihc,bjhc->bhij", torch.tensor(q), torch.tensor(k)) * sc
    logits = logits + torch.tensor(bias).unsqueeze(0) + addmask
    np.testing.assert_allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=1e-12,
                               atol=1e-12)


# ------------------------------------------------------------------------------------
# closed-form invariants
# ------------------------------------------------------------------------------------

def _case(seed=7, B=3, H=2, Nq=6, Nk=6, C=4, masked=(4,), gate=True):
    rng = np.random.default_rng(seed)
    d = dict(q=_rand(rng, B, Nq, H, C), k=_rand(rng, B, Nk, H, C), v=_rand(rng, B, Nk, H, C),
             bias=_rand(rng, H, Nq, Nk), g=_rand(rng, B, Nq, H, C) if gate else None,
             dout=_rand(rng, B, Nq, H, C))
    keep = np.ones(Nk, np.uint8)
    for j in masked:
        keep[j] = 0
    d["keep"] = keep
    return d


def test_softmax_rows_sum_to_one():
    d = _case()
    for b in range(3):
        for h in range(2):
            _, _, P = oracle.fwd_slice(d["q"][b, :, h], d["k"][b, :, h], d["v"][b, :, h],
                                       d["bias"][h], d["keep"], None, want_P=True)
            np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
            assert np.all(P[:, 4] == 0.0)


def test_constant_v_gives_gated_v_and_zero_grads():
    d = _case()
    d["v"][:] = 1.7
    out, _ = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    sig = 1.0 / (1.0 + np.exp(-d["g"]))
    np.testing.assert_allclose(out, sig * 1.7, rtol=1e-14, atol=1e-14)
    dq, dk, dv, dg, db = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"],
                                    d["dout"])
    assert np.max(np.abs(dq)) < 1e-13 and np.max(np.abs(dk)) < 1e-13
    assert np.max(np.abs(db)) < 1e-13


def test_masked_key_gets_nothing():
    d = _case()
    dq, dk, dv, dg, db = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"],
                                    d["dout"])
    assert np.all(dk[:, 4] == 0.0) and np.all(dv[:, 4] == 0.0) and np.all(db[:, :, 4] == 0.0)
    # the masked key's values do not reach the output at all
    d2 = {k: (None if v is None else v.copy()) for k, v in d.items()}
    d2["k"][:, 4] += 10.0
    d2["v"][:, 4] -= 5.0
    o1, l1 = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    o2, l2 = oracle.fwd(d2["q"], d2["k"], d2["v"], d2["bias"], d2["keep"], d2["g"])
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_dbias_rows_sum_to_zero():
    d = _case(B=4, Nq=7, Nk=9, masked=(2, 8))
    *_, db = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"], d["dout"])
    assert np.max(np.abs(db.sum(axis=-1))) < 1e-13
    assert np.max(np.abs(db)) > 1e-3


def test_row_constant_bias_shift_invariance():
    d = _case()
    shift = np.random.default_rng(3).standard_normal((2, 6, 1)) * 5
    o1, l1 = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    o2, l2 = oracle.fwd(d["q"], d["k"], d["v"], d["bias"] + shift, d["keep"], d["g"])
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2 - l1, np.broadcast_to(shift[None, :, :, 0], l1.shape),
                               rtol=1e-12, atol=1e-12)


def test_duplicated_broadcast_rows_double_dbias():
    d = _case(B=2)
    rep = lambda a: None if a is None else np.concatenate([a, a], axis=0)
    o1, _ = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    o2, _ = oracle.fwd(rep(d["q"]), rep(d["k"]), rep(d["v"]), d["bias"], d["keep"], rep(d["g"]))
    np.testing.assert_allclose(o2[:2], o1, rtol=0, atol=0)
    np.testing.assert_allclose(o2[2:], o1, rtol=0, atol=0)
    *_, db1 = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"], d["dout"])
    *_, db2 = oracle.bwd(rep(d["q"]), rep(d["k"]), rep(d["v"]), d["bias"], d["keep"],
                         rep(d["g"]), rep(d["dout"]))
    np.testing.assert_allclose(db2, 2 * db1, rtol=1e-13, atol=1e-15)


def test_key_permutation_invariance():
    d = _case(Nk=8, masked=(1, 6))
    perm = np.random.default_rng(5).permutation(8)
    o1, l1 = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    o2, l2 = oracle.fwd(d["q"], d["k"][:, perm], d["v"][:, perm], d["bias"][:, :, perm],
                        d["keep"][perm], d["g"])
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-14)
    *_, db1 = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"], d["dout"])
    *_, db2 = oracle.bwd(d["q"], d["k"][:, perm], d["v"][:, perm], d["bias"][:, :, perm],
                         d["keep"][perm], d["g"], d["dout"])
    np.testing.assert_allclose(db1[:, :, perm], db2, rtol=1e-12, atol=1e-14)


def test_fully_masked_row_is_zero():
    d = _case(masked=tuple(range(6)))
    out, lse = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    assert np.all(out == 0.0) and np.all(np.isneginf(lse))
    dq, dk, dv, dg, db = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"],
                                    d["dout"])
    for a in (dq, dk, dv, dg, db):
        assert np.all(a == 0.0)


def test_per_row_mask_and_shared_mask_agree():
    d = _case(B=3, masked=(1, 5))
    keep_b = np.stack([d["keep"]] * 3)
    o1, l1 = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    o2, l2 = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], keep_b, d["g"])
    np.testing.assert_array_equal(o1, o2)
    # a per-row mask that differs by row equals the row-by-row problems
    keep_b[1, 2] = 0
    o3, _ = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], keep_b, d["g"])
    k2 = d["keep"].copy()
    k2[2] = 0
    o4, _ = oracle.fwd(d["q"][1:2], d["k"][1:2], d["v"][1:2], d["bias"], k2, d["g"][1:2])
    np.testing.assert_array_equal(o3[1:2], o4)
    np.testing.assert_array_equal(o3[0], o1[0])


def test_slices_and_dbias_row_match_full():
    d = _case(B=3, H=2, Nq=5, Nk=7, C=3, masked=(3,))
    out, lse = oracle.fwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"])
    dq, dk, dv, dg, db = oracle.bwd(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"],
                                    d["dout"])
    for b in range(3):
        for h in range(2):
            o_s, l_s = oracle.fwd_slice(d["q"][b, :, h], d["k"][b, :, h], d["v"][b, :, h],
                                        d["bias"][h], d["keep"], d["g"][b, :, h])
            np.testing.assert_array_equal(o_s, out[b, :, h])
            np.testing.assert_array_equal(l_s, lse[b, h])
    for h in range(2):
        for i in range(5):
            row = oracle.dbias_row(d["q"], d["k"], d["v"], d["bias"], d["keep"], d["g"],
                                   d["dout"], h, i)
            np.testing.assert_allclose(row, db[h, i], rtol=1e-13, atol=1e-15)


def test_no_bias_no_gate_is_plain_attention():
    """Zero bias, no mask, no gate: textbook attention, checked against numpy's own
    matrix product and exp on an explicit two-row case."""
    q = np.array([[[[1.0, 0.0]]], [[[0.0, 2.0]]]]).reshape(1, 2, 1, 2)
    k = np.array([[1.0, 1.0], [0.0, -1.0], [2.0, 0.0]]).reshape(1, 3, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]]).reshape(1, 3, 1, 2)
    out, lse = oracle.fwd(q, k, v, None, None, None, scale=1.0)
    S = q[0, :, 0] @ k[0, :, 0].T
    P = np.exp(S) / np.exp(S).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(out[0, :, 0], P @ v[0, :, 0], rtol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.log(np.exp(S).sum(axis=1)), rtol=1e-14)
