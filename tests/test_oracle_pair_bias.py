"""Pins of the oracle for the pair-bias projection (oracle.pair_bias_fwd / pair_bias_bwd):
a hand-worked example, torch's own LayerNorm and matmul in fp64 with autograd (an
independent library routine), central finite differences, and closed-form invariants."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pair_bias_two_positions.json")


def _inputs(Ni, Nj, Cz, H, seed=0, scale=1.0, shift=0.0):
    rng = np.random.default_rng(seed)
    z = rng.normal(shift, scale, (Ni, Nj, Cz))
    gamma = rng.normal(1.0, 0.3, Cz)
    beta = rng.normal(0.0, 0.3, Cz)
    w = rng.normal(0.0, 1.0 / math.sqrt(Cz), (Cz, H))
    dbias = rng.normal(0.0, 1.0, (H, Ni, Nj))
    return z, gamma, beta, w, dbias


def _ev(x):
    if isinstance(x, list):
        return [_ev(v) for v in x]
    if isinstance(x, str):
        return float(eval(x, {"__builtins__": {}}, {"sqrt2": math.sqrt(2.0)}))
    return float(x)


def test_two_positions_golden():
    g = json.load(open(GOLDEN))
    inp = g["inputs"]
    z, gamma, beta, w = (np.array(inp[k], dtype=np.float64) for k in ("z", "gamma", "beta", "w"))
    dbias = np.array(inp["dbias"], dtype=np.float64)
    bias = oracle.pair_bias_fwd(z, gamma, beta, w, eps=inp["eps"])
    np.testing.assert_allclose(bias, np.array(_ev(g["expected"]["bias"])), atol=1e-12)
    dz, dw, dgamma, dbeta = oracle.pair_bias_bwd(z, gamma, beta, w, dbias, eps=inp["eps"])
    for name, got in (("dz", dz), ("dw", dw), ("dgamma", dgamma), ("dbeta", dbeta)):
        np.testing.assert_allclose(got, np.array(_ev(g["expected"][name])), atol=1e-12, err_msg=name)


@pytest.mark.parametrize("Ni,Nj,Cz,H,eps", [(3, 5, 8, 2, 1e-5), (4, 7, 16, 4, 1e-5), (2, 3, 32, 1, 0.1)])
def test_matches_torch_layer_norm_and_autograd(Ni, Nj, Cz, H, eps):
    torch = pytest.importorskip("torch")
    z, gamma, beta, w, dbias = _inputs(Ni, Nj, Cz, H, seed=Ni * 7 + Cz)
    tz, tg, tb, tw = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (z, gamma, beta, w))
    y = torch.nn.functional.layer_norm(tz, (Cz,), tg, tb, eps)
    tbias = torch.einsum("ijc,ch->hij", y, tw)
    np.testing.assert_allclose(oracle.pair_bias_fwd(z, gamma, beta, w, eps), tbias.detach().numpy(), atol=1e-12)
    tbias.backward(torch.tensor(dbias, dtype=torch.float64))
    dz, dw, dgamma, dbeta = oracle.pair_bias_bwd(z, gamma, beta, w, dbias, eps)
    np.testing.assert_allclose(dz, tz.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dw, tw.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dgamma, tg.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dbeta, tb.grad.numpy(), atol=1e-11)


def test_finite_differences():
    z, gamma, beta, w, dbias = _inputs(2, 3, 6, 3, seed=5)
    eps, h = 1e-3, 1e-6

    def loss(z_, g_, b_, w_):
        return float((oracle.pair_bias_fwd(z_, g_, b_, w_, eps) * dbias).sum())

    dz, dw, dgamma, dbeta = oracle.pair_bias_bwd(z, gamma, beta, w, dbias, eps)
    for arr, grad, idx in ((z, dz, 0), (gamma, dgamma, 1), (beta, dbeta, 2), (w, dw, 3)):
        fd = np.zeros_like(arr)
        for k in range(arr.size):
            args = [z, gamma, beta, w]
            p, m = arr.copy(), arr.copy()
            p.flat[k] += h
            m.flat[k] -= h
            args[idx] = p
            lp = loss(*args)
            args[idx] = m
            lm = loss(*args)
            fd.flat[k] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, fd, atol=1e-7, rtol=1e-6)


def test_constant_rows_give_the_beta_projection():
    # a constant z row has no deviation: xh = 0, y = beta, bias = beta . w
    _, gamma, beta, w, _ = _inputs(1, 1, 16, 4, seed=2)
    z = np.full((3, 4, 16), 2.5)
    z[1] = -7.0
    bias = oracle.pair_bias_fwd(z, gamma, beta, w)
    want = (beta @ w)[:, None, None] * np.ones((1, 3, 4))
    np.testing.assert_allclose(bias, want, atol=1e-12)


def test_shift_and_scale_invariance():
    # with eps = 0, LayerNorm removes any per-row affine map a z + b (a > 0)
    z, gamma, beta, w, _ = _inputs(3, 4, 12, 3, seed=3)
    a = np.linspace(0.5, 4.0, 12).reshape(3, 4, 1)
    b = np.linspace(-3.0, 3.0, 12).reshape(3, 4, 1)
    np.testing.assert_allclose(oracle.pair_bias_fwd(a * z + b, gamma, beta, w, 0.0),
                               oracle.pair_bias_fwd(z, gamma, beta, w, 0.0), atol=1e-12)


def test_identity_projection_gives_normalised_rows():
    # gamma = 1, beta = 0, w = I: bias[:, i, j] is the normalised row (zero mean, unit
    # variance with eps = 0)
    z, _, _, _, _ = _inputs(3, 5, 8, 8, seed=4, scale=3.0, shift=2.0)
    bias = oracle.pair_bias_fwd(z, np.ones(8), np.zeros(8), np.eye(8), 0.0)
    np.testing.assert_allclose(bias.mean(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose((bias ** 2).mean(axis=0), 1.0, atol=1e-12)


def test_dz_is_orthogonal_to_ones_and_to_the_normalised_row():
    # LayerNorm's output does not change along z + t 1 (any eps) nor along z + t (z - mu)
    # (eps = 0), so the input gradient is orthogonal to both directions
    z, gamma, beta, w, dbias = _inputs(4, 6, 16, 4, seed=6)
    eps = 0.0
    dz, _, _, _ = oracle.pair_bias_bwd(z, gamma, beta, w, dbias, eps)
    mu = z.mean(axis=2, keepdims=True)
    xh = (z - mu) / np.sqrt(((z - mu) ** 2).mean(axis=2, keepdims=True) + eps)
    np.testing.assert_allclose(dz.sum(axis=2), 0.0, atol=1e-11)
    np.testing.assert_allclose((dz * xh).sum(axis=2), 0.0, atol=1e-10)
