"""Helpers shared by the GPU parity tests: seeded inputs on the device, oracle slices,
and the tolerances the comparisons use.

Tolerances (stated for bf16 inputs and outputs): out max |err| <= 2e-2 and mean |err| <=
2e-3; lse max |err| <= 1e-3; dq, dk, dv, dgate, dbias relative L2 error <= 1e-2.
"""
from __future__ import annotations

import numpy as np

import oracle
import pba_inputs as pi

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def to_dev(inp: dict, device="cuda"):
    """bf16 bit arrays -> torch bf16 CUDA tensors; keep mask -> uint8 CUDA tensor."""
    import torch
    out = {}
    for k, a in inp.items():
        if k == "keep":
            out[k] = torch.from_numpy(np.ascontiguousarray(a)).to(device)
        else:
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
            out[k] = t.to(device)
    return out


def bf16_to_f64_tensor(t) -> np.ndarray:
    import torch
    return t.detach().float().cpu().numpy().astype(np.float64)


def f64(inp: dict, name: str):
    a = inp.get(name)
    return None if a is None else pi.bf16_bits_to_f64(a)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((got - ref).ravel()) / max(den, 1e-30))


def assert_out_close(got, ref, what="out"):
    err = np.abs(got - ref)
    assert err.max() <= OUT_MAX_ABS, "%s max abs err %.3g" % (what, err.max())
    assert err.mean() <= OUT_MEAN_ABS, "%s mean abs err %.3g" % (what, err.mean())


def assert_lse_close(got, ref):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), "lse finiteness differs"
    assert np.all(got[~fin] == ref[~fin])
    if fin.any():
        err = np.abs(got[fin] - ref[fin]).max()
        assert err <= LSE_MAX_ABS, "lse max abs err %.3g" % err


def assert_grad_close(got, ref, what):
    r = rel_l2(got, ref)
    assert r <= GRAD_REL_L2, "%s relative L2 err %.3g" % (what, r)
