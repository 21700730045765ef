"""Python access to the fp64 CPU oracle (`pba_oracle.c`).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package's smoke check and by
the benchmark's CPU-baseline leg, never by the product path.  It shares no code with
the CUDA library.  Inputs are numpy float64 arrays (bf16 values widened exactly);
keep masks are uint8 (1 = key attended).

Functions follow the definition of pair-biased gated attention stated in
`pba_oracle.c` ("AlphaFold3 open-source implementation" page, Model Efficiency).
Every function here is pinned by tests/test_oracle.py (hand-worked example, finite
differences, closed-form invariants, an independent autograd cross-check).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pba_oracle.c")
_LIB = os.path.join(_HERE, "libpba_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        d = ctypes.POINTER(ctypes.c_double)
        u8 = ctypes.POINTER(ctypes.c_uint8)
        i, f, ll = ctypes.c_int, ctypes.c_double, ctypes.c_longlong
        lib.pba_oracle_fwd_slice.argtypes = [i, i, i, f, d, d, d, d, u8, d, d, d, d]
        lib.pba_oracle_bwd_slice.argtypes = [i, i, i, f, d, d, d, d, u8, d, d, d, d, d, d, d]
        lib.pba_oracle_fwd.argtypes = [i, i, i, i, i, f, d, d, d, d, u8, ll, d, d, d]
        lib.pba_oracle_bwd.argtypes = [i, i, i, i, i, f, d, d, d, d, u8, ll, d, d, d, d, d,
                                       d, d]
        lib.pba_oracle_dbias_row.argtypes = [i, i, i, i, i, f, i, i, d, d, d, d, u8, ll, d, d,
                                             d]
        lib.pba_oracle_pwa_fwd.argtypes = [i, i, i, i, d, d, u8, d, d, d]
        lib.pba_oracle_pwa_bwd.argtypes = [i, i, i, i, d, d, u8, d, d, d, d, d]
        lib.pba_oracle_pair_bias_fwd.argtypes = [i, i, i, i, f, d, d, d, d, d]
        lib.pba_oracle_pair_bias_bwd.argtypes = [i, i, i, i, f, d, d, d, d, d, d, d, d, d]
        lib.pba_oracle_threads.argtypes = []
        lib.pba_oracle_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def threads() -> int:
    """OpenMP threads available to the oracle's parallel loops."""
    return int(_load().pba_oracle_threads())


def _d(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _u8(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.dtype == np.uint8 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _keep(keep, B):
    """keep: None, [Nk] (shared by all b) or [B, Nk]; returns (array, row stride)."""
    if keep is None:
        return None, 0
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    if keep.ndim == 1:
        return keep, 0
    assert keep.shape[0] == B
    return keep, keep.shape[1]


def default_scale(c: int) -> float:
    """1/sqrt(c) with the true head dimension."""
    return 1.0 / math.sqrt(c)


def fwd(q, k, v, bias=None, keep=None, g=None, scale=None):
    """out [B,Nq,H,C] and lse [B,H,Nq] for full tensors in the library layout."""
    lib = _load()
    q, k, v, bias, g = map(_f64, (q, k, v, bias, g))
    B, Nq, H, C = q.shape
    Nk = k.shape[1]
    scale = default_scale(C) if scale is None else float(scale)
    keep, ksb = _keep(keep, B)
    out = np.empty((B, Nq, H, C))
    lse = np.empty((B, H, Nq))
    lib.pba_oracle_fwd(B, H, Nq, Nk, C, scale, _d(q), _d(k), _d(v), _d(bias), _u8(keep), ksb,
                       _d(g), _d(out), _d(lse))
    return out, lse


def bwd(q, k, v, bias, keep, g, dout, scale=None):
    """dq, dk, dv, dg (None without gate), dbias [H,Nq,Nk]."""
    lib = _load()
    q, k, v, bias, g, dout = map(_f64, (q, k, v, bias, g, dout))
    B, Nq, H, C = q.shape
    Nk = k.shape[1]
    scale = default_scale(C) if scale is None else float(scale)
    keep, ksb = _keep(keep, B)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    dg = np.empty_like(q) if g is not None else None
    dbias = np.empty((H, Nq, Nk))
    lib.pba_oracle_bwd(B, H, Nq, Nk, C, scale, _d(q), _d(k), _d(v), _d(bias), _u8(keep), ksb,
                       _d(g), _d(dout), _d(dq), _d(dk), _d(dv), _d(dg), _d(dbias))
    return dq, dk, dv, dg, dbias


def fwd_slice(q, k, v, bias=None, keep=None, g=None, scale=None, want_P=False):
    """One (b, h) problem: q [Nq,C], k/v [Nk,C], bias [Nq,Nk], keep [Nk], g [Nq,C]."""
    lib = _load()
    q, k, v, bias, g = map(_f64, (q, k, v, bias, g))
    Nq, C = q.shape
    Nk = k.shape[0]
    scale = default_scale(C) if scale is None else float(scale)
    keep = None if keep is None else np.ascontiguousarray(keep, dtype=np.uint8)
    out = np.empty((Nq, C))
    lse = np.empty(Nq)
    P = np.empty((Nq, Nk)) if want_P else None
    lib.pba_oracle_fwd_slice(Nq, Nk, C, scale, _d(q), _d(k), _d(v), _d(bias), _u8(keep), _d(g),
                             _d(out), _d(lse), _d(P))
    return (out, lse, P) if want_P else (out, lse)


def bwd_slice(q, k, v, bias, keep, g, dout, scale=None):
    """One (b, h) problem: dq, dk, dv, dg (None without gate), dS [Nq, Nk]."""
    lib = _load()
    q, k, v, bias, g, dout = map(_f64, (q, k, v, bias, g, dout))
    Nq, C = q.shape
    Nk = k.shape[0]
    scale = default_scale(C) if scale is None else float(scale)
    keep = None if keep is None else np.ascontiguousarray(keep, dtype=np.uint8)
    dq = np.empty((Nq, C))
    dk = np.empty((Nk, C))
    dv = np.empty((Nk, C))
    dg = np.empty((Nq, C)) if g is not None else None
    ds = np.empty((Nq, Nk))
    lib.pba_oracle_bwd_slice(Nq, Nk, C, scale, _d(q), _d(k), _d(v), _d(bias), _u8(keep), _d(g),
                             _d(dout), _d(dq), _d(dk), _d(dv), _d(dg), _d(ds))
    return dq, dk, dv, dg, ds


def dbias_row(q, k, v, bias, keep, g, dout, h, i, scale=None):
    """dbias[h, i, :] (sum over all b) for full tensors in the library layout."""
    lib = _load()
    q, k, v, bias, g, dout = map(_f64, (q, k, v, bias, g, dout))
    B, Nq, H, C = q.shape
    Nk = k.shape[1]
    scale = default_scale(C) if scale is None else float(scale)
    keep, ksb = _keep(keep, B)
    row = np.empty(Nk)
    lib.pba_oracle_dbias_row(B, H, Nq, Nk, C, scale, int(h), int(i), _d(q), _d(k), _d(v),
                             _d(bias), _u8(keep), ksb, _d(g), _d(dout), _d(row))
    return row


def pwa_fwd(v, bias=None, keep=None, g=None):
    """MSA pair-weighted averaging: out [B,N,H,C] and lse_w [H,N] (weights softmax_j(bias
    + mask), shared by every row b; keep is one [N] row or None)."""
    lib = _load()
    v, bias, g = map(_f64, (v, bias, g))
    B, N, H, C = v.shape
    keep = None if keep is None else np.ascontiguousarray(keep, dtype=np.uint8).reshape(N)
    out = np.empty((B, N, H, C))
    lse = np.empty((H, N))
    lib.pba_oracle_pwa_fwd(B, H, N, C, _d(v), _d(bias), _u8(keep), _d(g), _d(out), _d(lse))
    return out, lse


def pwa_bwd(v, bias, keep, g, dout):
    """dv [B,N,H,C], dg (None without gate), dbias [H,N,N] of MSA pair-weighted averaging."""
    lib = _load()
    v, bias, g, dout = map(_f64, (v, bias, g, dout))
    B, N, H, C = v.shape
    keep = None if keep is None else np.ascontiguousarray(keep, dtype=np.uint8).reshape(N)
    dv = np.empty_like(v)
    dg = np.empty_like(v) if g is not None else None
    dbias = np.empty((H, N, N))
    lib.pba_oracle_pwa_bwd(B, H, N, C, _d(v), _d(bias), _u8(keep), _d(g), _d(dout), _d(dv), _d(dg),
                           _d(dbias))
    return dv, dg, dbias


def pair_bias_fwd(z, gamma, beta, w, eps=1e-5):
    """Pair-bias projection: bias [H,Ni,Nj] = LayerNorm(z[i,j,:]; gamma, beta, eps) . w[:,h],
    z [Ni,Nj,Cz], w [Cz,H]."""
    lib = _load()
    z, gamma, beta, w = map(_f64, (z, gamma, beta, w))
    Ni, Nj, Cz = z.shape
    H = w.shape[1]
    bias = np.zeros((H, Ni, Nj))
    lib.pba_oracle_pair_bias_fwd(Ni, Nj, Cz, H, float(eps), _d(z), _d(gamma), _d(beta), _d(w), _d(bias))
    return bias


def pair_bias_bwd(z, gamma, beta, w, dbias, eps=1e-5):
    """dz [Ni,Nj,Cz], dw [Cz,H], dgamma [Cz], dbeta [Cz] of the pair-bias projection."""
    lib = _load()
    z, gamma, beta, w, dbias = map(_f64, (z, gamma, beta, w, dbias))
    Ni, Nj, Cz = z.shape
    H = w.shape[1]
    dz = np.zeros_like(z)
    dw = np.zeros((Cz, H))
    dgamma = np.zeros(Cz)
    dbeta = np.zeros(Cz)
    lib.pba_oracle_pair_bias_bwd(Ni, Nj, Cz, H, float(eps), _d(z), _d(gamma), _d(beta), _d(w), _d(dbias),
                                 _d(dz), _d(dw), _d(dgamma), _d(dbeta))
    return dz, dw, dgamma, dbeta
