"""Python binding of libpba (pair-biased gated attention for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
`libpba.so`, reached through its C ABI (`include/pba.h`).  PyTorch provides device memory
and streams.  There is no fallback: if the library is missing this import fails.

Tensor layouts (bf16 unless noted): q, gate, out, dout [B, Nq, H, C]; k, v [B, Nk, H, C];
bias [H, Nq, Nk]; key_mask uint8/bool [Nk] (shared by all B) or [B, Nk] (1 = attended);
lse fp32 [B, H, Nq]; dbias fp32 [H, Nq, Nk].
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpba.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libpba.so is not built; run `python pair_biased_attention_gated_b200/build.py` "
        "(there is no non-CUDA implementation of this package)")

lib = ctypes.CDLL(LIB_PATH)

PBA_OK = 0
STATUS = {0: "PBA_OK", 1: "PBA_ERR_INVALID_ARG", 2: "PBA_ERR_UNSUPPORTED", 3: "PBA_ERR_CUDA",
          4: "PBA_ERR_TIMEOUT", 5: "PBA_ERR_WORKSPACE"}


class PbaDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("Nq", ctypes.c_int32),
                ("Nk", ctypes.c_int32), ("C", ctypes.c_int32), ("scale", ctypes.c_float),
                ("sq", ctypes.c_int64 * 3), ("sk", ctypes.c_int64 * 3),
                ("sv", ctypes.c_int64 * 3), ("sg", ctypes.c_int64 * 3),
                ("so", ctypes.c_int64 * 3), ("sbias", ctypes.c_int64 * 2),
                ("smask_b", ctypes.c_int64)]


_vp = ctypes.c_void_p
lib.pba_dims_dense.argtypes = [ctypes.POINTER(PbaDims)] + [ctypes.c_int32] * 5 + [ctypes.c_float]
lib.pba_dims_dense.restype = None
lib.pba_fwd.argtypes = [_vp] * 8 + [ctypes.POINTER(PbaDims), _vp]
lib.pba_fwd.restype = ctypes.c_int
lib.pba_bwd_workspace_size.argtypes = [ctypes.POINTER(PbaDims)]
lib.pba_bwd_workspace_size.restype = ctypes.c_size_t
lib.pba_bwd.argtypes = [_vp] * 14 + [_vp, ctypes.c_size_t, ctypes.POINTER(PbaDims), _vp]
lib.pba_bwd.restype = ctypes.c_int
lib.pba_bwd_noalloc.argtypes = [_vp] * 14 + [ctypes.POINTER(PbaDims), _vp]
lib.pba_fwd_local.argtypes = [_vp] * 8 + [ctypes.POINTER(PbaDims), ctypes.c_int, _vp]
lib.pba_fwd_local.restype = ctypes.c_int
lib.pba_bwd_local.argtypes = [_vp] * 14 + [_vp, ctypes.c_size_t, ctypes.POINTER(PbaDims), ctypes.c_int, _vp]
lib.pba_bwd_local.restype = ctypes.c_int
lib.pba_bwd_noalloc.restype = ctypes.c_int
lib.pba_pwa_fwd_workspace_size.argtypes = [ctypes.POINTER(PbaDims)]
lib.pba_pwa_fwd_workspace_size.restype = ctypes.c_size_t
lib.pba_pwa_bwd_workspace_size.argtypes = [ctypes.POINTER(PbaDims)]
lib.pba_pwa_bwd_workspace_size.restype = ctypes.c_size_t
lib.pba_pwa_fwd.argtypes = [_vp] * 7 + [ctypes.c_size_t, ctypes.POINTER(PbaDims), _vp]
lib.pba_pwa_fwd.restype = ctypes.c_int
lib.pba_pwa_bwd.argtypes = [_vp] * 10 + [ctypes.c_size_t, ctypes.POINTER(PbaDims), _vp]
lib.pba_pwa_bwd.restype = ctypes.c_int


class PbaPairBiasDims(ctypes.Structure):
    _fields_ = [("Ni", ctypes.c_int32), ("Nj", ctypes.c_int32), ("Cz", ctypes.c_int32),
                ("H", ctypes.c_int32), ("eps", ctypes.c_float), ("sz", ctypes.c_int64 * 2),
                ("sbias", ctypes.c_int64 * 2), ("sdbias", ctypes.c_int64 * 2)]


lib.pba_pair_bias_fwd.argtypes = [_vp] * 5 + [ctypes.POINTER(PbaPairBiasDims), _vp]
lib.pba_pair_bias_fwd.restype = ctypes.c_int
lib.pba_pair_bias_bwd_workspace_size.argtypes = [ctypes.POINTER(PbaPairBiasDims)]
lib.pba_pair_bias_bwd_workspace_size.restype = ctypes.c_size_t
lib.pba_pair_bias_bwd.argtypes = [_vp] * 10 + [ctypes.c_size_t, ctypes.POINTER(PbaPairBiasDims), _vp]
lib.pba_pair_bias_bwd.restype = ctypes.c_int
lib.pba_dbias_sum.argtypes = [_vp, ctypes.c_int, ctypes.c_int64, _vp, _vp]
lib.pba_dbias_sum.restype = ctypes.c_int
lib.pba_device_status.argtypes = [_vp]
lib.pba_device_status.restype = ctypes.c_int
lib.pba_status_string.argtypes = [ctypes.c_int]
lib.pba_status_string.restype = ctypes.c_char_p
lib.pba_last_error.argtypes = []
lib.pba_last_error.restype = ctypes.c_char_p
lib.pba_debug_skip_load.argtypes = [ctypes.c_int]
lib.pba_debug_skip_load.restype = None
lib.pba_version.argtypes = []
lib.pba_version.restype = ctypes.c_int


class PbaKernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double)]


lib.pba_profile_enable.argtypes = [ctypes.c_int]
lib.pba_profile_enable.restype = ctypes.c_int
lib.pba_profile_read.argtypes = [ctypes.POINTER(PbaKernelStat), ctypes.c_int]
lib.pba_profile_read.restype = ctypes.c_int


class PbaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__("%s: %s" % (STATUS.get(status, status), detail))
        self.status = status


def _check(status: int) -> None:
    if status != PBA_OK:
        raise PbaError(status, lib.pba_last_error().decode())


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _s3(t):
    st = t.stride()
    if st[3] != 1:
        raise ValueError("the channel (last) dimension must have stride 1")
    return (ctypes.c_int64 * 3)(st[0], st[1], st[2])


def make_dims(q, k, v, gate=None, out=None, bias=None, key_mask=None, scale: float = 0.0,
              dout=None) -> PbaDims:
    """pba_dims from tensors: q/gate/out [B,Nq,H,C], k/v [B,Nk,H,C], bias [H,Nq,Nk]."""
    B, Nq, H, C = q.shape
    Nk = k.shape[1]
    d = PbaDims()
    d.B, d.H, d.Nq, d.Nk, d.C = B, H, Nq, Nk, C
    d.scale = float(scale or 0.0)
    d.sq, d.sk, d.sv = _s3(q), _s3(k), _s3(v)
    d.sg = _s3(gate) if gate is not None else _s3(q)
    ref_o = out if out is not None else dout
    d.so = _s3(ref_o) if ref_o is not None else _s3(q)
    if bias is not None:
        if bias.stride(2) != 1:
            raise ValueError("bias key stride must be 1")
        d.sbias = (ctypes.c_int64 * 2)(bias.stride(0), bias.stride(1))
    if key_mask is not None:
        if key_mask.stride(-1) != 1:
            raise ValueError("key_mask key stride must be 1")
        d.smask_b = 0 if key_mask.dim() == 1 else key_mask.stride(0)
    return d


def dims_dense(B, H, Nq, Nk, C, scale=0.0) -> PbaDims:
    d = PbaDims()
    lib.pba_dims_dense(ctypes.byref(d), B, H, Nq, Nk, C, float(scale))
    return d


def pba_fwd(q, k, v, bias, key_mask, gate, out, lse, scale: float = 0.0, stream=None,
            window: int = -1) -> None:
    """Forward pass into preallocated `out` (bf16, like q) and `lse` (fp32 [B,H,Nq]).
    `window` >= 0: block-sparse local attention, query tile t (128 rows) attends key tiles
    [t - window, t + window] only (pba_fwd_local)."""
    d = make_dims(q, k, v, gate, out, bias, key_mask, scale)
    _check(lib.pba_fwd_local(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(key_mask), _ptr(gate),
                             _ptr(out), _ptr(lse), ctypes.byref(d), int(window), _stream(stream)))


def pba_bwd_workspace_size(dims: PbaDims) -> int:
    return int(lib.pba_bwd_workspace_size(ctypes.byref(dims)))


def pba_bwd(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate,
            workspace, scale: float = 0.0, stream=None, window: int = -1) -> None:
    """Backward pass into preallocated dq, dk, dv (like q/k/v), dbias (fp32 [H,Nq,Nk] or
    None), dgate (like gate, or None).  `workspace`: a uint8 CUDA tensor of at least
    pba_bwd_workspace_size(dims) bytes."""
    d = make_dims(q, k, v, gate, out, bias, key_mask, scale, dout=dout)
    for name, a, b in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v), ("dgate", dgate, gate),
                       ("dout", dout, out)):
        if a is not None and b is not None and a.stride() != b.stride():
            raise ValueError("%s must have the same strides as its forward tensor" % name)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pba_bwd_local(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(key_mask), _ptr(gate),
                             _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(dbias), _ptr(dgate), _ptr(workspace), ws_bytes, ctypes.byref(d),
                             int(window), _stream(stream)))


def pba_bwd_noalloc(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate,
                    scale: float = 0.0, stream=None) -> None:
    """pba_bwd without a workspace argument, for callers that cannot allocate device
    memory: the library's built-in 64 MiB scratch array is used instead (see pba.h)."""
    d = make_dims(q, k, v, gate, out, bias, key_mask, scale, dout=dout)
    _check(lib.pba_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(key_mask),
                               _ptr(gate), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                               _ptr(dk), _ptr(dv), _ptr(dbias), _ptr(dgate),
                               ctypes.byref(d), _stream(stream)))


def pwa_dims(v, gate=None, out=None, bias=None, key_mask=None, dout=None) -> PbaDims:
    """pba_dims for MSA pair-weighted averaging: v/gate/out [B,N,H,C], bias [H,N,N],
    key_mask one [N] row shared by every b."""
    d = make_dims(v, v, v, gate, out, bias, key_mask, 0.0, dout=dout)
    d.smask_b = 0
    return d


def pba_pwa_fwd(v, bias, key_mask, gate, out, lse_w, workspace, stream=None) -> None:
    """Pair-weighted averaging forward into preallocated `out` (like v) and `lse_w` (fp32
    [H,N]); `workspace`: uint8 CUDA tensor of pba_pwa_fwd_workspace_size bytes."""
    if key_mask is not None and key_mask.dim() != 1:
        raise ValueError("pair-weighted averaging takes one [N] key mask shared by every row")
    d = pwa_dims(v, gate, out, bias, key_mask)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pba_pwa_fwd(_ptr(v), _ptr(bias), _ptr(key_mask), _ptr(gate), _ptr(out), _ptr(lse_w),
                           _ptr(workspace), ws_bytes, ctypes.byref(d), _stream(stream)))


def pba_pwa_bwd(v, bias, key_mask, gate, out, dout, dv, dbias, dgate, workspace, stream=None) -> None:
    """Pair-weighted averaging backward into preallocated dv (like v), dbias (fp32 [H,N,N] or
    None) and dgate (like gate, or None)."""
    if key_mask is not None and key_mask.dim() != 1:
        raise ValueError("pair-weighted averaging takes one [N] key mask shared by every row")
    d = pwa_dims(v, gate, out, bias, key_mask, dout=dout)
    for name, a, b in (("dv", dv, v), ("dgate", dgate, gate), ("dout", dout, out)):
        if a is not None and b is not None and a.stride() != b.stride():
            raise ValueError("%s must have the same strides as its forward tensor" % name)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pba_pwa_bwd(_ptr(v), _ptr(bias), _ptr(key_mask), _ptr(gate), _ptr(out), _ptr(dout),
                           _ptr(dv), _ptr(dbias), _ptr(dgate), _ptr(workspace), ws_bytes,
                           ctypes.byref(d), _stream(stream)))


def pba_device_status(stream=None) -> None:
    """Synchronize the stream and raise if a kernel's bounded wait ran out."""
    _check(lib.pba_device_status(_stream(stream)))


# ---------------------------------------------------------------------------------------
# allocating conveniences (torch allocates; the library computes)
# ---------------------------------------------------------------------------------------

def attention_fwd(q, k, v, bias=None, key_mask=None, gate=None, scale: float = 0.0,
                  stream=None, window: int = -1):
    import torch
    B, Nq, H, C = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    pba_fwd(q, k, v, bias, key_mask, gate, out, lse, scale, stream, window)
    return out, lse


def attention_bwd(q, k, v, bias, key_mask, gate, out, lse, dout, scale: float = 0.0,
                  want_dbias: bool = True, stream=None, window: int = -1):
    import torch
    B, Nq, H, C = q.shape
    Nk = k.shape[1]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dgate = torch.empty_like(gate) if gate is not None else None
    dbias = (torch.empty((H, Nq, Nk), dtype=torch.float32, device=q.device)
             if want_dbias else None)
    d = make_dims(q, k, v, gate, out, bias, key_mask, scale, dout=dout)
    ws = torch.empty(max(pba_bwd_workspace_size(d), 1), dtype=torch.uint8, device=q.device)
    pba_bwd(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate, ws,
            scale, stream, window)
    return dq, dk, dv, dgate, dbias


# ---------------------------------------------------------------------------------------
# kernel timing (CUDA events around every launch of the library)
# ---------------------------------------------------------------------------------------

def profile_enable(on: bool = True) -> None:
    _check(lib.pba_profile_enable(1 if on else 0))


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since the last read."""
    arr = (PbaKernelStat * 32)()
    n = lib.pba_profile_read(arr, 32)
    if n < 0:
        raise PbaError(3, "reading kernel timing events failed")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(n)}


def pwa_fwd(v, bias=None, key_mask=None, gate=None, stream=None):
    """MSA pair-weighted averaging: out = sigmoid(gate) * sum_j softmax_j(bias + mask) v."""
    import torch
    B, N, H, C = v.shape
    out = torch.empty_like(v)
    lse_w = torch.empty((H, N), dtype=torch.float32, device=v.device)
    d = pwa_dims(v, gate, out, bias, key_mask)
    ws = torch.empty(max(int(lib.pba_pwa_fwd_workspace_size(ctypes.byref(d))), 1), dtype=torch.uint8,
                     device=v.device)
    pba_pwa_fwd(v, bias, key_mask, gate, out, lse_w, ws, stream)
    return out, lse_w


def pwa_bwd(v, bias, key_mask, gate, out, dout, want_dbias: bool = True, stream=None):
    import torch
    B, N, H, C = v.shape
    dv = torch.empty_like(v)
    dgate = torch.empty_like(gate) if gate is not None else None
    dbias = torch.empty((H, N, N), dtype=torch.float32, device=v.device) if want_dbias else None
    d = pwa_dims(v, gate, out, bias, key_mask, dout=dout)
    ws = torch.empty(max(int(lib.pba_pwa_bwd_workspace_size(ctypes.byref(d))), 1), dtype=torch.uint8,
                     device=v.device)
    pba_pwa_bwd(v, bias, key_mask, gate, out, dout, dv, dbias, dgate, ws, stream)
    return dv, dgate, dbias


def pair_bias_dims(z, bias=None, dbias=None, eps: float = 1e-5) -> PbaPairBiasDims:
    """pba_pair_bias_dims for z [Ni, Nj, Cz] (channel stride 1), bias [H, Ni, Nj] and dbias
    [H, Ni, Nj] (j stride 1); H is taken from bias or dbias."""
    Ni, Nj, Cz = z.shape
    assert z.stride(2) == 1, "z: channel stride must be 1"
    ref = bias if bias is not None else dbias
    d = PbaPairBiasDims()
    d.Ni, d.Nj, d.Cz, d.H = Ni, Nj, Cz, ref.shape[0]
    d.eps = eps
    d.sz[0], d.sz[1] = z.stride(0), z.stride(1)
    if bias is not None:
        assert bias.stride(2) == 1, "bias: j stride must be 1"
        d.sbias[0], d.sbias[1] = bias.stride(0), bias.stride(1)
    if dbias is not None:
        assert dbias.stride(2) == 1, "dbias: j stride must be 1"
        d.sdbias[0], d.sdbias[1] = dbias.stride(0), dbias.stride(1)
    return d


def pba_pair_bias_fwd(z, gamma, beta, w, bias, eps: float = 1e-5, stream=None) -> None:
    """Pair-bias projection into a preallocated bf16 `bias` [H, Ni, Nj]: LayerNorm over the
    channels of z [Ni, Nj, Cz] (bf16; gamma, beta fp32 [Cz]) then w (fp32 [Cz, H])."""
    d = pair_bias_dims(z, bias=bias, eps=eps)
    _check(lib.pba_pair_bias_fwd(_ptr(z), _ptr(gamma), _ptr(beta), _ptr(w), _ptr(bias),
                                 ctypes.byref(d), _stream(stream)))


def pba_pair_bias_bwd(z, gamma, beta, w, dbias, dz, dw, dgamma, dbeta, workspace, eps: float = 1e-5,
                      stream=None) -> None:
    """Backward of pba_pair_bias_fwd for a given fp32 dbias [H, Ni, Nj], into preallocated dz
    (like z), dw (fp32 [Cz, H]), dgamma and dbeta (fp32 [Cz])."""
    d = pair_bias_dims(z, dbias=dbias, eps=eps)
    _check(lib.pba_pair_bias_bwd(_ptr(z), _ptr(gamma), _ptr(beta), _ptr(w), _ptr(dbias), _ptr(dz),
                                 _ptr(dw), _ptr(dgamma), _ptr(dbeta), _ptr(workspace),
                                 workspace.numel() if workspace is not None else 0, ctypes.byref(d),
                                 _stream(stream)))


def pair_bias_fwd(z, gamma, beta, w, eps: float = 1e-5, stream=None):
    """bias [H, Ni, Nj] (bf16) = LayerNorm(z[i, j, :]; gamma, beta, eps) . w[:, h]."""
    import torch
    Ni, Nj, Cz = z.shape
    bias = torch.empty((w.shape[1], Ni, Nj), dtype=torch.bfloat16, device=z.device)
    pba_pair_bias_fwd(z, gamma, beta, w, bias, eps, stream)
    return bias


def pair_bias_bwd(z, gamma, beta, w, dbias, eps: float = 1e-5, stream=None):
    """(dz, dw, dgamma, dbeta) of the pair-bias projection for a given fp32 dbias."""
    import torch
    Cz = z.shape[2]
    dz = torch.empty_like(z)
    dw = torch.empty((Cz, w.shape[1]), dtype=torch.float32, device=z.device)
    dgamma = torch.empty(Cz, dtype=torch.float32, device=z.device)
    dbeta = torch.empty(Cz, dtype=torch.float32, device=z.device)
    d = pair_bias_dims(z, dbias=dbias, eps=eps)
    ws = torch.empty(max(int(lib.pba_pair_bias_bwd_workspace_size(ctypes.byref(d))), 256),
                     dtype=torch.uint8, device=z.device)
    pba_pair_bias_bwd(z, gamma, beta, w, dbias, dz, dw, dgamma, dbeta, ws, eps, stream)
    return dz, dw, dgamma, dbeta
