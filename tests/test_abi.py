"""The C-ABI library loads on a machine without a GPU, exports every function that
include/pba.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pba():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "pba_build", os.path.join(ROOT, "pair_biased_attention_gated_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import pair_biased_attention_gated_b200 as p
    return p


def _declared_functions():
    names = []
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if not hdr.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(pba_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("pba_fwd", "pba_bwd", "pba_bwd_workspace_size", "pba_status_string",
                     "pba_device_status", "pba_dims_dense", "pba_last_error", "pba_version"):
        assert required in names


def test_every_declared_symbol_is_exported(pba):
    lib = ctypes.CDLL(pba.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(pba):
    assert pba.lib.pba_version() == 1
    for code, name in pba.STATUS.items():
        assert pba.lib.pba_status_string(code).decode() == name


def test_dims_dense(pba):
    d = pba.dims_dense(3, 4, 5, 6, 32)
    assert (d.B, d.H, d.Nq, d.Nk, d.C) == (3, 4, 5, 6, 32)
    assert list(d.sq) == [5 * 4 * 32, 4 * 32, 32]
    assert list(d.sk) == [6 * 4 * 32, 4 * 32, 32]
    assert list(d.sbias) == [5 * 6, 6]
    assert d.smask_b == 0


def _fwd_status(pba, d, q=16, k=16, v=16, out=16, lse=16, bias=None, gate=None):
    st = pba.lib.pba_fwd(q, k, v, bias, None, gate, out, lse, ctypes.byref(d), None)
    return st, pba.lib.pba_last_error().decode()


def test_host_side_argument_errors(pba):
    d = pba.dims_dense(2, 2, 64, 64, 32)
    assert _fwd_status(pba, d, q=None)[0] == 1
    assert _fwd_status(pba, d, out=None)[0] == 1
    assert _fwd_status(pba, d, q=24)[0] == 1          # misaligned pointer
    d2 = pba.dims_dense(2, 2, 64, 64, 12)            # C not a multiple of 8
    assert _fwd_status(pba, d2)[0] == 2
    d3 = pba.dims_dense(2, 2, 64, 64, 128)           # C > 64
    assert _fwd_status(pba, d3)[0] == 2
    d4 = pba.dims_dense(2, 2, 64, 64, 32)
    d4.sq[1] = 100                                    # stride not a multiple of 8
    st, msg = _fwd_status(pba, d4)
    assert st == 1 and "stride" in msg
    d5 = pba.dims_dense(2, 2, 64, 64, 32)
    d5.scale = float("nan")
    assert _fwd_status(pba, d5)[0] == 1
    d6 = pba.dims_dense(-1, 2, 64, 64, 32)
    assert _fwd_status(pba, d6)[0] == 1
    d7 = pba.dims_dense(2, 2, 64, 60, 32)            # bias row stride 60: not TMA-able
    assert _fwd_status(pba, d7, bias=16)[0] == 1


def test_empty_problem_is_a_no_op(pba):
    d = pba.dims_dense(0, 2, 64, 64, 32)
    assert _fwd_status(pba, d, q=None, k=None, v=None, out=None, lse=None)[0] == 0
    d = pba.dims_dense(2, 2, 0, 64, 32)
    assert _fwd_status(pba, d, q=None, k=None, v=None, out=None, lse=None)[0] == 0


def _pb_dims(pba, Ni=8, Nj=8, Cz=128, H=4, eps=1e-5):
    d = pba.PbaPairBiasDims()
    d.Ni, d.Nj, d.Cz, d.H, d.eps = Ni, Nj, Cz, H, eps
    d.sz[0], d.sz[1] = Nj * Cz, Cz
    d.sbias[0], d.sbias[1] = Ni * Nj, Nj
    d.sdbias[0], d.sdbias[1] = Ni * Nj, Nj
    return d


def _pb_fwd_status(pba, d, z=16, bias=16):
    st = pba.lib.pba_pair_bias_fwd(z, 16, 16, 16, bias, ctypes.byref(d), None)
    return st, pba.lib.pba_last_error().decode()


def test_pair_bias_host_side_argument_errors(pba):
    assert _pb_fwd_status(pba, _pb_dims(pba, Cz=100))[0] == 2          # Cz not supported
    assert _pb_fwd_status(pba, _pb_dims(pba, H=17))[0] == 2            # too many heads
    assert _pb_fwd_status(pba, _pb_dims(pba, eps=0.0))[0] == 1         # eps must be > 0
    assert _pb_fwd_status(pba, _pb_dims(pba, eps=float("nan")))[0] == 1
    assert _pb_fwd_status(pba, _pb_dims(pba, Ni=-1))[0] == 1
    d = _pb_dims(pba)
    d.sz[1] = 100                                                        # not a multiple of 8
    st, msg = _pb_fwd_status(pba, d)
    assert st == 1 and "stride" in msg
    assert _pb_fwd_status(pba, _pb_dims(pba), z=None)[0] == 1
    assert _pb_fwd_status(pba, _pb_dims(pba), z=24)[0] == 1             # misaligned z
    assert _pb_fwd_status(pba, _pb_dims(pba, Ni=0), z=None, bias=None)[0] == 0   # empty: no-op
    d = _pb_dims(pba)
    need = pba.lib.pba_pair_bias_bwd_workspace_size(ctypes.byref(d))
    assert need > 0
    st = pba.lib.pba_pair_bias_bwd(16, 16, 16, 16, 16, 16, 16, 16, 16, 256, need - 4, ctypes.byref(d), None)
    assert st == 5                                                       # workspace too small
    assert pba.lib.pba_pair_bias_bwd_workspace_size(ctypes.byref(_pb_dims(pba, Cz=100))) == 0


def test_local_window_refusals(pba):
    d = pba.dims_dense(2, 2, 128, 1024, 32)          # 1 query tile, 8 key tiles
    st = pba.lib.pba_fwd_local(16, 16, 16, None, None, None, 16, 16, ctypes.byref(d), 0, None)
    assert st == 2 and "window" in pba.lib.pba_last_error().decode()
    st = pba.lib.pba_bwd_local(*([16] * 9), 16, 16, 16, None, None, 256, 1 << 30, ctypes.byref(d), 0, None)
    assert st == 2
    d0 = pba.dims_dense(0, 2, 128, 1024, 32)         # empty problem, but the window is still checked
    assert pba.lib.pba_fwd_local(None, None, None, None, None, None, None, None, ctypes.byref(d0), 0, None) == 2
    # window -1 is the dense operator: the same empty problem is a no-op
    assert pba.lib.pba_fwd_local(None, None, None, None, None, None, None, None, ctypes.byref(d0), -1, None) == 0
