"""The benchmark's algorithmic work counts (the numerators of every throughput and roofline
figure) against counts worked out by hand, and the tile-window pair mask they use."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import pba_inputs as pi  # noqa: E402


def test_dense_attention_work():
    import bench
    cfg = pi.CONFIGS["C2"]   # 128 rows, 8 heads, 256 tokens (13 masked), c = 32
    w = bench.work(cfg)
    unit = 128 * 8 * 256 * (256 - 13) * 32
    assert w["fwd_flops"] == 4 * unit and w["bwd_flops"] == 10 * unit
    e = 128 * 256 * 8 * 32
    assert w["fwd_bytes"] == 5 * e * 2 + 128 * 8 * 256 * 4 + 8 * 256 * 256 * 2 + 256


def test_local_attention_work_counts_only_the_window():
    import bench
    cfg = pi.CONFIGS["C6"]   # 3072 atoms = 24 tiles, window 1, keys 3040..3071 masked
    w = bench.work(cfg)
    # key tiles seen per query tile: 2 at either end, 3 elsewhere; the masked keys all sit in
    # tile 23, which query tiles 22 and 23 see
    pairs = 128 * 128 * (2 + 22 * 3 + 2) - 2 * 128 * 32
    assert w["fwd_flops"] == 4 * 48 * 4 * pairs * 32
    band = 128 * 128 * (2 + 22 * 3 + 2)
    e = 48 * 3072 * 4 * 32
    assert w["fwd_bytes"] == 5 * e * 2 + 48 * 4 * 3072 * 4 + 4 * band * 2 + 3072


def test_window_pair_mask():
    m = pi.window_pair_mask(300, 520, 1)
    assert m.shape == (300, 520)
    assert m[0, 255] and not m[0, 256]          # query tile 0 sees key tiles 0 and 1
    assert m[129, 0] and m[129, 383] and not m[129, 384]
    assert m[299, 128] and not m[299, 127]      # query tile 2 sees key tiles 1..3
    assert pi.window_pair_mask(5, 7, -1).all()
    d = pi.window_pair_mask(640, 640, 0)
    assert np.array_equal(d, d.T) and d.sum() == 5 * 128 * 128


def test_nominal_peak_fractions():
    import bench
    assert bench.nominal(4000.0, "hbm") == {"peak": 8000.0, "unit": "GB/s", "frac": 0.5}
    assert bench.nominal(225.0, "tensor") == {"peak": 2250.0, "unit": "TFLOP/s", "frac": 0.1}


def test_kernel_code_keeps_one_kernel_and_its_helpers():
    import bench
    path = os.path.join(ROOT, "pair_biased_attention_gated_b200", "csrc", "pba_bwd.cuh")
    with open(path) as fh:
        text = fh.read()
    main = bench.kernel_code(text, "pba_bwd_main_kernel")
    dbias = bench.kernel_code(text, "pba_dbias_kernel")
    assert "pba_bwd_main_kernel(" in main and "pba_dbias_kernel(" not in main
    assert "pba_dbias_kernel(" in dbias and "pba_bwd_main_kernel(" not in dbias
    assert "struct BwdArgs" in main and "struct BwdArgs" in dbias   # shared helpers stay
    # a change inside one kernel's body changes its code only; a comment changes nothing
    marker = "if (!s_last) return;"
    assert text.count(marker) == 1
    edited = text.replace(marker, "if (!s_last) { return; }")
    assert bench.kernel_code(edited, "pba_dbias_kernel") != dbias
    assert bench.kernel_code(edited, "pba_bwd_main_kernel") == main
    assert bench.kernel_code(text + "\n// a note\n", "pba_dbias_kernel") == dbias
    # text that cannot be parsed is kept whole
    broken = "__global__ void k(int a { x"
    assert bench.kernel_code(broken, "other") == bench._code_only(broken)
