"""The oracle and the CUDA path stay independent, and the product never reaches the oracle:
no source file of the package or the C ABI names the oracle, no oracle file names the
package, its kernels or its header, and the shared input generator imports neither."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _files(sub, exts):
    for dirpath, _, names in os.walk(os.path.join(ROOT, sub)):
        if "__pycache__" in dirpath:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def _read(path):
    with open(path, encoding="utf-8") as fh:
        return fh.read()


def test_product_never_names_the_oracle():
    for path in list(_files("pair_biased_attention_gated_b200", (".py", ".cu", ".cuh", ".h"))) + \
            list(_files("include", (".h",))):
        assert not re.search(r"\boracle\b", _read(path)), path


def test_oracle_shares_nothing_with_the_cuda_path():
    for path in _files("oracle", (".py", ".c", ".h")):
        text = _read(path)
        for name in ("pair_biased_attention_gated_b200", "pba.h", "pba_device", "csrc", "libpba.so"):
            assert name not in text, (path, name)


def test_input_generator_imports_neither_side():
    for path in _files("pba_inputs", (".py",)):
        text = _read(path)
        assert not re.search(r"^\s*(from|import)\s+(oracle|pair_biased_attention_gated_b200)\b", text, re.M), path
