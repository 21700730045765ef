"""Compile libpba (csrc/*.cu) for sm_100a into this package directory.

Run as `python pair_biased_attention_gated_b200/build.py` or through the repository's
build entry point.  nvcc cross-compiles without a GPU.
"""
import glob
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libpba.so")
SRC = os.path.join(HERE, "csrc", "pba_api.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2", "-shared",
    "--expt-relaxed-constexpr",
]


def _inputs():
    return (glob.glob(os.path.join(HERE, "csrc", "*")) +
            [os.path.join(ROOT, "include", "pba.h"), os.path.abspath(__file__)])


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


# Kernels that split their registers between warpgroups with setmaxnreg.  The split adds
# up to at most the registers the CTA is launched with (threads x the count ptxas assigns);
# if ptxas assigned a different count the split could wait forever, so the build refuses.
SETMAXNREG_KERNELS = {"pba_fwd_kernel": 128}


def check_registers(ptxas_log: str) -> None:
    current = None
    seen = {}
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current:
            seen[current] = int(m.group(1))
            current = None
    for name, want in SETMAXNREG_KERNELS.items():
        hits = {k: v for k, v in seen.items() if name in k}
        if not hits:
            raise RuntimeError("ptxas output has no register count for %s" % name)
        bad = {k: v for k, v in hits.items() if v != want}
        if bad:
            raise RuntimeError("register count of %s is %s, expected %d: the setmaxnreg split "
                               "would not match the launch" % (name, bad, want))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + NVCC_FLAGS + ["-Xptxas", "-v", "-o", tmp, SRC]
    proc = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if verbose or proc.returncode != 0:
        print(proc.stdout)
    if proc.returncode != 0:
        raise subprocess.CalledProcessError(proc.returncode, cmd, proc.stdout)
    check_registers(proc.stdout)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
