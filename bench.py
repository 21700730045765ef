#!/usr/bin/env python
"""Benchmark of pair-biased gated attention on B200: fwd+bwd TFLOP/s and % of roofline.

A step is one pass of the whole hot path: the forward kernel (out, lse) and the backward
kernels (dq, dk, dv, dgate, dbias) over one batch of synthetic, seeded bf16 input.  The
default workload is the large triangle attention (768 rows x 768 keys, 4 heads, c = 32,
the largest workload that the target names and that fits one GPU); `--config` selects
another.  Inputs are resident in HBM when the timed region starts; L2 is flushed before
every timed step, outside the timed events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config C5] [--impl ours|reference]
                  [--op attention|pwa|pairbias] [--also C1,C2,C3,C4]

The line reports the whole step (value, step_roofline), the dominant kernel's roofline,
each pass's roofline fraction (fwd_roofline_frac, bwd_roofline_frac), and under
`workloads` the same per-pass figures for the other workloads (`--also`, device timing
only).  Tensor-bound fractions use the burst bf16 peak (kernels timed per launch); the
sustained peak is reported beside it.

N > 1 runs under torchrun, one process per GPU, each an independent replica of the
workload (the path has no exchange step); rank 0 prints one JSON line.  `--impl
reference` times the fp64 CPU oracle (the only other implementation of the operation)
on the host cores instead.  `--config C6` is the block-sparse local (atom) attention
workload; `--op pwa` times MSA pair-weighted averaging and `--op pairbias` the LayerNorm +
projection that makes the bias, each with its own metric line.  The end-to-end figure
copies every step's inputs in and results out of pinned host memory, pipelined over a
copy-in, a compute and a copy-out stream.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import pba_inputs as pi  # noqa: E402

METRIC = "pair-bias attention fwd / fwd+bwd TFLOP/s and %roofline on 1 B200"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 data-sheet figures (dense bf16, HBM3e), reported beside the measured-peak fractions
NOMINAL_PEAKS = {"hbm": (8000.0, "GB/s"), "tensor": (2250.0, "TFLOP/s")}


def nominal(achieved, bound):
    """The achieved rate as a fraction of the data-sheet peak of its bound."""
    peak, unit = NOMINAL_PEAKS[bound]
    return {"peak": peak, "unit": unit, "frac": round(achieved / peak, 4)}


# ---------------------------------------------------------------------------------------
# algorithmic work (unmasked keys only; c is the true head dim)
# ---------------------------------------------------------------------------------------

def oracle_inputs(cfg: pi.Config, d):
    """The oracle's fp64 view of one draw; under a tile window the bias carries -inf at the
    pairs the window excludes, which is what local attention computes."""
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    if cfg.window >= 0 and "bias" in f:
        f["bias"] = np.where(pi.window_pair_mask(cfg.N, cfg.N, cfg.window)[None], f["bias"], -np.inf)
    return f


def work(cfg: pi.Config, B=None):
    """Algorithmic flops and bytes: products over attended (query, key) pairs only (unmasked
    keys, and under a tile window only the pairs it keeps); the bias read where it is used."""
    B = cfg.B if B is None else B
    H, N, c = cfg.H, cfg.N, cfg.c
    pairs = pi.window_pair_mask(N, N, cfg.window)
    attended = int((pairs & (cfg.keep()[None, :] != 0)).sum())   # sum over rows of attended keys
    unit = B * H * attended * c
    e = B * N * H * c                       # elements of one [B, N, H, c] tensor
    bias_b = H * int(pairs.sum()) * 2
    lse_b = B * H * N * 4
    mask_b = N
    f = {
        "fwd_flops": 4 * unit,
        "bwd_flops": 10 * unit,
        # q, k, v, g in; out out; lse out; bias; mask
        "fwd_bytes": 5 * e * 2 + lse_b + bias_b + mask_b,
        # q, k, v, g, out, dout in; dq, dk, dv, dg out; lse; bias; mask; dbias out
        "bwd_bytes": 10 * e * 2 + lse_b + bias_b + mask_b + H * N * N * 4,
    }
    # per-kernel algorithmic figures (what each kernel must move / multiply at minimum)
    f["kernels"] = {
        "pba_fwd_kernel": (4 * unit, 5 * e * 2 + lse_b + bias_b + mask_b),
        # q, k, v, dOa, (lse, D) in; dq, dk, dv out; bias; mask
        "pba_bwd_main_kernel": (10 * unit, 7 * e * 2 + B * H * N * 8 + bias_b + mask_b),
        # q, k, v, dOa, (lse, D) in; bias; dbias out (the split partials are workspace)
        "pba_dbias_kernel": (0, 4 * e * 2 + B * H * N * 8 + bias_b + H * N * N * 4),
        # out, dout, g, lse in; dOa, dg, (lse, D) out
        "pba_bwd_pre_kernel": (0, 5 * e * 2 + lse_b + B * H * N * 8),
        "pba_dq_convert_kernel": (0, e * 4 + e * 2),
    }
    return f


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def peak_rates(peaks):
    """(HBM GB/s, burst bf16 TFLOP/s, sustained bf16 TFLOP/s).  The kernels are timed per
    launch, each well under a millisecond, so a tensor-bound fraction is taken against the
    burst figure; the sustained one is reported beside it."""
    tens = float(peaks["bf16_tflops"])
    return float(peaks["hbm_gbs"]), tens, float(peaks.get("bf16_tflops_sustained", tens))



def pass_figures(w, fwd_ms, bwd_ms, hbm, tens):
    """Per-pass device time (events on the launching stream around each pass, averaged over
    the timed steps; the backward pass runs its dbias kernel beside the dq conversion, so a
    sum of kernel times would count that overlap twice) and roofline fraction: roofline time
    = max(flops / tensor peak, bytes / HBM peak) of the pass."""
    out = {}
    for name, ms, fl, by in (("fwd", fwd_ms, w["fwd_flops"], w["fwd_bytes"]),
                             ("bwd", bwd_ms, w["bwd_flops"], w["bwd_bytes"])):
        t_roof = max(fl / (tens * 1e12), by / (hbm * 1e9))
        out[name + "_us"] = round(ms * 1e3, 2) if ms > 0 else None
        out[name + "_tflops"] = round(fl / (ms / 1e3) / 1e12, 3) if ms > 0 else None
        out[name + "_roofline_us"] = round(t_roof * 1e6, 2)
        out[name + "_roofline_bound"] = "tensor" if fl / (tens * 1e12) > by / (hbm * 1e9) else "hbm"
        out[name + "_roofline_frac"] = round(t_roof * 1e3 / ms, 4) if ms > 0 else None
    return out


def time_workload(pba, cfg, args):
    """Device timing of one more workload (fwd + bwd step, L2 flushed before each step):
    per-pass time, TFLOP/s and roofline fraction from the library's per-kernel events."""
    import torch
    d = pi.make_inputs(cfg, seed=args.seed)
    t = {}
    for k, a in d.items():
        t[k] = (torch.from_numpy(np.ascontiguousarray(a)) if k == "keep" else
                torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)).cuda()
    q, kk, v, g, bias, keep, dout = t["q"], t["k"], t["v"], t.get("g"), t["bias"], t["keep"], t["dout"]
    B, N, H, C = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(kk), torch.empty_like(v)
    dg = torch.empty_like(g) if g is not None else None
    db = torch.empty(H, N, N, dtype=torch.float32, device="cuda")
    dims = pba.make_dims(q, kk, v, g, out, bias, keep)
    ws = torch.empty(pba.pba_bwd_workspace_size(dims), dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def step():
        pba.pba_fwd(q, kk, v, bias, keep, g, out, lse, window=cfg.window)
        pba.pba_bwd(q, kk, v, bias, keep, g, out, lse, dout, dq, dk, dv, db, dg, ws, window=cfg.window)

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step()
    pba.pba_device_status()
    K = max(3, min(args.steps, 20))
    stream = torch.cuda.current_stream()
    pev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(K)]
    torch.cuda.synchronize()
    pba.profile_read()
    pba.profile_enable(True)
    for i in range(K):
        flush.fill_(i & 0xFF)
        pev[i][0].record(stream)
        pba.pba_fwd(q, kk, v, bias, keep, g, out, lse, window=cfg.window)
        pev[i][1].record(stream)
        pba.pba_bwd(q, kk, v, bias, keep, g, out, lse, dout, dq, dk, dv, db, dg, ws, window=cfg.window)
        pev[i][2].record(stream)
    torch.cuda.synchronize()
    pba.profile_enable(False)
    kstats = pba.profile_read()
    pba.pba_device_status()
    peaks, _ = load_peaks()
    hbm, tens, _ = peak_rates(peaks)
    w = work(cfg)
    fwd_ms = sum(a.elapsed_time(b) for a, b, _ in pev) / K
    bwd_ms = sum(b.elapsed_time(c) for _, b, c in pev) / K
    res = {"workload": cfg.desc, "passes_named": "fwd+bwd" if cfg.passes == "fwdbwd" else "fwd",
           "steps": K, **pass_figures(w, fwd_ms, bwd_ms, hbm, tens),
           "kernels_us": {n: round(ms / l * 1e3, 2) for n, (l, ms) in kstats.items()}}
    del q, kk, v, g, bias, keep, dout, out, lse, dq, dk, dv, dg, db, ws, flush, t
    torch.cuda.empty_cache()
    return res


KERNEL_SOURCES = {"pba_fwd_kernel": "pba_fwd.cuh"}   # every other attention kernel: pba_bwd.cuh


def kernel_source_file(kernel: str) -> str:
    if kernel.startswith("pba_pwa_"):
        return "pba_pwa.cuh"
    if kernel.startswith("pba_pair_bias_"):
        return "pba_pairbias.cuh"
    return KERNEL_SOURCES.get(kernel, "pba_bwd.cuh")


def _code_only(text: str) -> str:
    """Source text without comments and blank lines: a comment edit is not a kernel change."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def _without_other_kernels(code: str, kernel: str) -> str:
    """`code` without the definitions of its __global__ functions other than `kernel`
    (helpers, structures and the kernel itself stay); the whole of `code` if it cannot be
    parsed."""
    import re
    try:
        out, pos = [], 0
        for m in re.finditer(r"__global__\s+void\s+(?:__launch_bounds__\s*\([^)]*\)\s*)?(\w+)\s*\(", code):
            i, depth = m.end(), 1
            while depth:                      # the parameter list
                depth += (code[i] == "(") - (code[i] == ")")
                i += 1
            k = code.index("{", i) + 1
            depth = 1
            while depth:                      # the body
                depth += (code[k] == "{") - (code[k] == "}")
                k += 1
            if m.group(1) != kernel:
                out.append(code[pos:m.start()])
                pos = k
        out.append(code[pos:])
        return "".join(out)
    except (IndexError, ValueError):
        return code


def kernel_code(text: str, kernel: str) -> str:
    """The part of a source file's text that one kernel is compiled from: no comments, and
    none of the other kernels defined beside it (`kernel` may carry a suffix, e.g.
    "pba_pwa_gemm_kernel (dv)")."""
    return _without_other_kernels(_code_only(text), kernel.split()[0].split("<")[0])


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code one kernel is compiled from: its own definition with the helpers of
    its file, and the shared device header, comments left out (launch configuration in the
    API file is not covered)."""
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "pair_biased_attention_gated_b200", "csrc")
    for name in (kernel_source_file(kernel), "pba_device.cuh"):
        with open(os.path.join(cdir, name), encoding="utf-8") as fh:
            text = fh.read()
        code = kernel_code(text, kernel) if name != "pba_device.cuh" else _code_only(text)
        h.update(name.encode() + code.encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None when the
    summary is missing or was taken on different kernel sources."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    ent = d.get("kernels", {}).get(kernel, {}).get(workload)
    if ent is None or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------------------
# clocks during the timed region (NVML polling thread; reads only)
# ---------------------------------------------------------------------------------------

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # no NVML: clocks are reported as unavailable
            self._nv = None
        self.period = period_s
        self._t = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[local_rank])
        except (ValueError, IndexError):
            return local_rank
    return local_rank


# ---------------------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the `--impl reference` arm)
# ---------------------------------------------------------------------------------------

def time_oracle(cfg: pi.Config, target_s: float, seed: int = 0, max_rows=None):
    """fp64 oracle fwd+bwd on the first B_s broadcast rows of the workload, B_s sized for
    about `target_s` seconds (the whole workload, repeated, when that is faster)."""
    import oracle
    import numpy as np

    def run(Bs):
        d = pi.make_inputs(cfg, seed=seed, B=Bs)
        f = oracle_inputs(cfg, d)
        t0 = time.perf_counter()
        oracle.fwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f.get("g"))
        oracle.bwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f.get("g"), f["dout"])
        return time.perf_counter() - t0

    t1 = run(1)
    per_row = max(t1, 1e-4)
    Bs = int(max(1, min(cfg.B, target_s / per_row)))
    if max_rows:
        Bs = min(Bs, max_rows)
    reps, elapsed = 0, 0.0
    while True:
        elapsed += run(Bs)
        reps += 1
        if elapsed >= target_s * 0.5 or Bs < cfg.B:
            break
    w = work(cfg, B=Bs)
    flops = (w["fwd_flops"] + w["bwd_flops"]) * reps
    threads = oracle.threads()
    return {
        "value": flops / elapsed / 1e12, "unit": "TFLOP/s",
        "cores": min(threads, Bs * cfg.H), "kind": "oracle",
        "sample": "%s fwd+bwd on %d of %d broadcast rows, x%d, %.1f s; fp64 C loops, OpenMP: "
                  "fwd over (b,h) pairs, bwd over the %d heads (%d threads available)"
                  % (cfg.name, Bs, cfg.B, reps, elapsed, cfg.H, threads),
        "seconds": elapsed, "rows": Bs, "reps": reps,
    }


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(pg, values, device="cuda"):
    """Every rank's timings -> their maximum over the ranks (the slowest replica sets the
    job's time); `pg` is torch.distributed or None for one process."""
    if pg is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(world, units_per_step, steps, elapsed_ms):
    """Whole-job units per second: every replica processed `steps` steps of `units_per_step`
    within the slowest rank's `elapsed_ms`."""
    return world * units_per_step * steps / (elapsed_ms / 1e3)


def run_ours(args, cfg):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    lib_path = os.path.join(ROOT, "pair_biased_attention_gated_b200", "libpba.so")
    if not os.path.exists(lib_path):
        if rank == 0:
            import importlib.util
            spec = importlib.util.spec_from_file_location(
                "pba_build", os.path.join(ROOT, "pair_biased_attention_gated_b200", "build.py"))
            mod = importlib.util.module_from_spec(spec)
            spec.loader.exec_module(mod)
            mod.build()
        if pg:
            pg.barrier()
    import numpy as np
    import pair_biased_attention_gated_b200 as pba

    d = pi.make_inputs(cfg, seed=args.seed)
    host = {}
    for k, a in d.items():
        t = torch.from_numpy(np.ascontiguousarray(a)) if k == "keep" else \
            torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        host[k] = t.pin_memory()
    dev = {k: v.cuda() for k, v in host.items()}
    q, kk, v, g, bias, keep, dout = (dev["q"], dev["k"], dev["v"], dev.get("g"), dev["bias"],
                                     dev["keep"], dev["dout"])
    B, N, H, C = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(kk), torch.empty_like(v)
    dg = torch.empty_like(g) if g is not None else None
    db = torch.empty(H, N, N, dtype=torch.float32, device="cuda")
    dims = pba.make_dims(q, kk, v, g, out, bias, keep)
    ws = torch.empty(pba.pba_bwd_workspace_size(dims), dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        pba.pba_fwd(q, kk, v, bias, keep, g, out, lse, window=cfg.window)
        pba.pba_bwd(q, kk, v, bias, keep, g, out, lse, dout, dq, dk, dv, db, dg, ws, window=cfg.window)

    def l2_flush(i):
        flush.fill_(i & 0xFF)

    for i in range(args.warmup):
        l2_flush(i)
        step()
    pba.pba_device_status()

    # ---- device-timed region: inputs resident in HBM.  Each step is bracketed by events on
    # the launching stream, with one more between its forward and backward pass.
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    evm = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(physical_gpu_index(local))
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    pba.profile_read()                   # drop anything recorded before
    pba.profile_enable(True)
    sampler.start()
    for i in range(K):
        l2_flush(i)
        ev[i][0].record(stream)
        pba.pba_fwd(q, kk, v, bias, keep, g, out, lse, window=cfg.window)
        evm[i].record(stream)
        pba.pba_bwd(q, kk, v, bias, keep, g, out, lse, dout, dq, dk, dv, db, dg, ws, window=cfg.window)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clocks = sampler.stop()
    pba.profile_enable(False)
    kstats = pba.profile_read()
    pba.pba_device_status()
    elapsed_ms = sum(a.elapsed_time(b) for a, b in ev)
    fwd_ms = sum(a.elapsed_time(m) for (a, _), m in zip(ev, evm)) / K
    bwd_ms = sum(m.elapsed_time(b) for (_, b), m in zip(ev, evm)) / K

    # ---- end-to-end region: host buffers, every step's copies inside the timed region.
    # Three streams and two tensor sets: step i's inputs go in (copy-in stream) while step
    # i - 1 computes and step i - 2's results come out (copy-out stream); PCIe carries both
    # directions at once.  The region runs from the first input copy to the last result copy.
    douts = {"out": out, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "db": db}
    if dg is not None:
        douts["dg"] = dg
    sets = [dict(dev, ws=ws, **douts)]
    sets.append({k2: torch.empty_like(t2) for k2, t2 in sets[0].items()})
    hbufs = [{k2: torch.empty(t2.shape, dtype=t2.dtype).pin_memory() for k2, t2 in douts.items()}
             for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in hbufs[0].values())

    def step_on(S):
        pba.pba_fwd(S["q"], S["k"], S["v"], S["bias"], S["keep"], S.get("g"), S["out"], S["lse"],
                    window=cfg.window)
        pba.pba_bwd(S["q"], S["k"], S["v"], S["bias"], S["keep"], S.get("g"), S["out"], S["lse"],
                    S["dout"], S["dq"], S["dk"], S["dv"], S["db"], S.get("dg"), S["ws"], window=cfg.window)

    K2 = max(2, min(K, 20))
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    t_begin.record(copy_in)
    for i in range(K2):
        x = i & 1
        S = sets[x]
        if i >= 2:
            copy_in.wait_event(ev_comp[x])     # step i - 2 no longer reads this set's inputs
        with torch.cuda.stream(copy_in):
            for k2, t in host.items():
                S[k2].copy_(t, non_blocking=True)
        ev_in[x].record(copy_in)
        stream.wait_event(ev_in[x])
        if i >= 2:
            stream.wait_event(ev_out[x])       # step i - 2's results have left this set
        l2_flush(i)
        step_on(S)
        ev_comp[x].record(stream)
        copy_out.wait_event(ev_comp[x])
        with torch.cuda.stream(copy_out):
            for k2, t in hbufs[x].items():
                t.copy_(S[k2], non_blocking=True)
        ev_out[x].record(copy_out)
    t_end.record(copy_out)   # after the last result copy (the stream runs in order)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    e2e_ms = t_begin.elapsed_time(t_end)
    pba.pba_device_status()

    elapsed_ms, e2e_ms = max_over_ranks(pg, [elapsed_ms, e2e_ms])

    w = work(cfg)
    step_flops = w["fwd_flops"] + w["bwd_flops"]
    value = job_throughput(world, step_flops, K, elapsed_ms) / 1e12
    e2e_value = job_throughput(world, step_flops, K2, e2e_ms) / 1e12

    peaks, peak_src = load_peaks()
    hbm, tens, tens_sus = peak_rates(peaks)
    # dominant kernel and its roofline
    total_k = sum(ms for _, ms in kstats.values()) or 1.0
    dom = max(kstats.items(), key=lambda kv: kv[1][1])[0] if kstats else None
    roof = None
    if dom:
        launches, ms = kstats[dom]
        avg_s = ms / launches / 1e3
        kf, kb = w["kernels"].get(dom, (0, 0))
        t_tensor, t_hbm = kf / (tens * 1e12), kb / (hbm * 1e9)
        if t_tensor > t_hbm:
            achieved, peak, unit, bound = kf / avg_s / 1e12, tens, "TFLOP/s", "tensor"
        else:
            achieved, peak, unit, bound = kb / avg_s / 1e9, hbm, "GB/s", "hbm"
        roof = {"kernel": dom, "bound": bound, "achieved": round(achieved, 2),
                "peak": peak, "unit": unit, "frac": round(achieved / peak, 4),
                "peak_source": "%s (%s)" % (peak_src, "burst bf16" if bound == "tensor" else "copy"),
                "algorithmic_per_launch": {"flops": kf, "bytes": kb},
                "avg_launch_us": round(avg_s * 1e6, 2),
                "traffic": ncu_traffic(dom, cfg.name),
                "nominal": nominal(achieved, bound)}
        if bound == "tensor":
            roof["sustained"] = {"peak": tens_sus, "frac": round(achieved / tens_sus, 4)}
    # the whole step against its own roofline
    t_step_roof = max(step_flops / (tens * 1e12),
                      (w["fwd_bytes"] + w["bwd_bytes"]) / (hbm * 1e9))
    ms_per_step = elapsed_ms / K
    kernels = {n: {"launches": l, "avg_us": round(ms / l * 1e3, 2), "share": round(ms / total_k, 4)}
               for n, (l, ms) in sorted(kstats.items(), key=lambda kv: -kv[1][1])}
    launches_total = sum(l for l, _ in kstats.values())

    res = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 q/k/v/gate/dout, N(0,%g^2) bias, shapes of "
                "the named workload" % cfg.bias_std,
        "config": {"workload": "%s: %s" % (cfg.name, cfg.desc), "B": cfg.B, "H": cfg.H,
                   "N": cfg.N, "c": cfg.c, "masked_keys": cfg.N - cfg.n_valid_keys,
                   "gate": cfg.gate, "passes": "fwd+bwd (dq, dk, dv, dgate, dbias)",
                   "l2": "flushed before every timed step (256 MiB write outside the events)",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roof,
        "step_roofline": {"time_us": round(t_step_roof * 1e6, 2),
                          "frac": round(t_step_roof * 1e3 / ms_per_step, 4)},
        **pass_figures(w, fwd_ms, bwd_ms, hbm, tens),
        "kernels": kernels,
        "gpu_launches": launches_total,
        "clocks": clocks,
        "e2e": {"value": round(e2e_value, 4), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": K2},
    }
    if world == 1 and args.also:
        res["workloads"] = {}
        for name in [x for x in args.also.split(",") if x and x != cfg.name]:
            res["workloads"][name] = time_workload(pba, pi.CONFIGS[name], args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = time_oracle(cfg, target_s=args.cpu_seconds, seed=args.seed)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return res if rank == 0 else None


def run_reference(args, cfg):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    W, K = args.warmup, args.steps
    # size one step so the whole run stays within a few minutes
    per_step_s = max(0.2, min(4.0, 150.0 / max(1, K + W)))
    cal = time_oracle(cfg, target_s=per_step_s, seed=args.seed)
    Bs = cal["rows"]
    import oracle
    import numpy as np  # noqa: F401
    d = pi.make_inputs(cfg, seed=args.seed, B=Bs)
    f = oracle_inputs(cfg, d)

    def step():
        oracle.fwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f.get("g"))
        oracle.bwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f.get("g"), f["dout"])

    for _ in range(W):
        step()
    t0 = time.perf_counter()
    for _ in range(K):
        step()
    el = time.perf_counter() - t0
    w = work(cfg, B=Bs)
    value = (w["fwd_flops"] + w["bwd_flops"]) * K / el / 1e12
    threads = oracle.threads()
    sample = ("%s fwd+bwd on %d of %d broadcast rows per step; fp64 C loops, OpenMP (fwd over "
              "(b,h), bwd over the %d heads; %d threads available)"
              % (cfg.name, Bs, cfg.B, cfg.H, threads))
    return {
        "metric": METRIC, "impl": "reference", "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(el / K * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded bf16 inputs of the named workload, widened to fp64",
        "config": {"workload": "%s: %s" % (cfg.name, cfg.desc), "B": cfg.B, "H": cfg.H,
                   "N": cfg.N, "c": cfg.c, "sample_rows": Bs,
                   "passes": "fwd+bwd (dq, dk, dv, dgate, dbias)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                         "cores": min(threads, Bs * cfg.H), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }

# ---------------------------------------------------------------------------------------
# MSA pair-weighted averaging (--op pwa): the same contract on the second operator
# ---------------------------------------------------------------------------------------
PWA_METRIC = "MSA pair-weighted averaging fwd+bwd TFLOP/s and %roofline on 1 B200"


def pwa_work(cfg, B=None):
    """Algorithmic work of pair-weighted averaging (Nv = attended keys): fwd 2 B H N Nv c
    (W V), bwd 4 B H N Nv c (W^T dOa and dOa V^T); bytes as each pass must move."""
    B = cfg.B if B is None else B
    H, N, c, Nv = cfg.H, cfg.N, cfg.c, cfg.n_valid_keys
    e = B * N * H * c
    unit = B * H * N * Nv * c
    bias_b, nn4 = H * N * N * 2, H * N * N * 4
    f = {"fwd_flops": 2 * unit, "bwd_flops": 4 * unit,
         "fwd_bytes": 3 * e * 2 + bias_b + H * N * 4 + N,
         "bwd_bytes": 6 * e * 2 + bias_b + nn4 + N}
    f["kernels"] = {
        "pba_pwa_weights_kernel": (0, 2 * bias_b + H * N * 4),
        "pba_pwa_gemm_kernel (out)": (2 * unit, 3 * e * 2 + bias_b),
        "pba_pwa_pre_kernel": (0, 5 * e * 2),
        "pba_pwa_gemm_kernel (dv)": (2 * unit, 2 * e * 2 + bias_b),
        "pba_pwa_dw_kernel": (2 * unit, 2 * e * 2),
        "pba_pwa_dbias_kernel": (0, bias_b + nn4),
    }
    return f


def time_pwa_oracle(cfg, target_s, seed):
    import oracle
    B1 = max(1, min(cfg.B, 2))
    d = pi.make_inputs(cfg, seed=seed, B=B1)
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    t0 = time.perf_counter()
    oracle.pwa_fwd(f["v"], f["bias"], f["keep"], f.get("g"))
    oracle.pwa_bwd(f["v"], f["bias"], f["keep"], f.get("g"), f["dout"])
    per_row = (time.perf_counter() - t0) / B1
    rows = int(max(1, min(cfg.B, target_s / max(per_row, 1e-6))))
    d = pi.make_inputs(cfg, seed=seed, B=rows)
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    t0 = time.perf_counter()
    oracle.pwa_fwd(f["v"], f["bias"], f["keep"], f.get("g"))
    oracle.pwa_bwd(f["v"], f["bias"], f["keep"], f.get("g"), f["dout"])
    el = time.perf_counter() - t0
    w = pwa_work(cfg, B=rows)
    threads = oracle.threads()
    return {"value": (w["fwd_flops"] + w["bwd_flops"]) / el / 1e12, "unit": "TFLOP/s",
            "cores": min(threads, cfg.H), "kind": "oracle",
            "sample": "%s pair-weighted averaging fwd+bwd on %d of %d broadcast rows, %.1f s; fp64 C "
                      "loops, OpenMP over the %d heads (%d threads available)"
                      % (cfg.name, rows, cfg.B, el, cfg.H, threads),
            "seconds": el, "rows": rows}


def run_pwa(args, cfg):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    import numpy as np
    import pair_biased_attention_gated_b200 as pba
    d = pi.make_inputs(cfg, seed=args.seed)
    host = {}
    for k in ("v", "bias", "keep", "g", "dout"):
        if k not in d:
            continue
        a = d[k]
        t = torch.from_numpy(np.ascontiguousarray(a)) if k == "keep" else \
            torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        host[k] = t.pin_memory()
    dev = {k: v.cuda() for k, v in host.items()}
    v, bias, keep, g, dout = dev["v"], dev["bias"], dev["keep"], dev.get("g"), dev["dout"]
    B, N, H, C = v.shape
    out = torch.empty_like(v)
    lse = torch.empty(H, N, dtype=torch.float32, device="cuda")
    dv = torch.empty_like(v)
    dg = torch.empty_like(g) if g is not None else None
    db = torch.empty(H, N, N, dtype=torch.float32, device="cuda")
    dims = pba.pwa_dims(v, g, out, bias, keep)
    wsf = torch.empty(int(pba.lib.pba_pwa_fwd_workspace_size(ctypes.byref(dims))), dtype=torch.uint8, device="cuda")
    wsb = torch.empty(int(pba.lib.pba_pwa_bwd_workspace_size(ctypes.byref(dims))), dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        pba.pba_pwa_fwd(v, bias, keep, g, out, lse, wsf)
        pba.pba_pwa_bwd(v, bias, keep, g, out, dout, dv, db, dg, wsb)

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step()
    pba.pba_device_status()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(physical_gpu_index(local))
    torch.cuda.synchronize()
    pba.profile_read()
    pba.profile_enable(True)
    sampler.start()
    for i in range(K):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    pba.profile_enable(False)
    kstats = pba.profile_read()
    pba.pba_device_status()
    elapsed_ms = sum(a.elapsed_time(b) for a, b in ev)
    # end to end: host buffers, copies inside the events
    houts = {"out": out, "lse": lse, "dv": dv, "db": db}
    if dg is not None:
        houts["dg"] = dg
    hbufs = {k: torch.empty(t.shape, dtype=t.dtype).pin_memory() for k, t in houts.items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in hbufs.values())
    K2 = max(1, min(K, 20))
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K2)]
    torch.cuda.synchronize()
    for i in range(K2):
        flush.fill_(i & 0xFF)
        ev2[i][0].record(stream)
        for k2, t in host.items():
            dev[k2].copy_(t, non_blocking=True)
        step()
        for k2, t in hbufs.items():
            t.copy_(houts[k2], non_blocking=True)
        ev2[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in ev2)
    pba.pba_device_status()

    w = pwa_work(cfg)
    step_flops = w["fwd_flops"] + w["bwd_flops"]
    value = step_flops * K / (elapsed_ms / 1e3) / 1e12
    peaks, peak_src = load_peaks()
    hbm, tens, _ = peak_rates(peaks)
    total_k = sum(ms for _, ms in kstats.values()) or 1.0
    dom = max(kstats.items(), key=lambda kv: kv[1][1])[0] if kstats else None
    roof = None
    if dom:
        launches, ms = kstats[dom]
        avg_s = ms / launches / 1e3
        kf, kb = w["kernels"].get(dom, (0, 0))
        if kf / (tens * 1e12) > kb / (hbm * 1e9):
            achieved, peak, unit, bound = kf / avg_s / 1e12, tens, "TFLOP/s", "tensor"
        else:
            achieved, peak, unit, bound = kb / avg_s / 1e9, hbm, "GB/s", "hbm"
        roof = {"kernel": dom, "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                "frac": round(achieved / peak, 4),
                "peak_source": "%s (%s)" % (peak_src, "burst bf16" if bound == "tensor" else "copy"),
                "algorithmic_per_launch": {"flops": kf, "bytes": kb}, "avg_launch_us": round(avg_s * 1e6, 2),
                "traffic": ncu_traffic(dom, "pwa-" + cfg.name), "nominal": nominal(achieved, bound)}
    ms_per_step = elapsed_ms / K
    t_step_roof = max(step_flops / (tens * 1e12), (w["fwd_bytes"] + w["bwd_bytes"]) / (hbm * 1e9))
    kernels = {n: {"launches": l, "avg_us": round(ms / l * 1e3, 2), "share": round(ms / total_k, 4)}
               for n, (l, ms) in sorted(kstats.items(), key=lambda kv: -kv[1][1])}
    res = {
        "metric": PWA_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 v/gate/dout, N(0,%g^2) bias, shapes of the named workload"
                % cfg.bias_std,
        "config": {"workload": "%s: %s (pair-weighted averaging of its value rows)" % (cfg.name, cfg.desc),
                   "B": cfg.B, "H": cfg.H, "N": cfg.N, "c": cfg.c, "masked_keys": cfg.N - cfg.n_valid_keys,
                   "gate": cfg.gate, "passes": "fwd+bwd (dv, dgate, dbias)",
                   "l2": "flushed before every timed step (256 MiB write outside the events)",
                   "parallelism": "single GPU"},
        "roofline": roof,
        "step_roofline": {"time_us": round(t_step_roof * 1e6, 2), "frac": round(t_step_roof * 1e3 / ms_per_step, 4)},
        "kernels": kernels, "gpu_launches": sum(l for l, _ in kstats.values()), "clocks": clocks,
        "e2e": {"value": round(step_flops * K2 / (e2e_ms / 1e3) / 1e12, 4), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K2},
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = time_pwa_oracle(cfg, target_s=args.cpu_seconds, seed=args.seed)
    return res if rank == 0 else None

# ---------------------------------------------------------------------------------------
# pair-bias projection (--op pairbias): LayerNorm(z) -> linear -> bias, and its backward
# ---------------------------------------------------------------------------------------
PB_METRIC = "pair-bias projection (LayerNorm + linear) fwd+bwd GB/s and %roofline on 1 B200"


def pb_work(N, Cz, H, Ni=None):
    """Algorithmic bytes: forward reads z and writes the bf16 bias; backward reads z and the
    fp32 dbias and writes dz (parameters and their gradients are a few KB)."""
    Ni = N if Ni is None else Ni
    P = Ni * N
    fwd = P * Cz * 2 + H * P * 2
    bwd = P * Cz * 2 + H * P * 4 + P * Cz * 2
    return {"fwd_bytes": fwd, "bwd_bytes": bwd,
            "kernels": {"pba_pair_bias_fwd_kernel": (0, fwd), "pba_pair_bias_bwd_kernel": (0, bwd),
                        "pba_pair_bias_bwd_tc_kernel": (0, bwd),   # the backward at Cz = 128
                        "pba_pair_bias_reduce_kernel": (0, 0), "pba_pair_bias_param_kernel": (0, 0)}}


def time_pb_oracle(N, Cz, H, target_s, seed):
    import oracle
    rows = 1
    for _ in range(2):
        d = pi.make_pair_bias_inputs(rows, N, Cz, H, seed)
        z = pi.bf16_bits_to_f64(d["z"])
        args = [d[k].astype(np.float64) for k in ("gamma", "beta", "w")]
        t0 = time.perf_counter()
        oracle.pair_bias_fwd(z, *args)
        oracle.pair_bias_bwd(z, *args, d["dbias"].astype(np.float64))
        el = time.perf_counter() - t0
        if el >= target_s or rows >= N:
            break
        rows = int(max(1, min(N, rows * target_s / max(el, 1e-6))))
    w = pb_work(N, Cz, H, Ni=rows)
    return {"value": (w["fwd_bytes"] + w["bwd_bytes"]) / el / 1e9, "unit": "GB/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": "pair-bias projection fwd+bwd on %d of %d rows i (x %d positions j, Cz=%d, H=%d), %.1f s; "
                      "fp64 C loops, the forward over OpenMP threads, the backward on one (its sums run in one fixed order)"
                      % (rows, N, N, Cz, H, el),
            "seconds": el, "rows": rows}


def run_pairbias(args, cfg):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    import pair_biased_attention_gated_b200 as pba
    N, H, Cz = cfg.N, cfg.H, pi.CZ_PAIR
    d = pi.make_pair_bias_inputs(N, N, Cz, H, seed=args.seed)
    host = {"z": torch.from_numpy(d["z"].view(np.int16)).view(torch.bfloat16).pin_memory()}
    for k in ("gamma", "beta", "w", "dbias"):
        host[k] = torch.from_numpy(d[k]).pin_memory()
    dev = {k: v.cuda() for k, v in host.items()}
    bias = torch.empty((H, N, N), dtype=torch.bfloat16, device="cuda")
    dz = torch.empty_like(dev["z"])
    dw = torch.empty((Cz, H), dtype=torch.float32, device="cuda")
    dg = torch.empty(Cz, dtype=torch.float32, device="cuda")
    db = torch.empty(Cz, dtype=torch.float32, device="cuda")
    dims = pba.pair_bias_dims(dev["z"], dbias=dev["dbias"])
    ws = torch.empty(max(int(pba.lib.pba_pair_bias_bwd_workspace_size(ctypes.byref(dims))), 256),
                     dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        pba.pba_pair_bias_fwd(dev["z"], dev["gamma"], dev["beta"], dev["w"], bias)
        pba.pba_pair_bias_bwd(dev["z"], dev["gamma"], dev["beta"], dev["w"], dev["dbias"], dz, dw, dg, db, ws)

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step()
    pba.pba_device_status()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(physical_gpu_index(local))
    torch.cuda.synchronize()
    pba.profile_read()
    pba.profile_enable(True)
    sampler.start()
    for i in range(K):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    pba.profile_enable(False)
    kstats = pba.profile_read()
    pba.pba_device_status()
    elapsed_ms = sum(a.elapsed_time(b) for a, b in ev)
    houts = {"bias": bias, "dz": dz, "dw": dw, "dg": dg, "db": db}
    hbufs = {k: torch.empty(t.shape, dtype=t.dtype).pin_memory() for k, t in houts.items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in hbufs.values())
    K2 = max(1, min(K, 20))
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K2)]
    torch.cuda.synchronize()
    for i in range(K2):
        flush.fill_(i & 0xFF)
        ev2[i][0].record(stream)
        for k2, t in host.items():
            dev[k2].copy_(t, non_blocking=True)
        step()
        for k2, t in hbufs.items():
            t.copy_(houts[k2], non_blocking=True)
        ev2[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in ev2)
    pba.pba_device_status()

    w = pb_work(N, Cz, H)
    step_bytes = w["fwd_bytes"] + w["bwd_bytes"]
    value = step_bytes * K / (elapsed_ms / 1e3) / 1e9
    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    total_k = sum(ms for _, ms in kstats.values()) or 1.0
    dom = max(kstats.items(), key=lambda kv: kv[1][1])[0] if kstats else None
    roof = None
    if dom:
        launches, ms = kstats[dom]
        avg_s = ms / launches / 1e3
        kb = w["kernels"].get(dom, (0, 0))[1]
        achieved = kb / avg_s / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 2), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_source": "%s (copy)" % peak_src,
                "algorithmic_per_launch": {"flops": 0, "bytes": kb}, "avg_launch_us": round(avg_s * 1e6, 2),
                "traffic": ncu_traffic(dom, "pairbias-" + cfg.name), "nominal": nominal(achieved, "hbm")}
    ms_per_step = elapsed_ms / K
    kernels = {n: {"launches": l, "avg_us": round(ms / l * 1e3, 2), "share": round(ms / total_k, 4)}
               for n, (l, ms) in sorted(kstats.items(), key=lambda kv: -kv[1][1])}
    res = {
        "metric": PB_METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded bf16 z (N(0,1) channels, per-position offset and scale), fp32 "
                "LayerNorm and projection parameters and dbias",
        "config": {"workload": "%s pair representation: z [%d, %d, %d] -> bias [%d, %d, %d]" % (cfg.name, N, N, Cz, H, N, N),
                   "N": N, "Cz": Cz, "H": H, "passes": "fwd (bias) + bwd (dz, dw, dgamma, dbeta)",
                   "l2": "flushed before every timed step (256 MiB write outside the events)",
                   "parallelism": "single GPU"},
        "roofline": roof,
        "step_roofline": {"time_us": round(step_bytes / (hbm * 1e9) * 1e6, 2),
                          "frac": round(step_bytes / (hbm * 1e9) * 1e3 / ms_per_step, 4)},
        "kernels": kernels, "gpu_launches": sum(l for l, _ in kstats.values()), "clocks": clocks,
        "e2e": {"value": round(step_bytes * K2 / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K2},
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = time_pb_oracle(N, Cz, H, args.cpu_seconds, args.seed)
    return res if rank == 0 else None


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="C5", choices=sorted(pi.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--also", default="C1,C2,C3,C4",
                    help="other workloads whose per-pass device times and roofline fractions are "
                         "added under `workloads` (one GPU; empty: none)")
    ap.add_argument("--op", default="attention", choices=["attention", "pwa", "pairbias"],
                    help="pwa: MSA pair-weighted averaging of the workload's value rows; pairbias: "
                         "the LayerNorm + projection that makes the workload's bias (one GPU each)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = pi.CONFIGS[args.config]
    if args.op != "attention":
        if args.impl == "reference" or args.gpus != 1:
            ap.error("--op %s times our kernels on one GPU; its oracle baseline is the cpu_baseline key" % args.op)
        res = run_pwa(args, cfg) if args.op == "pwa" else run_pairbias(args, cfg)
    else:
        res = run_reference(args, cfg) if args.impl == "reference" else run_ours(args, cfg)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
