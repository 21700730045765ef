"""Seeded synthetic inputs for pair-biased gated attention.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It only draws random numbers and rounds them to bf16; it holds none
of the attention arithmetic.

Workload shapes follow the pages' workloads: MSA row attention with a pair bias
shared over all MSA rows, triangle attention where the pair representation's
rows form the broadcast axis, and the diffusion AttentionPairBias with 48
noise-level copies folded into the batch ("AlphaFold3 open-source
implementation", Model Efficiency section).

Layouts (the library's native ones):
  q, k, v, g, dout : [B, N, H, c]   (c innermost)
  bias             : [H, N, N]      (key index innermost)
  keep             : [N] uint8 (shared over B; 1 = key attended, 0 = masked)
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import numpy as np

# Stream ids: one independent generator stream per tensor.
STREAM = {"q": 1, "k": 2, "v": 3, "g": 4, "bias": 5, "dout": 6}


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int            # broadcast rows (triangle rows / MSA sequences / diffusion copies)
    H: int
    N: int            # queries = keys
    c: int            # head dim (true, unpadded)
    bias_std: float
    masked: Tuple[Tuple[int, int], ...]   # half-open key ranges that are masked out
    passes: str       # "fwd" or "fwdbwd": which passes the workload names
    gate: bool = True
    desc: str = ""
    window: int = -1  # local attention: query tile t sees key tiles [t - window, t + window]

    def keep(self) -> np.ndarray:
        keep = np.ones(self.N, dtype=np.uint8)
        for lo, hi in self.masked:
            keep[lo:hi] = 0
        return keep

    @property
    def n_valid_keys(self) -> int:
        return int(self.keep().sum())


CONFIGS: Dict[str, Config] = {
    "C1": Config("C1", B=64, H=4, N=64, c=32, bias_std=1.0, masked=((58, 64),),
                 passes="fwdbwd",
                 desc="tiny triangle attention: 64 rows x 64 keys, last 6 keys masked"),
    "C2": Config("C2", B=128, H=8, N=256, c=32, bias_std=1.0, masked=((243, 256),),
                 passes="fwd",
                 desc="MSA row attention with pair bias: 128 MSA rows, 256 residues, "
                      "~5% tail padding masked"),
    "C3": Config("C3", B=384, H=4, N=384, c=32, bias_std=1.0, masked=((346, 384),),
                 passes="fwdbwd",
                 desc="triangle attention (starting node): 384 rows x 384 keys, "
                      "10% tail keys masked"),
    "C4": Config("C4", B=48, H=16, N=384, c=24, bias_std=0.5, masked=(),
                 passes="fwd",
                 desc="diffusion AttentionPairBias: 48 noise-level copies, 384 tokens, "
                      "c=24, no mask"),
    "C5": Config("C5", B=768, H=4, N=768, c=32, bias_std=1.0,
                 masked=((160, 198), (448, 486), (729, 768)), passes="fwdbwd",
                 desc="large triangle attention: 768 rows x 768 keys, 15% keys masked in "
                      "three contiguous padding blocks"),
    "C6": Config("C6", B=48, H=4, N=3072, c=32, bias_std=1.0, masked=((3040, 3072),),
                 passes="fwdbwd", window=1,
                 desc="sequence-local atom attention of the diffusion module: 48 noise-level "
                      "copies, 3072 atoms, 4 heads, each 128-atom query tile sees the key tiles "
                      "within one tile of it (block-sparse), last 32 atoms padding"),
}


def window_pair_mask(Nq: int, Nk: int, window: int) -> np.ndarray:
    """[Nq, Nk] bool: True where query i may attend key j under a tile window (query tile
    i // 128 sees key tiles within `window` of it; window < 0: every pair)."""
    if window < 0:
        return np.ones((Nq, Nk), dtype=bool)
    ti = np.arange(Nq)[:, None] // 128
    tj = np.arange(Nk)[None, :] // 128
    return np.abs(ti - tj) <= window


def custom(name: str, B: int, H: int, N: int, c: int, bias_std: float = 1.0,
           masked=(), gate: bool = True, window: int = -1) -> Config:
    return Config(name, B=B, H=H, N=N, c=c, bias_std=bias_std, masked=tuple(masked),
                  passes="fwdbwd", gate=gate, window=window)


# ----------------------------------------------------------------------------------------
# bf16 helpers (bit patterns held in uint16)
# ----------------------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, round-to-nearest-even; returns uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding_bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding_bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(u: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(u).astype(np.float64)


def normal_bf16(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng([seed, stream])
    x = rng.standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x).reshape(shape)


def make_inputs(cfg: Config, seed: int = 0, with_dout: bool = True,
                B: Optional[int] = None) -> Dict[str, np.ndarray]:
    """bf16 bit patterns for every input of one configuration.

    `B` overrides the number of broadcast rows (used to draw a bounded sample of a
    workload); rows 0..B-1 are identical to the full draw's first rows only for
    the bias and mask, which do not depend on B.
    """
    B = cfg.B if B is None else B
    N, H, c = cfg.N, cfg.H, cfg.c
    d = {
        "q": normal_bf16(seed, STREAM["q"], (B, N, H, c)),
        "k": normal_bf16(seed, STREAM["k"], (B, N, H, c)),
        "v": normal_bf16(seed, STREAM["v"], (B, N, H, c)),
        "bias": normal_bf16(seed, STREAM["bias"], (H, N, N), cfg.bias_std),
        "keep": cfg.keep(),
    }
    if cfg.gate:
        d["g"] = normal_bf16(seed, STREAM["g"], (B, N, H, c))
    if with_dout:
        d["dout"] = normal_bf16(seed, STREAM["dout"], (B, N, H, c))
    return d


# ----------------------------------------------------------------------------------------
# pair-bias projection inputs (pair representation and LayerNorm / projection parameters)
# ----------------------------------------------------------------------------------------

PAIR_STREAM = {"z": 11, "zshift": 12, "zscale": 13, "gamma": 14, "beta": 15, "w": 16, "dbias": 17}
CZ_PAIR = 128   # channels of the pair representation in the AlphaFold3 family


def make_pair_bias_inputs(Ni: int, Nj: int, Cz: int, H: int, seed: int = 0) -> Dict[str, np.ndarray]:
    """z as bf16 bits [Ni, Nj, Cz]: N(0, 1) channels with a per-position offset N(0, 1) and
    scale U(0.5, 2) (so that the normalisation has work to do); gamma ~ 1 + N(0, 0.1^2),
    beta ~ N(0, 0.1^2), w ~ N(0, 1/Cz) [Cz, H] and dbias ~ N(0, 1) [H, Ni, Nj], all fp32."""
    def rng(name):
        return np.random.default_rng([seed, PAIR_STREAM[name]])
    x = rng("z").standard_normal((Ni, Nj, Cz), dtype=np.float32)
    shift = rng("zshift").standard_normal((Ni, Nj, 1), dtype=np.float32)
    scale = rng("zscale").uniform(0.5, 2.0, (Ni, Nj, 1)).astype(np.float32)
    z = f32_to_bf16_bits(x * scale + shift).reshape(Ni, Nj, Cz)
    return {
        "z": z,
        "gamma": (1.0 + 0.1 * rng("gamma").standard_normal(Cz)).astype(np.float32),
        "beta": (0.1 * rng("beta").standard_normal(Cz)).astype(np.float32),
        "w": (rng("w").standard_normal((Cz, H)) / np.sqrt(Cz)).astype(np.float32),
        "dbias": rng("dbias").standard_normal((H, Ni, Nj), dtype=np.float32),
    }
