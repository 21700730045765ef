"""Row-sharded pair-biased attention across GPUs: one process per GPU, torch.distributed.

The Design-CP page ("Context Parallelism for Design of Protein Nanoparticles", Method)
shards every attention block's rows over the GPUs and exchanges activations only between
blocks.  For pair-biased attention the rows are the broadcast rows b (triangle rows, MSA
sequences, diffusion copies): the forward pass and dq, dk, dv, dgate are computed row by
row, so a rank computes its own rows with no exchange.  The bias gradient is the sum of
the logits' gradient over all rows ("AlphaFold3 open-source implementation" page, Model
Efficiency section), so after the backward pass every rank holds part of it: that sum is
the one exchange step.

Deterministic reduction.  The rows are cut into `groups` contiguous row groups, a number
fixed by the caller and independent of the world size; rank r of W owns the groups
[r G / W, (r + 1) G / W).  A rank runs the backward pass once per group it owns (each call
yields that group's bias gradient), the ranks all-gather these partials, and every rank
adds them in group order with pba_dbias_sum.  The result therefore depends on the groups
alone: it is the same on every rank and bit-identical for every world size that divides
G (one GPU included).

The backward call per group and the ordered sum are parameters (`bwd_group`, `sum_parts`)
so that the sharding and the exchange can be exercised without a GPU; their defaults are
the library's kernels.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple


def row_groups(B: int, groups: int) -> List[Tuple[int, int]]:
    """The `groups` contiguous row ranges [lo, hi) that cover rows 0..B-1, as equal as
    possible (the first B % groups groups one row longer)."""
    if groups < 1:
        raise ValueError("groups must be >= 1")
    base, extra = divmod(B, groups)
    out, lo = [], 0
    for g in range(groups):
        hi = lo + base + (1 if g < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def rank_groups(groups: int, world: int, rank: int) -> range:
    """Indices of the row groups rank `rank` of `world` owns."""
    if groups % world != 0:
        raise ValueError("the group count (%d) must be a multiple of the world size (%d)" % (groups, world))
    per = groups // world
    return range(rank * per, (rank + 1) * per)


def rank_rows(B: int, groups: int, world: int, rank: int) -> Tuple[int, int]:
    """The rows [lo, hi) of rank `rank`: the union of its row groups."""
    gs = row_groups(B, groups)
    mine = rank_groups(groups, world, rank)
    return gs[mine.start][0], gs[mine.stop - 1][1]


def _library_bwd_group(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dgate, dbias, ws):
    from . import pba_bwd
    pba_bwd(q, k, v, bias, key_mask, gate, out, lse, dout, dq, dk, dv, dbias, dgate, ws)


def _library_sum_parts(parts, out):
    import ctypes

    import torch

    from . import _check, lib
    G = parts.shape[0]
    n = out.numel()
    _check(lib.pba_dbias_sum(ctypes.c_void_p(parts.data_ptr()), G, ctypes.c_int64(n),
                             ctypes.c_void_p(out.data_ptr()),
                             ctypes.c_void_p(torch.cuda.current_stream(out.device).cuda_stream)))


def local_backward(q, k, v, bias, key_mask, gate, out, lse, dout, *, B_total: int, groups: int,
                   world: int = 1, rank: int = 0, bwd_group: Optional[Callable] = None,
                   workspace=None):
    """This rank's part of the sharded backward pass, before any exchange: (dq, dk, dv,
    dgate) of its rows and the bias-gradient partial of each of its row groups, stacked
    [groups of the rank, H, Nq, Nk] fp32 in group order.  Inputs as in sharded_backward."""
    import torch
    bwd_group = bwd_group or _library_bwd_group
    lo, hi = rank_rows(B_total, groups, world, rank)
    if q.shape[0] != hi - lo:
        raise ValueError("this rank holds %d rows, its share is %d" % (q.shape[0], hi - lo))
    H, Nq, Nk = q.shape[2], q.shape[1], k.shape[1]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dgate = torch.empty_like(gate) if gate is not None else None
    mine = rank_groups(groups, world, rank)
    gs = row_groups(B_total, groups)
    local = torch.empty((len(mine), H, Nq, Nk), dtype=torch.float32, device=q.device)
    per_row_mask = key_mask is not None and key_mask.dim() == 2
    for x, g in enumerate(mine):
        a, b = gs[g][0] - lo, gs[g][1] - lo
        if a == b:
            local[x].zero_()   # an empty group adds nothing
            continue
        sl = lambda t: None if t is None else t[a:b]
        bwd_group(sl(q), sl(k), sl(v), bias, sl(key_mask) if per_row_mask else key_mask, sl(gate),
                  sl(out), sl(lse), sl(dout), sl(dq), sl(dk), sl(dv), sl(dgate), local[x], workspace)
    return dq, dk, dv, dgate, local


def sum_partials(parts, sum_parts: Optional[Callable] = None):
    """The bias gradient from every group's partial, stacked in group order: their sum in
    that order (pba_dbias_sum by default)."""
    import torch
    sum_parts = sum_parts or _library_sum_parts
    dbias = torch.empty(parts.shape[1:], dtype=torch.float32, device=parts.device)
    sum_parts(parts.contiguous(), dbias)
    return dbias


def sharded_backward(q, k, v, bias, key_mask, gate, out, lse, dout, *, B_total: int,
                     groups: int, pg=None, world: int = 1, rank: int = 0,
                     bwd_group: Optional[Callable] = None, sum_parts: Optional[Callable] = None,
                     workspace=None):
    """Backward pass of this rank's rows with the bias gradient summed over all ranks.

    q, gate, out, dout, lse and k, v hold this rank's rows only (rows rank_rows(B_total,
    groups, world, rank) of the whole batch, in order; a per-row key mask likewise); bias
    [H, Nq, Nk] is the shared pair bias.  Returns (dq, dk, dv, dgate, dbias): the first
    four for this rank's rows, dbias [H, Nq, Nk] fp32 for all rows, identical on every
    rank.  `pg` is torch.distributed (or None with world = 1); the exchange is one
    all-gather of the partials (NCCL between GPUs).
    """
    import torch
    if pg is not None:
        world, rank = pg.get_world_size(), pg.get_rank()
    elif world > 1:
        raise ValueError("a process group is needed for world > 1")
    dq, dk, dv, dgate, local = local_backward(q, k, v, bias, key_mask, gate, out, lse, dout,
                                              B_total=B_total, groups=groups, world=world,
                                              rank=rank, bwd_group=bwd_group, workspace=workspace)
    if world > 1:
        gathered = [torch.empty_like(local) for _ in range(world)]
        pg.all_gather(gathered, local)
        parts = torch.cat(gathered, dim=0)   # rank order = group order
    else:
        parts = local
    return dq, dk, dv, dgate, sum_partials(parts, sum_parts)


def workspace_for(q, k, v, gate, out, bias, key_mask, B_total: int, groups: int,
                  world: int = 1, rank: int = 0):
    """One backward workspace large enough for every row group of this rank."""
    import torch

    from . import make_dims, pba_bwd_workspace_size
    gs = row_groups(B_total, groups)
    rows = max((gs[g][1] - gs[g][0] for g in rank_groups(groups, world, rank)), default=0)
    if rows == 0:
        return torch.empty(256, dtype=torch.uint8, device=q.device)
    sl = lambda t: None if t is None else t[:rows]
    d = make_dims(sl(q), sl(k), sl(v), sl(gate), sl(out), bias, sl(key_mask) if (key_mask is not None and key_mask.dim() == 2) else key_mask)
    return torch.empty(max(pba_bwd_workspace_size(d), 256), dtype=torch.uint8, device=q.device)
