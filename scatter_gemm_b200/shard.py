"""Host-side sharding of one chunked-SGMV batch over several GPUs.

Every token's LoRA update depends only on its own x row and its segment's
adapter (sgl-kernel-xpu page "Decode LoRA kernels are optimized", section
"Summary"), so a batch splits over ranks with no exchange at all: rank k takes
a contiguous range of the SORTED rows, cut so the ranks get equal row counts
(a segment cut in two keeps its adapter on both sides), with its own
re-based tables, and runs lora_shrink / lora_expand on them.  Adapter stacks
are replicated.  Results are the rows of the unsharded call, bit for bit,
because no row's arithmetic changes.

This module only slices tables and arrays (numpy); the bench's multi-GPU mode
runs independent batches per rank (weak scaling) and uses `max_over_ranks`
for its timing.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List

import numpy as np


@dataclass
class Shard:
    rank: int
    row_lo: int              # first sorted row of the batch owned by this rank
    row_hi: int              # one past the last
    tokens: np.ndarray       # original token index of each local row (local row j <-> token tokens[j])
    seg_indptr: np.ndarray   # local tables (rows re-based to 0)
    weight_indices: np.ndarray
    permutation: np.ndarray  # local permutation: identity over the local rows


def split_rows(seg_indptr: np.ndarray, world: int) -> List[int]:
    """Row cut points [r_0, ..., r_world] giving each rank an equal share of
    the rows inside [seg_indptr[0], seg_indptr[-1])."""
    lo, hi = int(seg_indptr[0]), int(seg_indptr[-1])
    n = hi - lo
    return [lo + (n * k) // world for k in range(world + 1)]


def shard_batch(seg_indptr, weight_indices, permutation, rank: int, world: int) -> Shard:
    """Tables of rank `rank` out of `world` for one batch."""
    seg_indptr = np.asarray(seg_indptr, dtype=np.int64)
    weight_indices = np.asarray(weight_indices, dtype=np.int32)
    cuts = split_rows(seg_indptr, world)
    a, b = cuts[rank], cuts[rank + 1]
    starts = np.clip(seg_indptr[:-1], a, b)
    ends = np.clip(seg_indptr[1:], a, b)
    keep = ends > starts
    st, en = starts[keep], ends[keep]
    indptr = np.concatenate([[0], np.cumsum(en - st)]).astype(np.int32)
    return Shard(rank=rank, row_lo=a, row_hi=b,
                 tokens=np.asarray(permutation, dtype=np.int32)[a:b].copy(),
                 seg_indptr=indptr, weight_indices=weight_indices[keep].copy(),
                 permutation=np.arange(b - a, dtype=np.int32))


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the default process group (identity when
    no group is initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
