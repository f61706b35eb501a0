"""Seeded synthetic workloads for the chunked-SGMV LoRA shrink/expand pair.

This module only *builds inputs*: segment tables, permutations and random
bf16/fp16 tensors with the shapes and value distributions of the five
workloads on the sgl-kernel-xpu "Decode LoRA kernels are optimized" page
(section "Performance" and "Testing": token counts 50 ... 8192, K tails, odd
ranks, uneven and unaligned slice starts, misaligned pointers).  It holds none
of the method's arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any computation.

Tensors are returned as numpy ``uint16`` bit patterns (bf16 or fp16); the
caller moves them to the device or hands them to the oracle.  Storage padding
(rank columns ``j >= r`` of A, B and the rank activations) is filled with NaN
so that any read of it shows up in the results.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

DTYPES = ("bf16", "fp16")
NAN_BITS = {"bf16": 0x7FC0, "fp16": 0x7E00}


def to_bits(a: np.ndarray, dtype: str) -> np.ndarray:
    """float32 array -> uint16 bit patterns of bf16/fp16 (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16 if dtype == "bf16" else torch.float16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def from_bits(b: np.ndarray, dtype: str) -> np.ndarray:
    """uint16 bit patterns of bf16/fp16 -> float32 (exact)."""
    t = torch.from_numpy(np.ascontiguousarray(b).view(np.int16))
    t = t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)
    return t.to(torch.float32).numpy()


@dataclass
class Problem:
    """One shrink/expand problem instance (all host numpy arrays).

    Shapes (row-major, leading dimension given separately):
      x            [tok, ld_x]        uint16, valid columns [0, K)
      A            [L, S*rs, K]       uint16, rows q*rs+j with j >= r are NaN
      B            [L, N_tot, rs]     uint16, columns j >= r are NaN
      in_r         [tok, ld_r]        uint16 rank activations in sorted order
                                      (columns q*rs+j, j >= r, are NaN)
      base         [tok, ld_base]     uint16 base projection output
      seg_indptr   [nseg+1] int32,  weight_indices [nseg] int32,
      permutation  [tok] int32,     slice_offsets [S+1] int32,
      scalings     [L] float32
    """

    name: str
    dtype: str
    tok: int
    K: int
    S: int
    r: int
    rs: int
    L: int
    nseg: int
    slice_offsets: np.ndarray
    seg_indptr: np.ndarray
    weight_indices: np.ndarray
    permutation: np.ndarray
    scalings: np.ndarray
    x: np.ndarray
    A: np.ndarray
    B: np.ndarray
    in_r: np.ndarray
    base: np.ndarray
    ld_x: int
    ld_r: int
    ld_base: int
    misalign: int = 0  # elements by which device copies start past a 16-byte boundary
    meta: Dict = field(default_factory=dict)

    @property
    def n_tot(self) -> int:
        return int(self.slice_offsets[-1] - self.slice_offsets[0])

    def rows_used(self) -> int:
        return int(self.seg_indptr[-1] - self.seg_indptr[0])

    def adapters_used(self, nonzero_scaling: bool = False) -> int:
        lens = np.diff(self.seg_indptr)
        ids = self.weight_indices[lens > 0]
        if nonzero_scaling:
            ids = ids[self.scalings[ids] != 0.0]
        return int(np.unique(ids).size)


# --------------------------------------------------------------------------
# segment-length recipes
# --------------------------------------------------------------------------

def _composition(rng, total: int, parts: int) -> np.ndarray:
    """Random composition of `total` into `parts` parts, each >= 1."""
    if parts == 1:
        return np.array([total], dtype=np.int64)
    cuts = np.sort(rng.choice(np.arange(1, total), size=parts - 1, replace=False))
    edges = np.concatenate([[0], cuts, [total]])
    return np.diff(edges)


def _largest_remainder(weights: np.ndarray, total: int) -> np.ndarray:
    raw = weights / weights.sum() * total
    base = np.floor(raw).astype(np.int64)
    short = total - int(base.sum())
    order = np.argsort(-(raw - base), kind="stable")
    base[order[:short]] += 1
    return base


def segment_lengths(rng, recipe: str, tok: int, nseg: int, L: int):
    """Returns (lengths[nseg], adapter ids[nseg])."""
    if recipe == "random":  # random composition, ids drawn from all adapters
        lens = _composition(rng, tok, nseg)
        ids = rng.integers(0, L, size=nseg)
    elif recipe == "uniform":  # one segment per adapter, equal lengths
        lens = np.full(nseg, tok // nseg, dtype=np.int64)
        lens[: tok % nseg] += 1
        ids = rng.permutation(L)[:nseg]
    elif recipe == "dirichlet":  # Dirichlet(1) lengths, zeros allowed
        lens = _largest_remainder(rng.dirichlet(np.ones(nseg)), tok)
        ids = rng.permutation(L)[:nseg]
    elif recipe == "one_empty":  # one segment per adapter, one of them empty
        ids = rng.permutation(L)[:nseg]
        empty = int(rng.integers(0, nseg))
        lens = np.zeros(nseg, dtype=np.int64)
        rest = [s for s in range(nseg) if s != empty]
        lens[rest] = _composition(rng, tok, nseg - 1)
    elif recipe == "many_small":  # 1..16 tokens each, Zipf(1.1) adapter ids
        lens = np.ones(nseg, dtype=np.int64)
        extra = tok - nseg
        while extra > 0:
            elig = np.flatnonzero(lens < 16)
            take = rng.choice(elig, size=min(extra, elig.size), replace=False)
            lens[take] += 1
            extra -= take.size
        p = np.arange(1, L + 1, dtype=np.float64) ** -1.1
        ids = rng.choice(L, size=nseg, p=p / p.sum())
    elif recipe == "ones":  # one token per segment
        lens = np.ones(nseg, dtype=np.int64)
        ids = rng.integers(0, L, size=nseg)
    else:
        raise ValueError(recipe)
    return lens.astype(np.int64), ids.astype(np.int32)


# --------------------------------------------------------------------------
# the five workloads (plus the one-token-per-segment stress case)
# --------------------------------------------------------------------------

CONFIGS: Dict[str, Dict] = {
    # 2 adapters rank 8, one 512-wide slice, 3 random segments of 50 tokens
    "tiny": dict(dtype="bf16", tok=50, K=512, slices=[512], L=2, r=8, rs=8,
                 nseg=3, recipe="random", scaling=2.0),
    # Qwen3-8B-like q/k/v decode: 8 adapters rank 16, one segment per adapter
    "qkv": dict(dtype="bf16", tok=8192, K=4096, slices=[4096, 1024, 1024], L=8,
                r=16, rs=16, nseg=8, recipe="uniform", scaling=2.0),
    # gate_up MLP: 16 adapters rank 64, Dirichlet(1) segment lengths
    "gate_up": dict(dtype="bf16", tok=4096, K=4096, slices=[12288, 12288], L=16,
                    r=64, rs=64, nseg=16, recipe="dirichlet", scaling=2.0),
    # tails and alignment: odd K, odd slice widths/starts, odd rank, 4-byte offset
    "tail": dict(dtype="fp16", tok=777, K=3583, slices=[4097, 1031, 1031], L=5,
                 r=13, rs=16, nseg=5, recipe="one_empty", scaling=2.0, misalign=2),
    # 1024 segments of 1..16 tokens over 64 Zipf-distributed adapters
    "many_small": dict(dtype="bf16", tok=8192, K=5120, slices=[5120, 1024, 1024],
                       L=64, r=32, rs=32, nseg=1024, recipe="many_small",
                       scaling="uniform"),
    # 16,384 tokens, one token per segment (the launch-bound regression case)
    "ones16k": dict(dtype="bf16", tok=16384, K=4096, slices=[4096, 1024, 1024],
                    L=8, r=16, rs=16, nseg=16384, recipe="ones", scaling=2.0),
    # rank 128 on q/k/v slices: beyond the tensor-core kernels' range (rank
    # <= 64, S*rs <= 256), so both ops run on the CUDA-core kernels
    "wide_rank": dict(dtype="bf16", tok=1024, K=4096, slices=[4096, 1024, 1024], L=8,
                      r=128, rs=128, nseg=8, recipe="uniform", scaling=2.0),
}

QKV_TOK_SWEEP = (50, 128, 256, 512, 1024, 2048, 4096, 6144, 8192)


def _normal_bits(rng, shape, std, dtype):
    return to_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std), dtype)


def make_base_weight(p: "Problem", seed: int = 0, ld_pad: int = 0) -> np.ndarray:
    """Seeded base projection weight W [N_tot, K + ld_pad] (uint16 bits) for a
    problem, output-dimension-major like a linear layer's weight, entries
    N(0, 1/K) so that x W^T stays of order one; the ld_pad padding columns hold
    NaN, which no consumer may read."""
    n_tot = int(p.slice_offsets[-1] - p.slice_offsets[0])
    rng = np.random.default_rng([seed, 0x57])
    w = _normal_bits(rng, (n_tot, p.K), 1.0 / np.sqrt(p.K), p.dtype)
    if ld_pad:
        w = np.concatenate([w, np.full((n_tot, ld_pad), NAN_BITS[p.dtype], dtype=np.uint16)],
                           axis=1)
    return np.ascontiguousarray(w)


def make_problem(name: str, seed: int = 0, **over) -> Problem:
    """Builds one seeded instance of workload `name`.

    Overrides (keyword): tok, K, slices, L, r, rs, nseg, dtype, recipe,
    scaling, misalign, lead / trail (rows before/after the segments that no
    call may touch), col_lead (base columns before slice 0), ld_pad (extra
    leading-dimension elements on x, in_r and base).
    """
    cfg = dict(CONFIGS[name])
    cfg.update(over)
    rng = np.random.default_rng(seed)
    dt = cfg["dtype"]
    K, L, r, rs = cfg["K"], cfg["L"], cfg["r"], cfg["rs"]
    slices = list(cfg["slices"])
    S = len(slices)
    lead, trail = int(cfg.get("lead", 0)), int(cfg.get("trail", 0))
    col_lead = int(cfg.get("col_lead", 0))
    ld_pad = int(cfg.get("ld_pad", 0))
    nseg = int(cfg["nseg"])
    tok_seg = int(cfg["tok"])
    if cfg["recipe"] in ("uniform", "dirichlet", "one_empty") and nseg > L:
        nseg = L
    lens, ids = segment_lengths(rng, cfg["recipe"], tok_seg, nseg, L)
    tok = lead + tok_seg + trail
    seg_indptr = (lead + np.concatenate([[0], np.cumsum(lens)])).astype(np.int32)
    permutation = rng.permutation(tok).astype(np.int32)
    off = (col_lead + np.concatenate([[0], np.cumsum(slices)])).astype(np.int32)
    n_tot = int(off[-1] - off[0])
    if cfg["scaling"] == "uniform":
        scalings = rng.uniform(0.5, 4.0, size=L).astype(np.float32)
    else:
        scalings = np.full(L, float(cfg["scaling"]), dtype=np.float32)

    ld_x = K + ld_pad
    ld_r = S * rs + ld_pad
    ld_base = int(off[-1]) + ld_pad
    nan = np.uint16(NAN_BITS[dt])

    x = _normal_bits(rng, (tok, ld_x), 1.0, dt)
    A = _normal_bits(rng, (L, S, rs, K), 0.02, dt)
    A[:, :, r:, :] = nan
    A = A.reshape(L, S * rs, K)
    B = _normal_bits(rng, (L, n_tot, rs), 0.02, dt)
    B[:, :, r:] = nan
    in_r = _normal_bits(rng, (tok, ld_r), 1.0, dt)
    for q in range(S):
        in_r[:, q * rs + r:(q + 1) * rs] = nan
    base = _normal_bits(rng, (tok, ld_base), 1.0, dt)

    return Problem(name=name, dtype=dt, tok=tok, K=K, S=S, r=r, rs=rs, L=L, nseg=nseg,
                   slice_offsets=off, seg_indptr=seg_indptr,
                   weight_indices=ids, permutation=permutation, scalings=scalings,
                   x=x, A=A, B=B, in_r=in_r, base=base, ld_x=ld_x, ld_r=ld_r,
                   ld_base=ld_base, misalign=int(cfg.get("misalign", 0)),
                   meta=dict(cfg, seed=seed))


def bytes_shrink(p: Problem) -> int:
    """Algorithmic bytes of one shrink: gathered x rows + A of the adapters
    used + rank activations written (valid rank r, not the storage stride)."""
    e = 2
    rows = p.rows_used()
    return rows * p.K * e + p.adapters_used() * p.S * p.r * p.K * e + rows * p.S * p.r * e


def bytes_expand(p: Problem) -> int:
    """Algorithmic bytes of one expand: rank activations read + B of the
    adapters used (nonzero scaling) + base output read and written."""
    e = 2
    lens = np.diff(p.seg_indptr)
    live = (lens > 0) & (p.scalings[p.weight_indices] != 0.0)
    rows = int(lens[live].sum())
    return (rows * p.S * p.r * e + p.adapters_used(True) * p.n_tot * p.r * e
            + 2 * rows * p.n_tot * e)


def flops_shrink(p: Problem) -> int:
    return 2 * p.rows_used() * p.K * p.S * p.r


def flops_expand(p: Problem) -> int:
    return 2 * p.rows_used() * p.n_tot * p.r
