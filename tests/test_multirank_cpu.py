"""Multi-rank host path on CPU (gloo, world size 2): sharding one batch over
ranks needs no exchange -- the shards' oracle results reassemble into the
unsharded oracle result bit for bit -- and the timing reduction is a max over
ranks."""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from scatter_gemm_b200.shard import max_over_ranks, shard_batch
    from scatter_gemm_b200.workloads import make_problem

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p = make_problem("many_small", seed=5, tok=700, nseg=90, K=96, slices=[64, 16, 16])
        sh = shard_batch(p.seg_indptr, p.weight_indices, p.permutation, rank, world)
        n = sh.row_hi - sh.row_lo
        # the rank's own data: its tokens' x rows, base rows and rank activations
        from scatter_gemm_b200.workloads import Problem
        loc = Problem(name="shard", dtype=p.dtype, tok=n, K=p.K, S=p.S, r=p.r, rs=p.rs,
                      L=p.L, nseg=len(sh.weight_indices), slice_offsets=p.slice_offsets,
                      seg_indptr=sh.seg_indptr, weight_indices=sh.weight_indices,
                      permutation=sh.permutation, scalings=p.scalings,
                      x=p.x[sh.tokens], A=p.A, B=p.B, in_r=p.in_r[sh.row_lo:sh.row_hi],
                      base=p.base[sh.tokens], ld_x=p.ld_x, ld_r=p.ld_r, ld_base=p.ld_base)
        h = oracle.shrink_problem(loc)
        e = oracle.expand_problem(loc)
        parts = [None] * world
        dist.all_gather_object(parts, (sh.row_lo, sh.row_hi, sh.tokens, h, e))
        t = max_over_ranks(float(rank + 1) * 1.5)
        if rank == 0:
            full_h = oracle.shrink_problem(p)
            full_e = oracle.expand_problem(p)
            got_h = np.full_like(full_h, 0x7FFF)
            got_e = p.base.copy()
            for lo, hi, toks, hh, ee in parts:
                got_h[lo:hi] = hh
                got_e[toks] = ee
            q.put((bool(np.array_equal(got_h, full_h)), bool(np.array_equal(got_e, full_e)), t))
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_reassemble_exactly():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=240)
    assert all(pr.exitcode == 0 for pr in procs), [pr.exitcode for pr in procs]
    same_h, same_e, t = q.get(timeout=10)
    assert same_h and same_e
    assert t == 3.0


def test_split_rows_is_a_balanced_partition():
    from scatter_gemm_b200.shard import shard_batch, split_rows
    si = np.array([3, 10, 10, 40, 41, 77], dtype=np.int32)
    wi = np.array([0, 1, 2, 1, 0], dtype=np.int32)
    pm = np.random.default_rng(0).permutation(80).astype(np.int32)
    for world in (1, 2, 3, 5):
        cuts = split_rows(si, world)
        assert cuts[0] == 3 and cuts[-1] == 77
        sizes = np.diff(cuts)
        assert sizes.max() - sizes.min() <= 1
        covered = []
        for k in range(world):
            sh = shard_batch(si, wi, pm, k, world)
            assert sh.seg_indptr[0] == 0 and sh.seg_indptr[-1] == sh.row_hi - sh.row_lo
            # every local row keeps the adapter of its global segment
            for s in range(len(sh.weight_indices)):
                for j in range(sh.seg_indptr[s], sh.seg_indptr[s + 1]):
                    g = sh.row_lo + j
                    gs = int(np.searchsorted(si, g, side="right")) - 1
                    assert wi[gs] == sh.weight_indices[s]
            covered.extend(range(sh.row_lo, sh.row_hi))
        assert covered == list(range(3, 77))
