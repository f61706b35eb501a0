"""Tensor-core path coverage: which kernel runs, and parity of the tcgen05
kernels across their shape classes (MMA N = padded S*rs of 16..256, rank
paddings 16/32/64 in the expand, split-K cluster sizes 1..16, grouped and
direct schedules, bf16 and fp16).  Same bar as test_parity_gpu.py."""
import numpy as np
import pytest

from scatter_gemm_b200 import lora
from scatter_gemm_b200.workloads import make_problem
from tests.test_parity_gpu import check_expand, check_shrink

pytestmark = pytest.mark.gpu

T, G, GEN, SPLIT = lora.PATH_TENSOR, lora.PATH_GROUPED, lora.PATH_GENERAL, lora.PATH_SPLITK


def test_aligned_inputs_take_the_tensor_core_path():
    p = make_problem("qkv", seed=20, tok=256, K=512)
    check_shrink(p)
    assert lora.last_path() & T
    check_expand(p)
    assert lora.last_path() & T


def test_misaligned_inputs_take_the_tensor_core_path_too():
    # element-aligned rows are staged and shifted for the tensor cores
    p = make_problem("tail", seed=21, tok=100)
    check_shrink(p)
    assert lora.last_path() & T
    check_expand(p)
    assert lora.last_path() & T


# element-aligned expand: pointer offsets, odd leading dimensions, odd slice
# starts and widths, odd ranks of every padding class, grouped schedule
@pytest.mark.parametrize("mis", [1, 2, 3, 5, 7])
def test_expand_element_aligned_offsets(mis):
    p = make_problem("qkv", seed=50 + mis, tok=300, K=64, slices=[200 + mis, 131, 67],
                     r=13, rs=16, misalign=mis, ld_pad=mis, col_lead=mis)
    check_expand(p)
    assert lora.last_path() & T


@pytest.mark.parametrize("r,rs", [(5, 7), (16, 16), (29, 33), (64, 64)])
def test_expand_element_aligned_ranks(r, rs):
    p = make_problem("qkv", seed=60 + r, tok=257, K=64, slices=[129, 7, 260], r=r, rs=rs,
                     misalign=1, ld_pad=3, col_lead=1)
    check_expand(p)
    assert lora.last_path() & T


@pytest.mark.parametrize("slices", [[300, 41], [64, 64, 64, 64]])
def test_expand_element_aligned_rank64_slice_counts(slices):
    # rank 64: one slice's staged rank rows fill the last stage's base area, the
    # others go to the B staging areas (two slices) or also stage 0's (S > 3 is
    # refused by the tensor path and runs on the CUDA cores)
    p = make_problem("qkv", seed=65, tok=200, K=64, slices=slices, r=64, rs=64,
                     misalign=1, ld_pad=3, col_lead=1)
    check_expand(p)
    if len(slices) <= 3:
        assert lora.last_path() & T


def test_expand_element_aligned_rank64_three_slices_grouped():
    # rank 64, three slices (the last slice's staged rank rows in stage 0, the
    # first B tile after them) on the grouped schedule
    p = make_problem("many_small", seed=66, tok=900, nseg=120, K=64, slices=[200, 72, 72],
                     r=64, rs=64, misalign=1)
    check_expand(p, workspace=True)
    assert lora.last_path() & G and lora.last_path() & T


def test_expand_element_aligned_grouped_zero_scaling_and_lead_trail():
    p = make_problem("many_small", seed=70, tok=900, nseg=120, K=64, slices=[250, 70, 70],
                     misalign=3, lead=9, trail=4, col_lead=5)
    sc = p.scalings.copy()
    sc[::3] = 0.0
    check_expand(p, workspace=True, scalings=sc)
    assert lora.last_path() & G and lora.last_path() & T


# element-aligned shrink: every pointer offset (elements past a 16-byte
# boundary), odd K and leading dimensions, odd ranks, split-K and grouped
@pytest.mark.parametrize("mis", [1, 2, 3, 4, 5, 6, 7])
def test_shrink_element_aligned_offsets(mis):
    p = make_problem("qkv", seed=30 + mis, tok=300, K=1000 + mis, slices=[64, 32, 32],
                     r=13, rs=16, misalign=mis, ld_pad=mis)
    check_shrink(p)
    assert lora.last_path() & T


@pytest.mark.parametrize("K", [1, 7, 63, 65, 129, 3583])
def test_shrink_element_aligned_k_tails(K):
    p = make_problem("qkv", seed=40, tok=150, K=K, slices=[64, 64], r=8, rs=8, misalign=1)
    check_shrink(p)
    assert lora.last_path() & T


def test_shrink_element_aligned_grouped_and_split():
    p = make_problem("many_small", seed=41, tok=900, nseg=120, K=777, slices=[256, 64, 64],
                     misalign=3)
    check_shrink(p, workspace=True)
    assert lora.last_path() & G and lora.last_path() & T
    p = make_problem("qkv", seed=42, tok=40, K=4093, misalign=5)
    check_shrink(p)
    assert lora.last_path() & T and lora.last_path() & SPLIT


def test_many_segments_with_workspace_are_grouped():
    p = make_problem("many_small", seed=22, tok=900, nseg=120, K=512, slices=[512, 128, 128])
    check_shrink(p, workspace=True)
    assert lora.last_path() & G and lora.last_path() & T
    check_expand(p, workspace=True)
    assert lora.last_path() & G and lora.last_path() & T
    check_shrink(p, workspace=False)
    assert not lora.last_path() & G


def test_grouping_skipped_when_it_saves_little():
    # 3 segments of 2 adapters, K = 512, rank 8: one extra piece saves 8 KB of
    # weight reads, under the grouping pass's 64 KB threshold, so a workspace
    # is left unused and the result is still the oracle's
    p = make_problem("tiny", seed=77)
    assert p.nseg > p.L
    check_shrink(p, workspace=True)
    assert lora.last_path() & T and not lora.last_path() & G
    check_expand(p, workspace=True)
    assert lora.last_path() & T and not lora.last_path() & G


@pytest.mark.parametrize("L,nseg,tok,K", [(8, 20, 2000, 192), (300, 400, 1200, 192),
                                           (16, 2100, 30000, 64)])
def test_grouping_long_segments_and_many_adapters(L, nseg, tok, K):
    # random segment lengths with repeated adapters: few segments (the pass
    # with block-wide counters); more adapters than the per-warp counters hold;
    # and over 2,048 segments (the per-warp pass), some longer than 64 rows
    # (listed by whole warps)
    p = make_problem("qkv", seed=24 + L, tok=tok, K=K, slices=[128, 64, 64], L=L, nseg=nseg,
                     recipe="random", lead=3, trail=2)
    assert int((np.diff(p.seg_indptr) > 64).sum()) > 0 or L > 256
    check_shrink(p, workspace=True)
    assert lora.last_path() & G and lora.last_path() & T
    check_expand(p, workspace=True)
    assert lora.last_path() & G and lora.last_path() & T


# beyond the tensor-core kernels' range (rank > 64; shrink S*rs > 256): the
# CUDA-core kernels, aligned and at any element offset
@pytest.mark.parametrize("mis", [0, 1])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_wide_rank_runs_on_the_cuda_cores(mis, dtype):
    p = make_problem("wide_rank", seed=27 + mis, tok=300, K=264, slices=[256, 64, 72], r=100,
                     rs=104, dtype=dtype, misalign=mis, ld_pad=mis, col_lead=mis)
    check_shrink(p)
    assert lora.last_path() & GEN
    check_expand(p)
    assert lora.last_path() & GEN


def test_small_token_counts_split_k_over_a_cluster():
    p = make_problem("qkv", seed=23, tok=50, K=4096)
    check_shrink(p)
    assert lora.last_path() & SPLIT


# shrink shape classes: (S, r, rs) -> MMA N = round_up(S*rs, 16)
@pytest.mark.parametrize("S,r,rs", [(1, 8, 8), (1, 5, 8), (5, 8, 8), (3, 16, 16), (2, 64, 64),
                                    (3, 32, 32), (1, 136, 136), (4, 64, 64), (2, 100, 104)])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_shrink_mma_widths(S, r, rs, dtype):
    slices = [64 + 8 * q for q in range(S)]
    p = make_problem("qkv", seed=24 + S + r, tok=333, K=776, slices=slices, r=r, rs=rs,
                     nseg=6, L=6, recipe="dirichlet", dtype=dtype)
    check_shrink(p)
    assert lora.last_path() & T


@pytest.mark.parametrize("tok,K", [(7, 64), (40, 4096), (300, 128), (1000, 8), (129, 2056),
                                   (2048, 6144)])
def test_shrink_split_k_and_k_tails(tok, K):
    p = make_problem("qkv", seed=25, tok=tok, K=K, slices=[64, 32, 32])
    check_shrink(p)
    assert lora.last_path() & T


# expand rank classes: rpad 16 (r<=16), 32 (r<=32), 64 (r<=64)
@pytest.mark.parametrize("r,rs", [(1, 8), (5, 8), (13, 16), (16, 16), (20, 24), (32, 32),
                                  (40, 40), (64, 64)])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_expand_rank_classes(r, rs, dtype):
    p = make_problem("qkv", seed=26 + r, tok=333, K=64, slices=[1000, 136, 264], r=r, rs=rs,
                     nseg=5, L=7, recipe="dirichlet", dtype=dtype, col_lead=8, ld_pad=8)
    check_expand(p)
    assert lora.last_path() & T


@pytest.mark.parametrize("tok", [1, 64, 129, 777, 4100])
def test_expand_tile_runs_per_cta(tok):
    p = make_problem("gate_up", seed=27, tok=tok, K=64, slices=[2048, 1288], nseg=4, L=4)
    check_expand(p)
    assert lora.last_path() & T


# Segments that start off the 128-row grid add partial pieces; aligned ones
# leave the segment-start slots empty.  Both layouts, at sizes where several
# CTAs share each piece's column tiles.
@pytest.mark.parametrize("tok,recipe", [(2048, "dirichlet"), (6144, "dirichlet"),
                                        (6144, "uniform")])
def test_expand_aligned_and_ragged_segment_layouts(tok, recipe):
    p = make_problem("qkv", seed=30, tok=tok, K=64, nseg=8, L=8, recipe=recipe)
    check_expand(p)
    assert lora.last_path() & T


def test_expand_empty_slice_and_single_column_tiles():
    p = make_problem("qkv", seed=28, tok=200, K=64, slices=[128, 0, 8, 120, 0, 136])
    check_expand(p)
    assert lora.last_path() & T


def test_one_token_per_segment_grouped_and_direct():
    p = make_problem("ones16k", seed=29, tok=3000, nseg=3000, K=512)
    check_shrink(p, workspace=True)
    check_expand(p, workspace=True)
    check_shrink(p, workspace=False)
    check_expand(p, workspace=False)


def test_no_device_side_wait_timed_out():
    assert lora.device_error(clear=True) == 0
