"""lora_shrink_expand: the fused decode kernel (one thread-block cluster per
piece runs the split-K shrink, shares the rounded rank activations through
distributed shared memory and runs the expand) and the two-kernel sequence it
uses for larger batches, against the CPU oracle.

The shrink half is checked like lora_shrink (write set exact, values within
|err| <= 2e-2 + 1e-2 |ref|); the expand half against the oracle expand of the
rank activations the call wrote (that is the composition's definition), and
bit for bit against lora_expand given the same activations."""
import numpy as np
import pytest
import torch

import oracle
from scatter_gemm_b200 import lora
from scatter_gemm_b200.workloads import make_problem
from tests.devutil import assert_close

pytestmark = pytest.mark.gpu
SENT = 0x7FFF


def dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(
        torch.bfloat16 if dtype == "bf16" else torch.float16)


def bits_of(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def tabs(p):
    c = lambda a: torch.from_numpy(a.astype(np.int32)).cuda()
    return c(p.seg_indptr), c(p.weight_indices), c(p.permutation)


def fused(p):
    out = dev(np.full((p.tok, p.S * p.rs), SENT, dtype=np.uint16), p.dtype)
    base = dev(p.base, p.dtype)
    si, wi, pm = tabs(p)
    sc = torch.from_numpy(p.scalings.astype(np.float32)).cuda()
    lora.lora_shrink_expand(dev(p.x, p.dtype)[:, : p.K], dev(p.A, p.dtype), dev(p.B, p.dtype),
                            si, wi, pm, [int(v) for v in p.slice_offsets], sc, out, base,
                            rank=p.r)
    torch.cuda.synchronize()
    return bits_of(out), bits_of(base), lora.last_path()


def expand_of(p, in_r_bits):
    base = dev(p.base, p.dtype)
    si, wi, pm = tabs(p)
    sc = torch.from_numpy(p.scalings.astype(np.float32)).cuda()
    lora.lora_expand(dev(in_r_bits, p.dtype), dev(p.B, p.dtype), si, wi, pm,
                     [int(v) for v in p.slice_offsets], sc, base, rank=p.r)
    torch.cuda.synchronize()
    return bits_of(base)


def check(p, want_fused):
    out, base, path = fused(p)
    assert bool(path & lora.PATH_FUSED) == want_fused, f"path bits {path}"
    ref = oracle.shrink_problem(p)
    w = ref != SENT
    assert np.array_equal(out[~w], ref[~w]), "out_r written outside the valid entries"
    assert_close(out[w], ref[w], p.dtype, what="out_r")
    assert_close(base, oracle.expand_problem(p, in_r=out), p.dtype, what="base_out")
    assert np.array_equal(base, expand_of(p, out)), "expand half differs from lora_expand"
    assert lora.device_error() == 0


@pytest.mark.parametrize("tok", [1, 50, 128, 300, 512])
def test_fused_qkv_decode(tok):
    check(make_problem("qkv", seed=70 + tok, tok=tok), want_fused=True)


def test_fused_fp16():
    check(make_problem("qkv", seed=71, tok=200, dtype="fp16"), want_fused=True)


@pytest.mark.parametrize("r,rs,slices", [(8, 8, None), (13, 16, None), (32, 32, None),
                                          (64, 64, (1024, 1024))])
def test_fused_rank_classes(r, rs, slices):
    # rs < rpad (r = 8: rank activations padded to 16 columns with zeros), an
    # odd rank with NaN storage padding, and the wide ranks (rank 64 with two
    # slices: three would leave no room for the split-K partial)
    over = {} if slices is None else {"slices": slices}
    p = make_problem("qkv", seed=72 + r, tok=160, K=1024, r=r, rs=rs, **over)
    check(p, want_fused=True)


def test_rank_64_three_slices_runs_the_two_kernels():
    p = make_problem("qkv", seed=78, tok=160, K=1024, r=64, rs=64)
    check(p, want_fused=False)


def test_fused_gate_up_many_adapters():
    p = make_problem("gate_up", seed=73, tok=256, K=2048, slices=(2048, 2048))
    check(p, want_fused=True)


def test_fused_zero_scaling_leaves_rows():
    p = make_problem("qkv", seed=74, tok=300, K=1024)
    p.scalings = p.scalings.copy()
    p.scalings[p.weight_indices[::2]] = 0.0  # every other segment's adapter
    out, base, path = fused(p)
    assert path & lora.PATH_FUSED
    ref_out = oracle.shrink_problem(p)
    w = ref_out != SENT
    assert_close(out[w], ref_out[w], p.dtype)
    ref = oracle.expand_problem(p, in_r=out)
    assert_close(base, ref, p.dtype)
    for s in range(p.nseg):
        if p.scalings[p.weight_indices[s]] == 0.0:
            rows = p.permutation[p.seg_indptr[s]: p.seg_indptr[s + 1]]
            assert np.array_equal(base[rows], p.base[rows])  # bit-identical


def test_large_batches_run_the_two_kernels():
    p = make_problem("qkv", seed=75, tok=2048, K=1024)
    check(p, want_fused=False)


def test_misaligned_inputs_run_the_two_kernels():
    p = make_problem("tail", seed=76)
    out, base, path = fused(p)
    assert not path & lora.PATH_FUSED
    ref = oracle.shrink_problem(p)
    w = ref != SENT
    assert_close(out[w], ref[w], p.dtype)
    assert_close(base, oracle.expand_problem(p, in_r=out), p.dtype)


def test_fused_launch_count():
    p = make_problem("qkv", seed=77, tok=64, K=512)
    lora.reset_launch_count()
    fused(p)
    assert lora.launch_count() == 1
