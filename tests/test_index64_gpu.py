"""int64 index tables (lora_shrink_i64 / lora_expand_i64): the same results,
bit for bit, as the int32 tables, and the same bar against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from scatter_gemm_b200 import lora
from scatter_gemm_b200.workloads import make_problem
from tests.devutil import assert_close

pytestmark = pytest.mark.gpu


def dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(
        torch.bfloat16 if dtype == "bf16" else torch.float16)


def bits_of(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def tabs(p, itype, identity=False):
    cast = lambda a: torch.from_numpy(a.astype(itype)).cuda()
    return (cast(p.seg_indptr), cast(p.weight_indices),
            None if identity else cast(p.permutation))


def shrink(p, itype, identity=False, workspace="auto"):
    out = dev(np.full((p.tok, p.S * p.rs), 0x7FFF, dtype=np.uint16), p.dtype)
    si, wi, pm = tabs(p, itype, identity)
    ws = None
    if workspace == "grouping":
        n = lora.workspace_size(p.tok, p.nseg, p.L)
        if itype == np.int64:
            n += lora.index64_workspace_size(p.tok, p.nseg)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    lora.lora_shrink(dev(p.x, p.dtype)[:, : p.K], dev(p.A, p.dtype), si, wi, pm, out,
                     num_slices=p.S, rank=p.r, workspace=ws)
    torch.cuda.synchronize()
    return bits_of(out)


def expand(p, itype, in_r, identity=False, workspace="auto"):
    base = dev(p.base, p.dtype)
    si, wi, pm = tabs(p, itype, identity)
    sc = torch.from_numpy(p.scalings.astype(np.float32)).cuda()
    ws = None
    if workspace == "grouping":
        n = lora.workspace_size(p.tok, p.nseg, p.L)
        if itype == np.int64:
            n += lora.index64_workspace_size(p.tok, p.nseg)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    lora.lora_expand(dev(in_r, p.dtype), dev(p.B, p.dtype), si, wi, pm,
                     [int(v) for v in p.slice_offsets], sc, base, rank=p.r, workspace=ws)
    torch.cuda.synchronize()
    return bits_of(base)


@pytest.mark.parametrize("name,tok", [("qkv", 200), ("qkv", 1500), ("tail", None),
                                      ("many_small", 2048)])
def test_int64_tables_match_int32_and_oracle(name, tok):
    over = {} if tok is None else {"tok": tok}
    if name == "many_small":
        over.update(K=1024)
    p = make_problem(name, seed=61, **over)
    s32 = shrink(p, np.int32, workspace="grouping")
    s64 = shrink(p, np.int64, workspace="grouping")
    assert np.array_equal(s32, s64)
    ref = oracle.shrink_problem(p)
    w = ref != 0x7FFF
    assert np.array_equal(s64[~w], np.full_like(s64[~w], 0x7FFF))
    assert_close(s64[w], ref[w], p.dtype)
    e32 = expand(p, np.int32, p.in_r, workspace="grouping")
    e64 = expand(p, np.int64, p.in_r, workspace="grouping")
    assert np.array_equal(e32, e64)
    assert_close(e64, oracle.expand_problem(p), p.dtype)
    assert lora.device_error() == 0


def test_int64_without_permutation_and_allocated_workspace():
    p = make_problem("qkv", seed=62, tok=300, K=1024)
    p.permutation = np.arange(p.tok, dtype=np.int32)
    s32 = shrink(p, np.int32, identity=True)
    s64 = shrink(p, np.int64, identity=True)  # the binding allocates the workspace
    assert np.array_equal(s32, s64)
    e64 = expand(p, np.int64, s64, identity=True)
    e32 = expand(p, np.int32, s64, identity=True)
    assert np.array_equal(e32, e64)
    assert_close(e64, oracle.expand_problem(p, in_r=s64), p.dtype)


def test_int64_call_adds_one_launch():
    p = make_problem("qkv", seed=63, tok=256, K=512)
    lora.reset_launch_count()
    shrink(p, np.int32)
    n32 = lora.launch_count()
    lora.reset_launch_count()
    shrink(p, np.int64)
    assert lora.launch_count() == n32 + 1


def test_mixed_index_types_are_rejected():
    p = make_problem("qkv", seed=64, tok=64, K=512)
    si, wi, pm = tabs(p, np.int32)
    out = dev(np.zeros((p.tok, p.S * p.rs), dtype=np.uint16), p.dtype)
    with pytest.raises(ValueError):
        lora.lora_shrink(dev(p.x, p.dtype)[:, : p.K], dev(p.A, p.dtype), si.long(), wi, pm,
                         out, num_slices=p.S, rank=p.r)
