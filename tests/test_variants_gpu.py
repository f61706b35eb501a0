"""The identity-permutation ops (sgemm_lora_a/b, qkv_lora_b, gate_up_lora_b)
and the embedding LoRA A against the CPU oracle, same bar as the pair."""
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


def identity(p):
    p.permutation = np.arange(p.tok, dtype=np.int32)
    return p


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_sgemm_lora_a(dtype):
    p = identity(make_problem("qkv", seed=51, tok=333, K=512, dtype=dtype))
    ref = oracle.shrink_problem(p)
    out = dev(np.full((p.tok, p.S * p.rs), 0x7FFF, dtype=np.uint16), dtype)
    lora.sgemm_lora_a_fwd(dev(p.x, dtype), dev(p.A, dtype), torch.from_numpy(p.seg_indptr).cuda(),
                          torch.from_numpy(p.weight_indices).cuda(), out, num_slices=p.S,
                          rank=p.r)
    got = bits_of(out)
    w = ref != 0x7FFF
    assert np.array_equal(got[~w], ref[~w])  # nothing written outside the valid columns
    assert_close(got[w], ref[w], dtype)


@pytest.mark.parametrize("op", ["sgemm_b", "qkv_b", "gate_up_b"])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_expand_variants(op, dtype):
    slices = {"sgemm_b": [640], "qkv_b": [512, 128, 128], "gate_up_b": [384, 384]}[op]
    # rows before and after the segments (and, for the op with explicit
    # offsets, columns before slice 0) that nothing may touch
    extra = dict(lead=7, trail=5, col_lead=16 if op == "qkv_b" else 0)
    p = identity(make_problem("qkv", seed=52, tok=300, K=64, slices=slices, dtype=dtype,
                              **extra))
    ref = oracle.expand_problem(p)
    base = dev(p.base, dtype)
    args = (dev(p.in_r, dtype), dev(p.B, dtype), torch.from_numpy(p.seg_indptr).cuda(),
            torch.from_numpy(p.weight_indices).cuda())
    sc = torch.from_numpy(p.scalings).cuda()
    if op == "sgemm_b":
        lora.sgemm_lora_b_fwd(*args, sc, base, rank=p.r)
    elif op == "qkv_b":
        lora.qkv_lora_b_fwd(*args, p.slice_offsets.tolist(), sc, base, rank=p.r)
    else:
        lora.gate_up_lora_b_fwd(*args, sc, base, rank=p.r)
    got = bits_of(base)
    # write set, bit for bit: only the rows of the segments (zero-scaled
    # adapters excluded) and the slice columns may change
    touched = np.zeros(got.shape, dtype=bool)
    off = p.slice_offsets
    for s in range(p.nseg):
        if p.scalings[p.weight_indices[s]] == 0.0:
            continue
        rows = np.arange(p.seg_indptr[s], p.seg_indptr[s + 1])
        touched[np.ix_(rows, np.arange(off[0], off[-1]))] = True
    assert np.array_equal(got[~touched], p.base[~touched]), f"{op} wrote outside its write set"
    assert_close(got[touched], ref[touched], dtype)


@pytest.mark.parametrize("nseg,tok", [(4, 500), (300, 300), (3000, 3000)])
def test_embedding_lora_a_is_an_exact_gather(nseg, tok):
    rng = np.random.default_rng(53)
    V, r, rs, L = 1000, 13, 16, 5
    p = make_problem("tiny", seed=53, tok=tok, K=8, slices=[8], L=L, r=r, rs=rs, nseg=nseg,
                     recipe="ones" if nseg == tok else "random")
    ids = rng.integers(0, V, size=tok).astype(np.int32)
    A_emb = (rng.standard_normal((L, rs, V)).astype(np.float32) * 0.02)
    from scatter_gemm_b200.workloads import to_bits
    A_bits = to_bits(A_emb, "bf16")
    ref = np.full((tok, rs), 0x7FFF, dtype=np.uint16)
    assert oracle.embedding_a(ids, A_bits, p.seg_indptr, p.weight_indices, ref, rs, tok, V, r,
                              rs, p.nseg, L) == 0
    out = dev(np.full((tok, rs), 0x7FFF, dtype=np.uint16), "bf16")  # the oracle's sentinel
    lora.embedding_lora_a_fwd(torch.from_numpy(ids).cuda(), dev(A_bits, "bf16"),
                              torch.from_numpy(p.seg_indptr).cuda(),
                              torch.from_numpy(p.weight_indices).cuda(), out, rank=r)
    assert np.array_equal(bits_of(out), ref)  # a gather: bit exact, write set included


def test_chunked_aliases_are_the_pair():
    assert lora.chunked_sgmv_lora_shrink_fwd is lora.lora_shrink
    assert lora.chunked_sgmv_lora_expand_fwd is lora.lora_expand
