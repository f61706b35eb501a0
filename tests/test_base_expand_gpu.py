"""lora_base_expand (the base projection with the expand folded into its
epilogue) against the CPU oracle: written entries within
|err| <= 2e-2 + 1e-2 |ref|, everything else untouched bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from scatter_gemm_b200 import lora
from scatter_gemm_b200.workloads import make_base_weight, make_problem
from tests.devutil import assert_close

pytestmark = pytest.mark.gpu
SENT = 0x7FFF


def dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(
        torch.bfloat16 if dtype == "bf16" else torch.float16)


def bits_of(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run(p, W, scalings=None):
    sc = p.scalings if scalings is None else scalings
    out0 = np.full(p.base.shape, SENT, dtype=np.uint16)
    out = dev(out0, p.dtype)
    c = lambda a: torch.from_numpy(a.astype(np.int32)).cuda()
    lora.lora_base_expand(dev(p.x, p.dtype)[:, : p.K], dev(W, p.dtype), dev(p.in_r, p.dtype),
                          dev(p.B, p.dtype), c(p.seg_indptr), c(p.weight_indices),
                          c(p.permutation), [int(v) for v in p.slice_offsets],
                          torch.from_numpy(sc.astype(np.float32)).cuda(), out, rank=p.r)
    torch.cuda.synchronize()
    got = bits_of(out)
    ref = oracle.base_expand_problem(p, W, out=out0, scalings=sc)
    w = ref != SENT
    assert np.array_equal(got[~w], ref[~w]), "written outside the segments' rows and slices"
    assert_close(got[w], ref[w], p.dtype, what="out")
    assert lora.device_error() == 0
    assert lora.last_path() & lora.PATH_FUSED
    return got, ref


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_base_expand_qkv(dtype):
    p = make_problem("qkv", seed=80, tok=300, K=1024, slices=(512, 256, 256), dtype=dtype)
    run(p, make_base_weight(p, 80, ld_pad=8))


@pytest.mark.parametrize("r,rs", [(8, 8), (13, 16), (64, 64)])
def test_base_expand_rank_classes(r, rs):
    p = make_problem("qkv", seed=81 + r, tok=200, K=512, slices=(256, 128, 128), r=r, rs=rs)
    run(p, make_base_weight(p, 81))


def test_base_expand_k_tail_ragged_slices_many_segments():
    # K not a multiple of 64, slice widths not multiples of 128, segments that
    # start off the 128-row grid
    p = make_problem("qkv", seed=82, tok=777, K=1000, slices=(200, 136, 64), L=5, nseg=9,
                     recipe="dirichlet")
    run(p, make_base_weight(p, 82, ld_pad=24))


def test_base_expand_zero_scaling_is_the_projection():
    p = make_problem("qkv", seed=83, tok=160, K=512, slices=(256, 128, 128))
    sc = p.scalings.copy()
    sc[p.weight_indices[::2]] = 0.0
    run(p, make_base_weight(p, 83), scalings=sc)


def test_base_expand_single_token():
    p = make_problem("qkv", seed=84, tok=1, K=256, slices=(128, 128, 128))
    run(p, make_base_weight(p, 84))


def test_base_expand_misaligned_is_unsupported():
    p = make_problem("qkv", seed=85, tok=16, K=256, slices=(128, 128, 128))
    W = make_base_weight(p, 85)
    x = dev(p.x, p.dtype)[:, : p.K]
    out = dev(p.base, p.dtype)
    c = lambda a: torch.from_numpy(a.astype(np.int32)).cuda()
    flat = torch.empty(p.tok * p.K + 1, dtype=x.dtype, device="cuda")
    x_off = flat[1:].view(p.tok, p.K)  # 2 bytes off a 16-byte boundary
    x_off.copy_(x)
    with pytest.raises(lora.LoraError) as e:
        lora.lora_base_expand(x_off, dev(W, p.dtype), dev(p.in_r, p.dtype), dev(p.B, p.dtype),
                              c(p.seg_indptr), c(p.weight_indices), c(p.permutation),
                              [int(v) for v in p.slice_offsets],
                              torch.from_numpy(p.scalings).cuda(), out, rank=p.r)
    assert e.value.status == lora.LORA_ERR_UNSUPPORTED


def test_base_expand_full_qkv_shape():
    # the projection at the qkv workload's K = 4096 with its 4096/1024/1024
    # slices and eight adapters of rank 16, at a token count the oracle
    # finishes in seconds (a few 128-row pieces per segment, ragged)
    p = make_problem("qkv", seed=86, tok=256)
    run(p, make_base_weight(p, 86))
