"""The scratch-free shrink entry point (lora_shrink_static_scratch).

Some callers are handed only input and output buffers by a host framework and
cannot allocate device memory, so they cannot pass the workspace that the
adapter-grouped schedule needs.  This entry point keeps that scratch in a
fixed array inside the library.  Its results must match the CPU oracle and the
ordinary lora_shrink called with a caller-provided workspace, call after call;
it must refuse problems whose scratch would not fit, and calls that need no
scratch (no more segments than adapters) must have no size limit.  The file is
named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from scatter_gemm_b200 import lora
from scatter_gemm_b200.workloads import make_problem
from tests.devutil import SENTINEL, Guarded, assert_close, tables

pytestmark = pytest.mark.gpu


def _problem():
    # many more segments than adapters, 16-byte-aligned: the grouped tensor-core path
    return make_problem("many_small", seed=41, tok=3000, nseg=400, K=1024,
                        slices=[1024, 256, 256])


def test_static_scratch_shrink_matches_the_workspace_shrink_twice():
    p = _problem()
    dt = torch.bfloat16
    x = Guarded(p.x, dt)
    A = Guarded(p.A, dt)
    si, wi, pm = tables(p)

    ref = Guarded(np.full((p.tok, p.S * p.rs), SENTINEL, np.uint16), dt)
    ws = lora.make_workspace(p.tok, p.nseg, p.L)
    lora.lora_shrink(x.t, A.t, si, wi, pm, ref.t, num_slices=p.S, rank=p.r, workspace=ws)
    torch.cuda.synchronize()
    assert lora.last_path() & lora.PATH_GROUPED
    ref_bits = ref.bits()
    written = ref_bits != SENTINEL
    # the oracle (its sentinel marks the rows and columns it leaves unwritten)
    want = oracle.shrink_problem(p)
    want_written = want != 0x7FFF
    assert np.array_equal(written, want_written), "write set differs from the oracle's"

    for call in range(2):
        out = Guarded(np.full((p.tok, p.S * p.rs), SENTINEL, np.uint16), dt)
        # straight through the C ABI
        f = lora.lib().lora_shrink_static_scratch
        f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64] + \
            [ctypes.c_int] * 8 + [ctypes.c_void_p]
        f.restype = ctypes.c_int
        st = f(x.t.data_ptr(), x.t.stride(0), A.t.data_ptr(), si.data_ptr(), wi.data_ptr(),
               pm.data_ptr(), out.t.data_ptr(), out.t.stride(0), p.tok, p.K, p.S, p.r, p.rs,
               p.nseg, p.L, 0, torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        assert st == lora.LORA_OK, lora.status_string(st)
        assert lora.last_path() & lora.PATH_GROUPED, "the static scratch was not used"
        got = out.bits()
        assert out.guards_intact()
        assert np.array_equal(got[~written], ref_bits[~written]), f"call {call}: write set"
        assert_close(got[written], ref_bits[written], p.dtype, what=f"call {call}")
        assert_close(got[written], want[written], p.dtype, what=f"call {call} vs oracle")
    assert lora.device_error(clear=True) == 0


def test_static_scratch_binding_matches_too():
    p = _problem()
    dt = torch.bfloat16
    x = torch.from_numpy(p.x.view(np.int16)).cuda().view(dt)
    A = torch.from_numpy(p.A.view(np.int16)).cuda().view(dt)
    si, wi, pm = tables(p)
    ref = torch.zeros(p.tok, p.S * p.rs, dtype=dt, device="cuda")
    lora.lora_shrink(x, A, si, wi, pm, ref, num_slices=p.S, rank=p.r,
                     workspace=lora.make_workspace(p.tok, p.nseg, p.L))
    got = torch.zeros_like(ref)
    lora.lora_shrink_static_scratch(x, A, si, wi, pm, got, num_slices=p.S, rank=p.r)
    torch.cuda.synchronize()
    r = ref.view(torch.int16).cpu().numpy().view(np.uint16)
    g = got.view(torch.int16).cpu().numpy().view(np.uint16)
    assert_close(g, r, p.dtype)


def test_static_scratch_refuses_problems_beyond_its_size():
    too_many = lora.STATIC_SCRATCH_BYTES // 4  # tok alone fills the array
    assert lora.workspace_size(too_many, 1024, 64) > lora.STATIC_SCRATCH_BYTES
    f = lora.lib().lora_shrink_static_scratch
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64] + \
        [ctypes.c_int] * 8 + [ctypes.c_void_p]
    f.restype = ctypes.c_int
    P = 0x10000  # never dereferenced: the size check comes first
    st = f(P, 64, P, P, P, P, P, 48, too_many, 64, 3, 16, 16, 1024, 64, 0, None)
    assert st == lora.LORA_ERR_UNSUPPORTED


@pytest.mark.parametrize("nseg", [4, 8])
def test_static_scratch_without_grouping_has_no_size_limit(nseg):
    # no grouping, so no scratch: either no more segments than adapters, or
    # 8 segments of 4 adapters whose pieces read 1 KB of weights each (4 KB
    # saved, under the pass's 64 KB threshold); a token count whose grouping
    # workspace would exceed the array still runs
    tok, K, S, rs, L = 270_000, 64, 1, 8, 4
    assert lora.workspace_size(tok, nseg, L) > lora.STATIC_SCRATCH_BYTES
    g = torch.Generator(device="cuda").manual_seed(5)
    x = torch.randn(tok, K, device="cuda", generator=g).to(torch.bfloat16)
    A = (0.02 * torch.randn(L, S * rs, K, device="cuda", generator=g)).to(torch.bfloat16)
    bounds = [0, 60_000, 130_000, 200_000, tok] if nseg == 4 else \
        [0, 30_000, 60_000, 95_000, 130_000, 165_000, 200_000, 235_000, tok]
    si = torch.tensor(bounds, dtype=torch.int32, device="cuda")
    wi = torch.tensor([2, 0, 3, 1, 2, 0, 3, 1][:nseg], dtype=torch.int32, device="cuda")
    pm = torch.randperm(tok, device="cuda", generator=g).to(torch.int32)
    ref = torch.zeros(tok, S * rs, dtype=torch.bfloat16, device="cuda")
    lora.lora_shrink(x, A, si, wi, pm, ref, num_slices=S)
    got = torch.zeros_like(ref)
    lora.lora_shrink_static_scratch(x, A, si, wi, pm, got, num_slices=S)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert lora.device_error(clear=True) == 0
