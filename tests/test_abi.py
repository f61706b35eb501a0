"""The C ABI library loads, exports every declared entry point and rejects bad
arguments before touching the GPU.  Runs on a machine without a GPU: every
call here returns before any CUDA call (argument errors, empty problems,
size queries)."""
import ctypes
import os
import re

import pytest

from scatter_gemm_b200 import lora
from scatter_gemm_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_sgmv.h")

OK, INVALID, UNSUPPORTED = 0, 1, 2
# fake but aligned addresses: the calls below must reject or no-op before use
P = 0x10000


@pytest.fixture(scope="module")
def L():
    build()
    return lora.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LORA_API\s+[\w\s\*]+?\b(lora_\w+)\s*\(", text)))


def test_header_declares_the_calls():
    syms = declared_symbols()
    for s in ("lora_shrink", "lora_expand", "lora_validate", "lora_status_string",
              "lora_workspace_size"):
        assert s in syms


def test_library_exports_every_declared_symbol(L):
    lib = ctypes.CDLL(LIB)
    for s in declared_symbols():
        assert hasattr(lib, s), f"{s} is declared in lora_sgmv.h but not exported"


def test_status_strings(L):
    for code in range(5):
        assert lora.status_string(code)
    assert lora.status_string(99) == "unknown status"


def shrink(lib, **kw):
    a = dict(x=P, ld_x=64, A=P, si=P, wi=P, pm=P, out=P, ld_out=48, tok=10, K=64, S=3, r=16,
             rs=16, nseg=2, nad=4, dt=0, ws=None, wsb=0, st=None)
    a.update(kw)
    return lib.lora_shrink(a["x"], a["ld_x"], a["A"], a["si"], a["wi"], a["pm"], a["out"],
                           a["ld_out"], a["tok"], a["K"], a["S"], a["r"], a["rs"], a["nseg"],
                           a["nad"], a["dt"], a["ws"], a["wsb"], a["st"])


def expand(lib, off=(0, 32, 40, 48), **kw):
    arr = (ctypes.c_int32 * len(off))(*off)
    a = dict(inr=P, ld_in=48, B=P, si=P, wi=P, pm=P, offp=ctypes.cast(arr, ctypes.c_void_p),
             sc=P, base=P, ld_base=48, tok=10, S=len(off) - 1, r=16, rs=16, nseg=2, nad=4, dt=0,
             ws=None, wsb=0, st=None)
    a.update(kw)
    return lib.lora_expand(a["inr"], a["ld_in"], a["B"], a["si"], a["wi"], a["pm"], a["offp"],
                           a["sc"], a["base"], a["ld_base"], a["tok"], a["S"], a["r"], a["rs"],
                           a["nseg"], a["nad"], a["dt"], a["ws"], a["wsb"], a["st"])


@pytest.mark.parametrize("kw,want", [
    (dict(x=None), INVALID), (dict(A=None), INVALID), (dict(si=None), INVALID),
    (dict(wi=None), INVALID), (dict(out=None), INVALID),
    (dict(tok=-1), INVALID), (dict(nseg=-1), INVALID), (dict(K=0), INVALID),
    (dict(S=0), INVALID), (dict(r=0), INVALID), (dict(rs=8), INVALID), (dict(nad=0), INVALID),
    (dict(S=9, ld_out=9 * 16), UNSUPPORTED), (dict(dt=2), UNSUPPORTED),
    (dict(ld_x=63), INVALID), (dict(ld_out=47), INVALID),
    (dict(wsb=16), INVALID),  # workspace bytes without a workspace
    (dict(x=P + 1), INVALID), (dict(out=P + 1), INVALID), (dict(si=P + 2), INVALID),
    (dict(pm=P + 2), INVALID),
    (dict(tok=0), OK), (dict(nseg=0), OK), (dict(tok=0, pm=None), OK),
])
def test_shrink_argument_checks(L, kw, want):
    assert shrink(L, **kw) == want


@pytest.mark.parametrize("kw,want", [
    (dict(inr=None), INVALID), (dict(B=None), INVALID), (dict(sc=None), INVALID),
    (dict(base=None), INVALID), (dict(offp=None), INVALID),
    (dict(r=17), INVALID), (dict(ld_in=47), INVALID), (dict(dt=7), UNSUPPORTED),
    (dict(ld_base=47), INVALID),  # off[S] > ld_base
    (dict(sc=P + 2), INVALID), (dict(base=P + 1), INVALID),
    (dict(tok=0), OK), (dict(nseg=0), OK),
])
def test_expand_argument_checks(L, kw, want):
    assert expand(L, **kw) == want


def test_expand_rejects_bad_slice_tables(L):
    assert expand(L, off=(0, 40, 32, 48)) == INVALID      # decreasing
    assert expand(L, off=(-1, 32, 40, 48)) == INVALID     # negative
    assert expand(L, off=(0, 32, 40, 48), ld_base=40) == INVALID
    assert expand(L, off=tuple(range(0, 80, 8)), ld_in=9 * 16) == UNSUPPORTED  # S = 9
    assert expand(L, off=(8, 8), S=1, tok=5) == OK        # no columns: nothing to do


def shrink64(lib, **kw):
    a = dict(x=P, ld_x=64, A=P, si=P, wi=P, pm=P, out=P, ld_out=48, tok=10, K=64, S=3, r=16,
             rs=16, nseg=2, nad=4, dt=0, ws=P, wsb=1 << 20, st=None)
    a.update(kw)
    return lib.lora_shrink_i64(a["x"], a["ld_x"], a["A"], a["si"], a["wi"], a["pm"], a["out"],
                               a["ld_out"], a["tok"], a["K"], a["S"], a["r"], a["rs"],
                               a["nseg"], a["nad"], a["dt"], a["ws"], a["wsb"], a["st"])


def expand64(lib, off=(0, 32, 40, 48), **kw):
    arr = (ctypes.c_int32 * len(off))(*off)
    a = dict(inr=P, ld_in=48, B=P, si=P, wi=P, pm=P, offp=ctypes.cast(arr, ctypes.c_void_p),
             sc=P, base=P, ld_base=48, tok=10, S=len(off) - 1, r=16, rs=16, nseg=2, nad=4, dt=0,
             ws=P, wsb=1 << 20, st=None)
    a.update(kw)
    return lib.lora_expand_i64(a["inr"], a["ld_in"], a["B"], a["si"], a["wi"], a["pm"],
                               a["offp"], a["sc"], a["base"], a["ld_base"], a["tok"], a["S"],
                               a["r"], a["rs"], a["nseg"], a["nad"], a["dt"], a["ws"], a["wsb"],
                               a["st"])


# every case returns before the narrowing kernel would be enqueued
@pytest.mark.parametrize("kw,want", [
    (dict(si=None), INVALID), (dict(wi=None), INVALID),
    (dict(si=P + 4), INVALID), (dict(wi=P + 4), INVALID), (dict(pm=P + 4), INVALID),
    (dict(ws=None, wsb=0), INVALID),     # the narrowed tables need a workspace
    (dict(wsb=16), INVALID),             # too small for them
    (dict(ws=P + 8), INVALID),           # not 16-byte aligned
    (dict(x=None), INVALID), (dict(out=P + 1), INVALID),
    (dict(tok=-1), INVALID), (dict(dt=2), UNSUPPORTED), (dict(rs=8), INVALID),
    (dict(tok=0), OK), (dict(nseg=0), OK),
])
def test_shrink_i64_argument_checks(L, kw, want):
    assert shrink64(L, **kw) == want


@pytest.mark.parametrize("kw,want", [
    (dict(si=None), INVALID), (dict(pm=P + 4), INVALID), (dict(ws=None, wsb=0), INVALID),
    (dict(wsb=8), INVALID), (dict(sc=None), INVALID), (dict(base=P + 1), INVALID),
    (dict(offp=None), INVALID), (dict(dt=3), UNSUPPORTED), (dict(tok=0), OK),
])
def test_expand_i64_argument_checks(L, kw, want):
    assert expand64(L, **kw) == want


def pair(lib, off=(0, 32, 40, 48), **kw):
    arr = (ctypes.c_int32 * len(off))(*off)
    a = dict(x=P, ld_x=64, A=P, B=P, si=P, wi=P, pm=P, offp=ctypes.cast(arr, ctypes.c_void_p),
             sc=P, out=P, ld_out=48, base=P, ld_base=48, tok=10, K=64, S=len(off) - 1, r=16,
             rs=16, nseg=2, nad=4, dt=0, ws=None, wsb=0, st=None)
    a.update(kw)
    return lib.lora_shrink_expand(a["x"], a["ld_x"], a["A"], a["B"], a["si"], a["wi"], a["pm"],
                                  a["offp"], a["sc"], a["out"], a["ld_out"], a["base"],
                                  a["ld_base"], a["tok"], a["K"], a["S"], a["r"], a["rs"],
                                  a["nseg"], a["nad"], a["dt"], a["ws"], a["wsb"], a["st"])


@pytest.mark.parametrize("kw,want", [
    (dict(x=None), INVALID), (dict(A=None), INVALID), (dict(B=None), INVALID),
    (dict(si=None), INVALID), (dict(wi=None), INVALID), (dict(sc=None), INVALID),
    (dict(out=None), INVALID), (dict(base=None), INVALID), (dict(offp=None), INVALID),
    (dict(K=0), INVALID), (dict(rs=8), INVALID), (dict(dt=2), UNSUPPORTED),
    (dict(ld_out=47), INVALID), (dict(ld_base=47), INVALID), (dict(ld_x=63), INVALID),
    (dict(B=P + 1), INVALID), (dict(sc=P + 2), INVALID), (dict(pm=P + 2), INVALID),
    (dict(wsb=16), INVALID),
    (dict(tok=0), OK), (dict(nseg=0), OK),
])
def test_shrink_expand_argument_checks(L, kw, want):
    assert pair(L, **kw) == want


def base_expand(lib, off=(0, 32, 40, 48), **kw):
    arr = (ctypes.c_int32 * len(off))(*off)
    a = dict(x=P, ld_x=64, W=P, ld_w=64, inr=P, ld_in=48, B=P, si=P, wi=P, pm=P,
             offp=ctypes.cast(arr, ctypes.c_void_p), sc=P, out=P, ld_out=48, tok=10, K=64,
             S=len(off) - 1, r=16, rs=16, nseg=2, nad=4, dt=0, st=None)
    a.update(kw)
    return lib.lora_base_expand(a["x"], a["ld_x"], a["W"], a["ld_w"], a["inr"], a["ld_in"],
                                a["B"], a["si"], a["wi"], a["pm"], a["offp"], a["sc"], a["out"],
                                a["ld_out"], a["tok"], a["K"], a["S"], a["r"], a["rs"],
                                a["nseg"], a["nad"], a["dt"], a["st"])


# all of these return before any CUDA call
@pytest.mark.parametrize("kw,want", [
    (dict(x=None), INVALID), (dict(W=None), INVALID), (dict(inr=None), INVALID),
    (dict(B=None), INVALID), (dict(sc=None), INVALID), (dict(out=None), INVALID),
    (dict(offp=None), INVALID), (dict(ld_w=32), INVALID), (dict(ld_in=40), INVALID),
    (dict(ld_out=40), INVALID), (dict(K=0), INVALID), (dict(dt=2), UNSUPPORTED),
    (dict(x=P + 2), UNSUPPORTED), (dict(W=P + 8), UNSUPPORTED), (dict(ld_w=68), UNSUPPORTED),
    (dict(K=60, ld_x=64, ld_w=64), UNSUPPORTED), (dict(r=65, rs=72, ld_in=3 * 72), UNSUPPORTED),
    (dict(pm=P + 2), INVALID), (dict(tok=0), OK), (dict(nseg=0), OK),
])
def test_base_expand_argument_checks(L, kw, want):
    assert base_expand(L, **kw) == want


def test_index64_workspace_size(L):
    # narrowed seg_indptr, weight_indices and permutation, each padded to 16 bytes
    assert lora.index64_workspace_size(100, 3) == 4 * (4 + 4 + 100)
    assert lora.index64_workspace_size(0, 0) == 16
    assert lora.index64_workspace_size(7, 5) == 4 * (8 + 8 + 8)
    assert L.lora_index64_workspace_size(-1, 2) == 0


def test_workspace_sizes(L):
    assert lora.workspace_size(0, 0, 1) > 0
    assert lora.workspace_size(8192, 1024, 64) >= 4 * (8192 + 65)
    assert L.lora_validate_workspace_size(1000) >= 4 * 32
    assert L.lora_workspace_size(-1, 0, 1) == 0


def test_validate_argument_checks(L):
    res = P
    assert L.lora_validate(None, P, P, None, 10, 2, 4, 1, 0, res, P, 64, None) == INVALID
    assert L.lora_validate(P, P, P, None, 10, 2, 4, 1, 0, None, P, 64, None) == INVALID
    # a permutation needs scratch for its bijection check
    assert L.lora_validate(P, P, P, None, 10, 2, 4, 1, 0, res, None, 0, None) == INVALID
    assert L.lora_validate(P, P, P, None, 100, 2, 4, 1, 0, res, P, 4, None) == INVALID


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(lora, "_lib", None)
    monkeypatch.setattr(lora, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        lora.lib()


@pytest.mark.parametrize("fn", ["lora_shrink", "lora_shrink_static_scratch"])
@pytest.mark.parametrize("case", ["short_out", "narrow_out", "narrow_x", "ragged_slices"])
def test_shrink_bindings_check_shapes_before_any_call(L, fn, case):
    """Both shrink bindings reject mismatched shapes on the host, before the
    library is called (the tensors here are CPU tensors: nothing reaches a GPU)."""
    import torch
    tok, K, S, rs = 12, 64, 3, 16
    x = torch.zeros(tok, K, dtype=torch.bfloat16)
    A = torch.zeros(2, S * rs, K, dtype=torch.bfloat16)
    out = torch.zeros(tok, S * rs, dtype=torch.bfloat16)
    S_arg = S
    if case == "short_out":
        out = torch.zeros(tok - 1, S * rs, dtype=torch.bfloat16)
    elif case == "narrow_out":
        out = torch.zeros(tok, S * rs - 8, dtype=torch.bfloat16)
    elif case == "narrow_x":
        x = torch.zeros(tok, 2 * K, dtype=torch.bfloat16)[:, : K - 8]
    else:
        S_arg = 5  # 48 rows of A are not a multiple of 5 slices
    si = torch.zeros(2, dtype=torch.int32)
    wi = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError):
        getattr(lora, fn)(x, A, si, wi, None, out, num_slices=S_arg)
