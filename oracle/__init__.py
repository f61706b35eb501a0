"""ctypes front end of the CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library: the
arithmetic lives in ``lora_oracle.c``; this file only marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np

from .build import build

_lib = None
_lock = threading.Lock()

BF16, FP16 = 0, 1
F32, F64, F64_IN = 0, 1, 2
BAD_DIMS, BAD_INDPTR, BAD_ADAPTER, BAD_PERMUTATION, BAD_SLICES = 1, 2, 4, 8, 16

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            l = ctypes.CDLL(path)
            l.oracle_check_tables.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _L]
            l.oracle_check_tables.restype = _I
            l.oracle_shrink.argtypes = [_P, _L, _P, _P, _P, _P, _P, _L] + [_I] * 9
            l.oracle_shrink.restype = _I
            l.oracle_expand.argtypes = [_P, _L, _P, _P, _P, _P, _P, _P, _P, _L] + [_I] * 8
            l.oracle_expand.restype = _I
            l.oracle_decode.argtypes = [ctypes.c_uint16, _I]
            l.oracle_decode.restype = ctypes.c_float
            l.oracle_encode.argtypes = [ctypes.c_float, _I]
            l.oracle_encode.restype = ctypes.c_uint16
            l.oracle_encode_f64.argtypes = [ctypes.c_double, _I]
            l.oracle_encode_f64.restype = ctypes.c_uint16
            l.oracle_embedding_a.argtypes = [_P, _P, _P, _P, _P, _L] + [_I] * 6
            l.oracle_embedding_a.restype = _I
            l.oracle_base_expand.argtypes = [_P, _L, _P, _L, _P, _L, _P, _P, _P, _P, _P, _P, _P,
                                             _L] + [_I] * 9
            l.oracle_base_expand.restype = _I
            l.oracle_set_threads.argtypes = [_I]
            l.oracle_set_threads.restype = None
            l.oracle_max_threads.argtypes = []
            l.oracle_max_threads.restype = _I
            _lib = l
    return _lib


def _dt(dtype: str) -> int:
    return BF16 if dtype == "bf16" else FP16


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def check_tables(seg_indptr, weight_indices, permutation, slice_offsets, tok, nseg, L, S,
                 ld_base=0) -> int:
    si, wi, pm = _c(seg_indptr, np.int32), _c(weight_indices, np.int32), _c(permutation, np.int32)
    so = None if slice_offsets is None else _c(slice_offsets, np.int32)
    return lib().oracle_check_tables(_ptr(si), _ptr(wi), _ptr(pm), _ptr(so), tok, nseg, L, S,
                                     ld_base)


def shrink(x, ld_x, A, seg_indptr, weight_indices, permutation, out_r, ld_out,
           tok, K, S, r, rs, nseg, L, dtype, mode=F32) -> int:
    """out_r is modified in place (uint16 for F32, float64 for F64)."""
    want = np.uint16 if mode == F32 else np.float64
    assert out_r.dtype == want and out_r.flags.c_contiguous
    x, A = _c(x, np.uint16), _c(A, np.uint16)
    si, wi, pm = _c(seg_indptr, np.int32), _c(weight_indices, np.int32), _c(permutation, np.int32)
    return lib().oracle_shrink(_ptr(x), ld_x, _ptr(A), _ptr(si), _ptr(wi), _ptr(pm),
                               _ptr(out_r), ld_out, tok, K, S, r, rs, nseg, L, _dt(dtype), mode)


def expand(in_r, ld_in, B, seg_indptr, weight_indices, permutation, slice_offsets,
           scalings, base_out, ld_base, tok, S, r, rs, nseg, L, dtype, mode=F32) -> int:
    """base_out is modified in place (uint16 for F32, float64 otherwise)."""
    want = np.uint16 if mode == F32 else np.float64
    assert base_out.dtype == want and base_out.flags.c_contiguous
    in_r = _c(in_r, np.float64 if mode == F64_IN else np.uint16)
    B = _c(B, np.uint16)
    si, wi, pm = _c(seg_indptr, np.int32), _c(weight_indices, np.int32), _c(permutation, np.int32)
    so, sc = _c(slice_offsets, np.int32), _c(scalings, np.float32)
    return lib().oracle_expand(_ptr(in_r), ld_in, _ptr(B), _ptr(si), _ptr(wi), _ptr(pm),
                               _ptr(so), _ptr(sc), _ptr(base_out), ld_base, tok, S, r, rs,
                               nseg, L, _dt(dtype), mode)


def embedding_a(ids, A_emb, seg_indptr, weight_indices, out, ld_out, tok, V, r, rs, nseg,
                L) -> int:
    """out (uint16 [tok, ld_out]) is modified in place."""
    assert out.dtype == np.uint16 and out.flags.c_contiguous
    ids = _c(ids, np.int32)
    A_emb = _c(A_emb, np.uint16)
    si, wi = _c(seg_indptr, np.int32), _c(weight_indices, np.int32)
    return lib().oracle_embedding_a(_ptr(ids), _ptr(A_emb), _ptr(si), _ptr(wi), _ptr(out),
                                    ld_out, tok, V, r, rs, nseg, L)


def base_expand(x, ld_x, W, ld_w, in_r, ld_in, B, seg_indptr, weight_indices, permutation,
                slice_offsets, scalings, out, ld_out, tok, K, S, r, rs, nseg, L, dtype,
                mode=F32) -> int:
    """out is modified in place (uint16 for F32, float64 for F64)."""
    want = np.uint16 if mode == F32 else np.float64
    assert out.dtype == want and out.flags.c_contiguous
    x, W, in_r, B = (_c(a, np.uint16) for a in (x, W, in_r, B))
    si, wi, pm = _c(seg_indptr, np.int32), _c(weight_indices, np.int32), _c(permutation, np.int32)
    so, sc = _c(slice_offsets, np.int32), _c(scalings, np.float32)
    return lib().oracle_base_expand(_ptr(x), ld_x, _ptr(W), ld_w, _ptr(in_r), ld_in, _ptr(B),
                                    _ptr(si), _ptr(wi), _ptr(pm), _ptr(so), _ptr(sc),
                                    _ptr(out), ld_out, tok, K, S, r, rs, nseg, L, _dt(dtype),
                                    mode)


# ---------------------------------------------------------------- problem helpers

def shrink_problem(p, mode=F32, x=None):
    """Runs the oracle shrink on a workloads.Problem; returns out_r.

    Unwritten entries keep a NaN sentinel (F32) / NaN (F64)."""
    x = p.x if x is None else x
    ld = p.S * p.rs
    if mode == F32:
        out = np.full((p.tok, ld), 0x7FFF, dtype=np.uint16)
    else:
        out = np.full((p.tok, ld), np.nan, dtype=np.float64)
    rc = shrink(x, p.ld_x, p.A, p.seg_indptr, p.weight_indices, p.permutation, out, ld,
                p.tok, p.K, p.S, p.r, p.rs, p.nseg, p.L, p.dtype, mode)
    if rc:
        raise ValueError(f"oracle_shrink rejected the problem (code {rc})")
    return out


def expand_problem(p, in_r=None, base=None, mode=F32, scalings=None):
    """Runs the oracle expand on a workloads.Problem; returns the new base."""
    in_r = p.in_r if in_r is None else in_r
    ld_in = in_r.shape[1]
    sc = p.scalings if scalings is None else scalings
    if mode == F32:
        out = (p.base if base is None else base).copy()
    else:
        out = (decode(p.base, p.dtype).astype(np.float64) if base is None
               else np.array(base, dtype=np.float64))
    rc = expand(in_r, ld_in, p.B, p.seg_indptr, p.weight_indices, p.permutation,
                p.slice_offsets, sc, out, p.ld_base, p.tok, p.S, p.r, p.rs, p.nseg, p.L,
                p.dtype, mode)
    if rc:
        raise ValueError(f"oracle_expand rejected the problem (code {rc})")
    return out


def base_expand_problem(p, W, in_r=None, out=None, mode=F32, scalings=None):
    """The base projection x W^T with the expand folded in, on a
    workloads.Problem; W is [N_tot, K] (uint16).  Starts from `out` (default
    p.base): rows of tokens outside segments keep it."""
    in_r = p.in_r if in_r is None else in_r
    sc = p.scalings if scalings is None else scalings
    if mode == F32:
        o = (p.base if out is None else out).copy()
    else:
        o = np.full(p.base.shape, np.nan, dtype=np.float64)
    rc = base_expand(p.x, p.ld_x, W, W.shape[1], in_r, in_r.shape[1], p.B, p.seg_indptr,
                     p.weight_indices, p.permutation, p.slice_offsets, sc, o, p.ld_base,
                     p.tok, p.K, p.S, p.r, p.rs, p.nseg, p.L, p.dtype, mode)
    if rc:
        raise ValueError(f"oracle_base_expand rejected the problem (code {rc})")
    return o


def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    """uint16 bf16/fp16 bit patterns -> float32 (bf16 is the top half of binary32)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32)
    return bits.view(np.float16).astype(np.float32)


def set_threads(n: int) -> None:
    """Sets the OpenMP thread count the oracle uses."""
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())
