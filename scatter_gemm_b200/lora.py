"""Thin ctypes binding of liblora_sgmv (argument marshalling only).

Every step of the shrink and expand runs in the CUDA library; this module
checks torch-side metadata (device, dtype, strides) on the host, takes
``data_ptr()`` of each tensor and the current CUDA stream, and calls the C
ABI declared in ``include/lora_sgmv.h``.  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LORA_SGMV_LIB may point at another build of the library (e.g. an installed copy)
LIB_PATH = os.environ.get("LORA_SGMV_LIB") or os.path.join(_HERE, "liblora_sgmv.so")

LORA_OK, LORA_ERR_INVALID_ARGUMENT, LORA_ERR_UNSUPPORTED, LORA_ERR_CUDA, LORA_ERR_BAD_VALUES = \
    range(5)
BAD_INDPTR, BAD_ADAPTER, BAD_PERMUTATION, BAD_SLICES = 2, 4, 8, 16
MAX_SLICES = 8

_P, _I, _L, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_lib = None
_lock = threading.Lock()


class LoraError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Loads liblora_sgmv.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m scatter_gemm_b200.build`")
            l = ctypes.CDLL(LIB_PATH)
            l.lora_shrink.argtypes = [_P, _L, _P, _P, _P, _P, _P, _L] + [_I] * 8 + [_P, _Z, _P]
            l.lora_shrink.restype = _I
            l.lora_expand.argtypes = [_P, _L, _P, _P, _P, _P, _P, _P, _P, _L] + [_I] * 7 + \
                [_P, _Z, _P]
            l.lora_expand.restype = _I
            l.lora_validate.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _L, _P, _P, _Z, _P]
            l.lora_validate.restype = _I
            l.lora_workspace_size.argtypes = [_I, _I, _I]
            l.lora_workspace_size.restype = _Z
            l.lora_validate_workspace_size.argtypes = [_I]
            l.lora_validate_workspace_size.restype = _Z
            l.lora_status_string.argtypes = [_I]
            l.lora_status_string.restype = ctypes.c_char_p
            l.lora_launch_count.argtypes = []
            l.lora_launch_count.restype = ctypes.c_uint64
            l.lora_reset_launch_count.argtypes = []
            l.lora_reset_launch_count.restype = None
            l.lora_last_path.argtypes = []
            l.lora_last_path.restype = _I
            l.lora_device_error.argtypes = [_P, _I]
            l.lora_device_error.restype = _I
            l.lora_shrink_i64.argtypes = l.lora_shrink.argtypes
            l.lora_shrink_i64.restype = _I
            l.lora_expand_i64.argtypes = l.lora_expand.argtypes
            l.lora_expand_i64.restype = _I
            l.lora_index64_workspace_size.argtypes = [_I, _I]
            l.lora_index64_workspace_size.restype = _Z
            l.lora_shrink_expand.argtypes = [_P, _L, _P, _P, _P, _P, _P, _P, _P, _P, _L, _P, _L] + \
                [_I] * 8 + [_P, _Z, _P]
            l.lora_shrink_expand.restype = _I
            l.lora_base_expand.argtypes = [_P, _L, _P, _L, _P, _L, _P, _P, _P, _P, _P, _P, _P,
                                           _L] + [_I] * 8 + [_P]
            l.lora_base_expand.restype = _I
            _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().lora_status_string(status).decode()


def launch_count() -> int:
    return int(lib().lora_launch_count())


def reset_launch_count() -> None:
    lib().lora_reset_launch_count()


PATH_GENERAL, PATH_TENSOR, PATH_GROUPED, PATH_SPLITK, PATH_FUSED = 1, 2, 4, 8, 16


def last_path() -> int:
    """LORA_PATH_* bits of the last call's kernel path on this thread."""
    return int(lib().lora_last_path())


def device_error(clear: bool = True) -> int:
    """Reads (and clears) the device-side failure code of the bounded waits."""
    v = ctypes.c_int32(0)
    st = lib().lora_device_error(ctypes.byref(v), int(clear))
    if st != LORA_OK:
        raise LoraError("lora_device_error", st)
    return int(v.value)


def workspace_size(tok: int, nseg: int, num_adapters: int) -> int:
    return int(lib().lora_workspace_size(tok, nseg, num_adapters))


def make_workspace(tok: int, nseg: int, num_adapters: int, device=None) -> torch.Tensor:
    """Allocates (through torch) the optional scratch that lets the calls
    group many small segments by adapter."""
    n = workspace_size(tok, nseg, num_adapters)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device or "cuda")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return 0
    if t.dtype == torch.float16:
        return 1
    raise TypeError(f"unsupported element type {t.dtype} (bf16 or fp16)")


def _row_major(t: torch.Tensor, name: str, dims: int = 2) -> int:
    if t.dim() != dims:
        raise ValueError(f"{name} must be {dims}-D, got {tuple(t.shape)}")
    if t.stride(-1) != 1:
        raise ValueError(f"{name} must have a unit inner stride")
    return t.stride(0) if dims == 2 else 0


def _table(t: Optional[torch.Tensor], name: str, allow_none: bool = False,
           dtype: torch.dtype = torch.int32):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} CUDA tensor")
    return t.data_ptr()


def _index_dtype(*tables: Optional[torch.Tensor]) -> torch.dtype:
    """int32 or int64: the one index type all given tables share."""
    kinds = {t.dtype for t in tables if t is not None}
    if len(kinds) != 1 or not kinds <= {torch.int32, torch.int64}:
        raise ValueError("index tables must all be int32 or all be int64")
    return kinds.pop()


def index64_workspace_size(tok: int, nseg: int) -> int:
    """Bytes at the front of an int64-table call's workspace (the narrowed tables)."""
    return int(lib().lora_index64_workspace_size(tok, nseg))


def _ws64(workspace: Optional[torch.Tensor], tok: int, nseg: int, num_adapters: int, device):
    """Workspace of an int64-table call: the caller's, or one allocated here
    (narrowed tables followed by the adapter-grouping scratch)."""
    if workspace is None:
        n = index64_workspace_size(tok, nseg) + workspace_size(tok, nseg, num_adapters)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=device)
    return workspace, _ws(workspace)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ws(workspace: Optional[torch.Tensor]):
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def _shrink_shapes(x: torch.Tensor, A_stack: torch.Tensor, out_r: torch.Tensor,
                   num_slices: int, rank: Optional[int]):
    """Host-side shape checks shared by the shrink entry points; returns
    (dtype code, ld_x, ld_out, tok, K, S, r, rs, L)."""
    dt = _dtype_code(x)
    if A_stack.dtype != x.dtype or out_r.dtype != x.dtype:
        raise TypeError("x, A_stack and out_r must share one element type")
    ld_x = _row_major(x, "x")
    ld_out = _row_major(out_r, "out_r")
    if not A_stack.is_contiguous():
        raise ValueError("A_stack must be contiguous")
    S = int(num_slices)
    if S < 1:
        raise ValueError("num_slices must be positive")
    if A_stack.dim() == 4:
        L, S4, rs, K = A_stack.shape
        if S4 != S:
            raise ValueError("A_stack slice dimension does not match num_slices")
    elif A_stack.dim() == 3:
        L, srs, K = A_stack.shape
        if srs % S:
            raise ValueError("A_stack rows are not a multiple of num_slices")
        rs = srs // S
    else:
        raise ValueError("A_stack must be [L, S*rs, K] or [L, S, rs, K]")
    tok, Kx = x.shape
    if Kx != K:
        raise ValueError(f"x has K={Kx}, A_stack has K={K}")
    r = rs if rank is None else int(rank)
    if out_r.shape[0] != tok:
        raise ValueError("out_r must have one row per token")
    if out_r.shape[1] < S * rs:
        raise ValueError(f"out_r must have at least S*rs = {S * rs} columns")
    return dt, ld_x, ld_out, tok, K, S, r, rs, L


def lora_shrink(x: torch.Tensor, A_stack: torch.Tensor, seg_indptr: torch.Tensor,
                weight_indices: torch.Tensor, permutation: Optional[torch.Tensor],
                out_r: torch.Tensor, *, num_slices: int, rank: Optional[int] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Shrink: out_r[i, q*rs+j] = sum_k x[perm[i], k] * A_stack[a, q*rs+j, k].

    x [tok, K] (unit inner stride), A_stack [L, S*rs, K] contiguous (or
    [L, S, rs, K]), out_r [tok, >= S*rs] (unit inner stride, sorted order).
    `rank` is the valid rank r <= rs (default rs).  The index tables are all
    int32, or all int64 (then lora_shrink_i64 runs, and a workspace is
    allocated when none is given)."""
    dt, ld_x, ld_out, tok, K, S, r, rs, L = _shrink_shapes(x, A_stack, out_r, num_slices, rank)
    nseg = seg_indptr.numel() - 1
    idt = _index_dtype(seg_indptr, weight_indices, permutation)
    if idt == torch.int64:
        # int64 tables: lora_shrink_i64 narrows them into the workspace first
        workspace, (ws, wsb) = _ws64(workspace, tok, nseg, L, x.device)
        fn, name = lib().lora_shrink_i64, "lora_shrink_i64"
    else:
        ws, wsb = _ws(workspace)
        fn, name = lib().lora_shrink, "lora_shrink"
    st = fn(x.data_ptr(), ld_x, A_stack.data_ptr(), _table(seg_indptr, "seg_indptr", dtype=idt),
            _table(weight_indices, "weight_indices", dtype=idt),
            _table(permutation, "permutation", True, dtype=idt), out_r.data_ptr(), ld_out,
            tok, K, S, r, rs, nseg, L, dt, ws, wsb, _stream(stream))
    if st != LORA_OK:
        raise LoraError(name, st)
    return out_r


def lora_expand(in_r: torch.Tensor, B_stack: torch.Tensor, seg_indptr: torch.Tensor,
                weight_indices: torch.Tensor, permutation: Optional[torch.Tensor],
                slice_offsets: Sequence[int], scalings: torch.Tensor, base_out: torch.Tensor,
                *, rank: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """Expand: base_out[perm[i], c] += scalings[a] * sum_j in_r[i, q*rs+j] * B_stack[a, c-off0, j].

    in_r [tok, >= S*rs] (sorted order), B_stack [L, N_tot, rs] contiguous,
    slice_offsets: S+1 host integers, scalings [L] fp32 CUDA, base_out
    [tok, >= off[S]] updated in place.  Index tables: all int32, or all int64
    (lora_expand_i64, as for lora_shrink)."""
    dt = _dtype_code(base_out)
    if in_r.dtype != base_out.dtype or B_stack.dtype != base_out.dtype:
        raise TypeError("in_r, B_stack and base_out must share one element type")
    if scalings.dtype != torch.float32 or not scalings.is_cuda or not scalings.is_contiguous():
        raise ValueError("scalings must be a contiguous fp32 CUDA tensor")
    ld_in = _row_major(in_r, "in_r")
    ld_base = _row_major(base_out, "base_out")
    if B_stack.dim() != 3 or not B_stack.is_contiguous():
        raise ValueError("B_stack must be a contiguous [L, N_tot, rs] tensor")
    L, n_tot, rs = B_stack.shape
    off = [int(v) for v in (slice_offsets.tolist() if torch.is_tensor(slice_offsets)
                            else slice_offsets)]
    S = len(off) - 1
    if S < 1 or S > MAX_SLICES:
        raise ValueError(f"need 2..{MAX_SLICES + 1} slice offsets")
    if off[-1] - off[0] != n_tot:
        raise ValueError("slice_offsets span does not match B_stack rows")
    r = rs if rank is None else int(rank)
    tok = base_out.shape[0]
    if in_r.shape[0] != tok:
        raise ValueError("in_r must have one row per token")
    nseg = seg_indptr.numel() - 1
    off_arr = (ctypes.c_int32 * len(off))(*off)
    idt = _index_dtype(seg_indptr, weight_indices, permutation)
    if idt == torch.int64:
        # int64 tables: lora_expand_i64 narrows them into the workspace first
        workspace, (ws, wsb) = _ws64(workspace, tok, nseg, L, base_out.device)
        fn, name = lib().lora_expand_i64, "lora_expand_i64"
    else:
        ws, wsb = _ws(workspace)
        fn, name = lib().lora_expand, "lora_expand"
    st = fn(in_r.data_ptr(), ld_in, B_stack.data_ptr(),
            _table(seg_indptr, "seg_indptr", dtype=idt),
            _table(weight_indices, "weight_indices", dtype=idt),
            _table(permutation, "permutation", True, dtype=idt),
            ctypes.cast(off_arr, ctypes.c_void_p), scalings.data_ptr(),
            base_out.data_ptr(), ld_base, tok, S, r, rs, nseg, L, dt, ws, wsb,
            _stream(stream))
    if st != LORA_OK:
        raise LoraError(name, st)
    return base_out


def lora_shrink_expand(x: torch.Tensor, A_stack: torch.Tensor, B_stack: torch.Tensor,
                       seg_indptr: torch.Tensor, weight_indices: torch.Tensor,
                       permutation: Optional[torch.Tensor], slice_offsets: Sequence[int],
                       scalings: torch.Tensor, out_r: torch.Tensor, base_out: torch.Tensor, *,
                       rank: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """The pair in one call: lora_shrink into out_r, then lora_expand of out_r
    into base_out (one fused launch for decode-sized batches).

    x [tok, K], A_stack [L, S*rs, K], B_stack [L, N_tot, rs], out_r
    [tok, >= S*rs] (written), base_out [tok, >= off[S]] (updated), int32 tables."""
    dt = _dtype_code(x)
    for t, n in ((A_stack, "A_stack"), (B_stack, "B_stack"), (out_r, "out_r"),
                 (base_out, "base_out")):
        if t.dtype != x.dtype:
            raise TypeError(f"{n} must have the element type of x")
    if scalings.dtype != torch.float32 or not scalings.is_cuda or not scalings.is_contiguous():
        raise ValueError("scalings must be a contiguous fp32 CUDA tensor")
    ld_x = _row_major(x, "x")
    ld_out = _row_major(out_r, "out_r")
    ld_base = _row_major(base_out, "base_out")
    if not A_stack.is_contiguous() or A_stack.dim() != 3:
        raise ValueError("A_stack must be a contiguous [L, S*rs, K] tensor")
    if B_stack.dim() != 3 or not B_stack.is_contiguous():
        raise ValueError("B_stack must be a contiguous [L, N_tot, rs] tensor")
    L, srs, K = A_stack.shape
    Lb, n_tot, rs = B_stack.shape
    off = [int(v) for v in (slice_offsets.tolist() if torch.is_tensor(slice_offsets)
                            else slice_offsets)]
    S = len(off) - 1
    if S < 1 or S > MAX_SLICES or srs != S * rs or Lb != L:
        raise ValueError("A_stack, B_stack and slice_offsets disagree on L, S or rs")
    if off[-1] - off[0] != n_tot:
        raise ValueError("slice_offsets span does not match B_stack rows")
    tok, Kx = x.shape
    if Kx != K or out_r.shape[0] != tok or base_out.shape[0] != tok:
        raise ValueError("x, out_r and base_out must have one row per token and K columns")
    r = rs if rank is None else int(rank)
    nseg = seg_indptr.numel() - 1
    off_arr = (ctypes.c_int32 * len(off))(*off)
    ws, wsb = _ws(workspace)
    st = lib().lora_shrink_expand(x.data_ptr(), ld_x, A_stack.data_ptr(), B_stack.data_ptr(),
                                  _table(seg_indptr, "seg_indptr"),
                                  _table(weight_indices, "weight_indices"),
                                  _table(permutation, "permutation", True),
                                  ctypes.cast(off_arr, ctypes.c_void_p), scalings.data_ptr(),
                                  out_r.data_ptr(), ld_out, base_out.data_ptr(), ld_base, tok,
                                  K, S, r, rs, nseg, L, dt, ws, wsb, _stream(stream))
    if st != LORA_OK:
        raise LoraError("lora_shrink_expand", st)
    return base_out


def lora_base_expand(x: torch.Tensor, W: torch.Tensor, in_r: torch.Tensor,
                     B_stack: torch.Tensor, seg_indptr: torch.Tensor,
                     weight_indices: torch.Tensor, permutation: Optional[torch.Tensor],
                     slice_offsets: Sequence[int], scalings: torch.Tensor, out: torch.Tensor, *,
                     rank: Optional[int] = None, stream=None) -> torch.Tensor:
    """The base projection with the expand folded in:
    out[perm[i], c] = rn(x[perm[i]] . W[c-off0] + s_a * in_r[i, q*rs:q*rs+r] . B_a[c-off0, :r])
    for the rows of every segment and the columns of the slices.

    x [tok, K], W [N_tot, >= K] (unit inner stride), in_r [tok, >= S*rs],
    B_stack [L, N_tot, rs], out [tok, >= off[S]] (written there only)."""
    dt = _dtype_code(x)
    for t, n in ((W, "W"), (in_r, "in_r"), (B_stack, "B_stack"), (out, "out")):
        if t.dtype != x.dtype:
            raise TypeError(f"{n} must have the element type of x")
    if scalings.dtype != torch.float32 or not scalings.is_cuda or not scalings.is_contiguous():
        raise ValueError("scalings must be a contiguous fp32 CUDA tensor")
    ld_x = _row_major(x, "x")
    ld_w = _row_major(W, "W")
    ld_in = _row_major(in_r, "in_r")
    ld_out = _row_major(out, "out")
    if B_stack.dim() != 3 or not B_stack.is_contiguous():
        raise ValueError("B_stack must be a contiguous [L, N_tot, rs] tensor")
    L, n_tot, rs = B_stack.shape
    off = [int(v) for v in (slice_offsets.tolist() if torch.is_tensor(slice_offsets)
                            else slice_offsets)]
    S = len(off) - 1
    if S < 1 or S > MAX_SLICES or off[-1] - off[0] != n_tot or W.shape[0] != n_tot:
        raise ValueError("slice_offsets, W and B_stack disagree on N_tot")
    tok, K = x.shape
    if W.shape[1] < K or in_r.shape[0] != tok or out.shape[0] != tok:
        raise ValueError("x, W, in_r and out disagree on tok or K")
    r = rs if rank is None else int(rank)
    nseg = seg_indptr.numel() - 1
    off_arr = (ctypes.c_int32 * len(off))(*off)
    st = lib().lora_base_expand(x.data_ptr(), ld_x, W.data_ptr(), ld_w, in_r.data_ptr(), ld_in,
                                B_stack.data_ptr(), _table(seg_indptr, "seg_indptr"),
                                _table(weight_indices, "weight_indices"),
                                _table(permutation, "permutation", True),
                                ctypes.cast(off_arr, ctypes.c_void_p), scalings.data_ptr(),
                                out.data_ptr(), ld_out, tok, K, S, r, rs, nseg, L, dt,
                                _stream(stream))
    if st != LORA_OK:
        raise LoraError("lora_base_expand", st)
    return out


def lora_validate(seg_indptr: torch.Tensor, weight_indices: torch.Tensor,
                  permutation: Optional[torch.Tensor], num_adapters: int, tok: int,
                  slice_offsets: Optional[Sequence[int]] = None, ld_base: int = 0,
                  stream=None) -> int:
    """Runs the device-side table checks and returns the LORA_BAD_* bitmask
    (0 = valid).  Synchronises the stream to read the result."""
    nseg = seg_indptr.numel() - 1
    dev = seg_indptr.device
    result = torch.empty(1, dtype=torch.int32, device=dev)
    ws = torch.empty(max(int(lib().lora_validate_workspace_size(tok)), 4), dtype=torch.uint8,
                     device=dev)
    if slice_offsets is not None:
        off = [int(v) for v in slice_offsets]
        S = len(off) - 1
        off_ptr = ctypes.cast((ctypes.c_int32 * len(off))(*off), ctypes.c_void_p)
    else:
        S, off_ptr = 1, None
    st = lib().lora_validate(_table(seg_indptr, "seg_indptr"), _table(weight_indices,
                                                                      "weight_indices"),
                             _table(permutation, "permutation", True), off_ptr, tok, nseg,
                             num_adapters, S, ld_base, result.data_ptr(), ws.data_ptr(),
                             ws.numel(), _stream(stream))
    if st != LORA_OK:
        raise LoraError("lora_validate", st)
    (torch.cuda.current_stream() if stream is None else stream).synchronize()
    return int(result.item())


STATIC_SCRATCH_BYTES = 1 << 20


def lora_shrink_static_scratch(x: torch.Tensor, A_stack: torch.Tensor, seg_indptr: torch.Tensor,
                               weight_indices: torch.Tensor, permutation: Optional[torch.Tensor],
                               out_r: torch.Tensor, *, num_slices: int,
                               rank: Optional[int] = None, stream=None) -> torch.Tensor:
    """lora_shrink for callers that cannot allocate device memory.

    Same arguments and result as :func:`lora_shrink` without a workspace: the
    library's own fixed 1 MiB device array holds the scratch.  Calls that
    overlap on the GPU race on that array, and problems whose workspace would
    exceed it raise LoraError (LORA_ERR_UNSUPPORTED)."""
    dt, ld_x, ld_out, tok, K, S, r, rs, L = _shrink_shapes(x, A_stack, out_r, num_slices, rank)
    f = lib().lora_shrink_static_scratch
    f.argtypes = [_P, _L, _P, _P, _P, _P, _P, _L] + [_I] * 8 + [_P]
    f.restype = _I
    st = f(x.data_ptr(), ld_x, A_stack.data_ptr(),
           _table(seg_indptr, "seg_indptr"), _table(weight_indices, "weight_indices"),
           _table(permutation, "permutation", True), out_r.data_ptr(), ld_out,
           tok, K, S, r, rs, seg_indptr.numel() - 1, L, dt, _stream(stream))
    if st != LORA_OK:
        raise LoraError("lora_shrink_static_scratch", st)
    return out_r


# ----------------------------------------------------------------------------
# identity-permutation ops of the same page (segments in token order)
# ----------------------------------------------------------------------------

def _fn(name, argtypes):
    f = getattr(lib(), name)
    f.argtypes = argtypes
    f.restype = _I
    return f


def _check(name, st):
    if st != LORA_OK:
        raise LoraError(name, st)


def sgemm_lora_a_fwd(x, A_stack, seg_indptr, weight_indices, out, *, num_slices=1, rank=None,
                     workspace=None, stream=None):
    """out[i, q*rs+j] = sum_k x[i, k] * A_stack[a, q*rs+j, k] (no permutation)."""
    L, srs, K = A_stack.shape
    S = int(num_slices)
    rs = srs // S
    r = rs if rank is None else int(rank)
    ws, wsb = _ws(workspace)
    f = _fn("lora_sgemm_a", [_P, _L, _P, _P, _P, _P, _L] + [_I] * 8 + [_P, _Z, _P])
    _check("lora_sgemm_a", f(x.data_ptr(), _row_major(x, "x"), A_stack.data_ptr(),
                             _table(seg_indptr, "seg_indptr"),
                             _table(weight_indices, "weight_indices"), out.data_ptr(),
                             _row_major(out, "out"), x.shape[0], K, S, r, rs,
                             seg_indptr.numel() - 1, L, _dtype_code(x), ws, wsb,
                             _stream(stream)))
    return out


def _expand_like(name, in_r, B_stack, seg_indptr, weight_indices, scalings, base_out, rank,
                 workspace, stream, extra_front=(), extra_types=(), n_arg=None):
    L, n_tot, rs = B_stack.shape
    r = rs if rank is None else int(rank)
    ws, wsb = _ws(workspace)
    types = [_P, _L, _P, _P, _P] + list(extra_types) + [_P, _P, _L, _I] + \
        ([_I] if n_arg is not None else []) + [_I] * 5 + [_P, _Z, _P]
    f = _fn(name, types)
    args = [in_r.data_ptr(), _row_major(in_r, "in_r"), B_stack.data_ptr(),
            _table(seg_indptr, "seg_indptr"), _table(weight_indices, "weight_indices")]
    args += list(extra_front)
    args += [scalings.data_ptr(), base_out.data_ptr(), _row_major(base_out, "base_out"),
             base_out.shape[0]]
    if n_arg is not None:
        args.append(n_arg)
    args += [r, rs, seg_indptr.numel() - 1, L, _dtype_code(base_out), ws, wsb, _stream(stream)]
    _check(name, f(*args))
    return base_out


def sgemm_lora_b_fwd(in_r, B_stack, seg_indptr, weight_indices, scalings, base_out, *, rank=None,
                     workspace=None, stream=None):
    """base_out[i, c] += scalings[a] * sum_j in_r[i, j] * B_stack[a, c, j] (one slice)."""
    return _expand_like("lora_sgemm_b", in_r, B_stack, seg_indptr, weight_indices, scalings,
                        base_out, rank, workspace, stream, n_arg=B_stack.shape[1])


def qkv_lora_b_fwd(in_r, B_stack, seg_indptr, weight_indices, qkv_offsets, scalings, base_out, *,
                   rank=None, workspace=None, stream=None):
    """Expand into three slices q, k, v at host column offsets qkv_offsets[0..3]."""
    off = [int(v) for v in qkv_offsets]
    if len(off) != 4:
        raise ValueError("qkv_offsets needs 4 entries")
    arr = (ctypes.c_int32 * 4)(*off)
    return _expand_like("lora_qkv_b", in_r, B_stack, seg_indptr, weight_indices, scalings,
                        base_out, rank, workspace, stream,
                        extra_front=[ctypes.cast(arr, ctypes.c_void_p)], extra_types=[_P])


def gate_up_lora_b_fwd(in_r, B_stack, seg_indptr, weight_indices, scalings, base_out, *,
                       rank=None, workspace=None, stream=None):
    """Expand into two equal slices (gate, up) at columns 0 and N."""
    return _expand_like("lora_gate_up_b", in_r, B_stack, seg_indptr, weight_indices, scalings,
                        base_out, rank, workspace, stream, n_arg=B_stack.shape[1] // 2)


def embedding_lora_a_fwd(ids, A_emb, seg_indptr, weight_indices, out, *, rank=None, stream=None):
    """out[i, j] = A_emb[a, j, ids[i]] for j < rank (A_emb [L, rs, V])."""
    L, rs, V = A_emb.shape
    r = rs if rank is None else int(rank)
    f = _fn("lora_embedding_a", [_P, _P, _P, _P, _P, _L] + [_I] * 7 + [_P])
    _check("lora_embedding_a", f(_table(ids, "ids"), A_emb.data_ptr(),
                                 _table(seg_indptr, "seg_indptr"),
                                 _table(weight_indices, "weight_indices"), out.data_ptr(),
                                 _row_major(out, "out"), ids.numel(), V, r, rs,
                                 seg_indptr.numel() - 1, L, _dtype_code(out), _stream(stream)))
    return out


# the chunked-SGMV pair under the names the pages use
chunked_sgmv_lora_shrink_fwd = lora_shrink
chunked_sgmv_lora_expand_fwd = lora_expand
